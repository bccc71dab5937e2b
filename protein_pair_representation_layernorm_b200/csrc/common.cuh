// common.cuh — shapes, argument blocks and small helpers shared by the kernels
// and the host code of the library.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace tri {

constexpr int kCz = 128;        // channels of a pair vector
constexpr int kHeads = 4;       // attention heads
constexpr int kD = 32;          // head width
constexpr int kHD = kHeads * kD;
constexpr float kLog2e = 1.4426950408889634f;
// Logit bias of a masked (or padding) key in the bf16 path.  Finite, so that
// every sum it enters (score + bias, minus the running offset) stays a finite
// number rather than an infinity; 2^(kMaskedLogit + s - m) is exactly 0 in
// fp32 for any finite score s and offset m, so the key gets probability 0.
constexpr float kMaskedLogit = -3.0e38f;

// Offset (in elements) of pair (i, j) of the problem inside Z / out.  The
// ending-node block reads and writes the pair representation through the
// swapped view: its pair (i, j) is Z[j][i].
__host__ __device__ __forceinline__ long long pair_offset(int orient, int N, int i, int j) {
  const long long a = orient == 0 ? i : j;
  const long long b = orient == 0 ? j : i;
  return (a * N + b) * kCz;
}

// ------------------------------------------------------------------ fp32 path
struct ProjArgsF32 {
  const float* Z;
  const uint8_t* mask;
  int N, orient, row0, rows;
  int write_qkvg, write_bias;
  const float *w_qkvg, *w_b, *gamma, *beta, *b_g;  // w_b pre-scaled by log2(e)
  float eps, q_scale;
  float *Q, *K, *V, *G, *bias;
  int ld_bias;
};

struct AttnArgsF32 {
  const float *Q, *K, *V, *bias;
  float* O;
  int N, rows, ld_bias;
};

struct GateArgsF32 {
  const float *Z, *O, *G, *w_o, *b_o;
  float* out;
  int N, orient, row0, rows;
};

// ------------------------------------------------------------------ bf16 path
struct ProjArgs {
  const __nv_bfloat16* Z;
  const uint8_t* mask;
  int N, orient, row0, rows;
  int write_qkv, write_bias;
  const uint8_t* w_img;  // [Wq; Wk; Wv] as the shared-memory image of the MMA B operand
  const float *w_b, *gamma, *beta;  // w_b pre-scaled by log2(e)
  float eps, q_scale;
  __nv_bfloat16 *Q, *K, *V, *bias;
  int ld_bias;
  // Z holds problem rows z_row0.. (a row slab; 0 for the whole tensor), and the
  // bias buffer holds, per head, bias_rows problem rows starting at bias_row0
  int z_row0, bias_row0, bias_rows;
  int debug_stall;  // fault injection: group 0 of CTA 0 never gets its first tile of Z
  int* status;
};

struct AttnArgs {
  __nv_bfloat16* O;  // [rows][H][N][d]
  float* lse;        // [rows][H][N]: each query's natural-log log-sum-exp, or nullptr
  int N, rows;
  int debug_stall;
  int* status;
};

struct GateArgs {
  const __nv_bfloat16 *Z, *O;
  // W_o / 2 and W_g / 2 (exact: a power-of-two scale) as shared-memory images of
  // the MMA B operand; the gate is recomputed from LayerNorm(z)
  const uint8_t* wo_img;
  const uint8_t* wg_img;
  const float *b_o, *b_g, *gamma, *beta;
  float eps;
  __nv_bfloat16* out;
  int N, orient, row0, rows;
  int z_row0;  // Z and out hold problem rows z_row0.. (a row slab; 0 for the whole tensor)
  int debug_stall;  // fault injection: the producer of CTA 0 withholds its first stage
  int* status;
};

// Device status word values (mirror the public codes).
constexpr int kStatusTimeout = -6;

__device__ __forceinline__ void report_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace tri
