// tri_attn.cu — host side of the C ABI declared in include/tri_attn.h, and the
// single translation unit that instantiates every kernel of the library.
//
// A forward call is three kernels on the caller's stream:
//   pair_ln_proj  (LayerNorm + Q/K/V/gate/bias, tcgen05)        HBM-bound
//   tri_attn_fwd  (online-softmax attention, tcgen05 + TMA)     tensor/ALU-bound
//   gate_out      (gate * o, output projection, residual)       HBM-bound
// (fp32 handles run the SIMT kernels of kernels_f32.cuh instead; the backward
// pass of the attention core runs the kernels of attn_bwd.cuh in fp32, or those
// of attn_bwd_tc.cuh on the tensor cores for bf16 operands).  The logit
// bias of every pair is needed by every row, so it is produced for all pairs
// before any attention runs; when the workspace for all rows exceeds the
// handle's limit, a bias-only pass runs first and the rest proceeds in row
// chunks.
#include "tri_attn.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <new>
#include <vector>

#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "common.cuh"
#include "gate_out.cuh"
#include "kernels_f32.cuh"
#include "merge.cuh"
#include "pair_ln_proj.cuh"
#include "sm100.cuh"
#include "tri_attn_fwd.cuh"

namespace {

using bf16 = __nv_bfloat16;
using tri::kCz;
using tri::kD;
using tri::kHD;
using tri::kHeads;

constexpr size_t kDefaultWorkspaceLimit = size_t(48) << 30;

bool log_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("TRIATTN_LOG");
    v = (e && e[0] && e[0] != '0') ? 1 : 0;
  }
  return v == 1;
}

#define TA_LOG(...)                                   \
  do {                                                \
    if (log_enabled()) {                              \
      std::fprintf(stderr, "[triattn] " __VA_ARGS__); \
      std::fprintf(stderr, "\n");                     \
    }                                                 \
  } while (0)

#define CUDA_TRY(expr)                                                     \
  do {                                                                     \
    cudaError_t err__ = (expr);                                            \
    if (err__ != cudaSuccess) {                                            \
      TA_LOG("%s failed: %s", #expr, cudaGetErrorString(err__));           \
      return err__ == cudaErrorMemoryAllocation ? TRI_ATTN_ERR_OOM          \
                                                : TRI_ATTN_ERR_CUDA;        \
    }                                                                      \
  } while (0)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 tensor map; dims/strides innermost first, strides in bytes (dims 1, 2).
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw,
                 uint32_t b2 = 1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) TA_LOG("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ weight packing
uint16_t f32_to_bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return static_cast<uint16_t>((u >> 16) | 0x40);  // NaN
  u += 0x7fffu + ((u >> 16) & 1u);  // round to nearest even
  return static_cast<uint16_t>(u >> 16);
}

float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Shared-memory image of a K-major bf16 MMA operand with 128-byte swizzle:
// rows n of 128 K-elements, split into two 64-element K slabs of rows x 128 B;
// the 16-byte chunk c of row n sits at chunk position c ^ (n % 8).
void pack_kmajor_sw128(const std::vector<uint16_t>& w, int rows, std::vector<uint16_t>& img) {
  img.assign(static_cast<size_t>(rows) * 128, 0);
  for (int n = 0; n < rows; ++n)
    for (int k = 0; k < 128; ++k) {
      const int slab = k / 64, c = (k % 64) / 8, e = k % 8;
      const size_t byte = static_cast<size_t>(slab) * rows * 128 + static_cast<size_t>(n) * 128 +
                          ((c ^ (n & 7)) * 16) + e * 2;
      img[byte / 2] = w[static_cast<size_t>(n) * 128 + k];
    }
}

int copy_to_host_f32(const void* dev, size_t n, tri_attn_dtype dt, std::vector<float>& out,
                     float fill) {
  out.assign(n, fill);
  if (!dev) return TRI_ATTN_OK;
  if (dt == TRI_ATTN_F32) {
    CUDA_TRY(cudaMemcpy(out.data(), dev, n * 4, cudaMemcpyDeviceToHost));
  } else {
    std::vector<uint16_t> tmp(n);
    CUDA_TRY(cudaMemcpy(tmp.data(), dev, n * 2, cudaMemcpyDeviceToHost));
    for (size_t k = 0; k < n; ++k) out[k] = bf16_bits_to_f32(tmp[k]);
  }
  return TRI_ATTN_OK;
}

// *dst is set whenever the allocation succeeded, also if the copy then fails.
template <class T>
int upload(const std::vector<T>& v, void** dst) {
  CUDA_TRY(cudaMalloc(dst, v.size() * sizeof(T)));
  CUDA_TRY(cudaMemcpy(*dst, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice));
  return TRI_ATTN_OK;
}

// cudaFuncSetAttribute applies to the current device only: record per device
// that the kernels' shared-memory limits were raised there.
constexpr int kMaxAttrDevices = 64;
std::mutex g_attrs_mutex;
bool g_attrs_set[kMaxAttrDevices] = {};

int set_kernel_attrs() {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxAttrDevices) return TRI_ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_attrs_mutex);
  if (g_attrs_set[dev]) return TRI_ATTN_OK;
  CUDA_TRY(cudaFuncSetAttribute(tri::plp::pair_ln_proj, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tri::plp::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(tri::attn::tri_attn_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tri::attn::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(tri::gout::gate_out, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tri::gout::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(tri::bwdtc::bwd_rows<tri::bwdtc::kDQ>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tri::bwdtc::RowsLayout<tri::bwdtc::kDQ>::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(tri::bwdtc::bwd_rows<tri::bwdtc::kDKDV>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tri::bwdtc::RowsLayout<tri::bwdtc::kDKDV>::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(tri::bwdtc::bwd_dbias_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tri::bwdtc::kDbSmemBytes));
  if (log_enabled()) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, tri::attn::tri_attn_fwd) == cudaSuccess)
      TA_LOG("tri_attn_fwd: regs %d, max threads %d, static smem %zu, local %zu", fa.numRegs,
             fa.maxThreadsPerBlock, fa.sharedSizeBytes, fa.localSizeBytes);
  }
  g_attrs_set[dev] = true;
  return TRI_ATTN_OK;
}

struct EventPair {
  cudaEvent_t a = nullptr, b = nullptr;
};

}  // namespace

struct tri_attn_handle {
  int device = 0;
  int num_sms = 148;
  tri_attn_dtype dtype = TRI_ATTN_BF16;
  float eps = 1e-5f;
  float q_scale = 0.f;
  // packed weights (device)
  void* w_qkvg = nullptr;  // bf16: [Wq; Wk; Wv] MMA B image (96 KB); f32: [Wq; Wk; Wv; Wg] [512][128]
  void* w_g = nullptr;     // bf16: Wg MMA B image (32 KB), for the gate recomputed in gate_out
  void* w_o = nullptr;     // bf16: MMA B image (32 KB);  f32: [128][128]
  float* w_b = nullptr;    // [H][c_z], times log2(e)
  float* gamma = nullptr;
  float* beta = nullptr;
  float* b_g = nullptr;
  float* b_o = nullptr;
  int* status = nullptr;   // device status word
  // workspace
  void* ws = nullptr;
  size_t ws_bytes = 0;
  size_t ws_limit = kDefaultWorkspaceLimit;
  // last forward, for tri_attn_debug_workspace
  void *q = nullptr, *k = nullptr, *v = nullptr, *g = nullptr, *bias = nullptr, *o = nullptr;
  int ld_bias = 0, rows_last = 0;
  // host-buffer entry points: a ring of device staging buffers (allocated on
  // first use), so that consecutive asynchronous calls overlap one call's
  // upload, another's computation and a third's download
  static constexpr int kRing = 3;
  void* stage[kRing] = {};
  size_t stage_bytes = 0;      // size of each staging buffer
  long long ring_next = 0;     // asynchronous calls issued
  cudaEvent_t slot_free[kRing] = {};  // recorded after the last download from the slot
  bool slot_pending[kRing] = {};
  uint8_t* stage_mask = nullptr;
  size_t stage_mask_bytes = 0;
  // the streams the uploads and the downloads run on, and the events that order
  // the computation after each uploaded piece and each download after the chunk
  // that produced it
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t chunk_ev = nullptr, up_ev = nullptr;
  static constexpr int kInRanges = 8;  // pieces of the upload, one event each
  cudaEvent_t in_ev[kInRanges] = {};
  // kernel timing
  std::vector<EventPair> ev[3];
  int ev_used[3] = {0, 0, 0};
};

namespace {

size_t esize(tri_attn_dtype dt) { return dt == TRI_ATTN_F32 ? 4 : 2; }

int ld_bias_for(int N) { return static_cast<int>(align_up(static_cast<size_t>(N), 64)); }

size_t bias_bytes(tri_attn_dtype dt, int N) {
  return align_up(static_cast<size_t>(kHeads) * N * ld_bias_for(N) * esize(dt), 256);
}

// Per-pair intermediates in the workspace: Q, K, V, O (H*d each), and for fp32
// handles also G; bf16 handles recompute the gate in gate_out from LayerNorm(z),
// so G never reaches memory.
int pair_buffers(tri_attn_dtype dt) { return dt == TRI_ATTN_F32 ? 5 : 4; }

size_t row_bytes(tri_attn_dtype dt, int N) {
  return static_cast<size_t>(N) * pair_buffers(dt) * kHD * esize(dt);
}

struct Layout {
  size_t q, k, v, g, o, bias, total;
  bool has_g;
};

Layout layout_for(tri_attn_dtype dt, int N, int rows) {
  Layout L{};
  const size_t per = align_up(static_cast<size_t>(rows) * N * kHD * esize(dt), 256);
  L.has_g = pair_buffers(dt) == 5;
  L.q = 0;
  L.k = per;
  L.v = 2 * per;
  L.g = L.has_g ? 3 * per : 0;
  L.o = (L.has_g ? 4 : 3) * per;
  L.bias = L.o + per;
  L.total = L.bias + bias_bytes(dt, N);
  return L;
}

// Grow the workspace to `bytes`.  The old buffer is released first, so a
// failed allocation leaves the handle holding no workspace (and nothing
// leaked); the next call allocates again.  fail_alloc injects that failure.
int ensure_workspace(tri_attn_handle* h, size_t bytes, bool fail_alloc = false) {
  if (h->ws_bytes >= bytes) return TRI_ATTN_OK;
  if (h->ws) CUDA_TRY(cudaFree(h->ws));
  h->ws = nullptr;
  h->ws_bytes = 0;
  if (fail_alloc) {
    TA_LOG("workspace allocation of %zu bytes failed (injected)", bytes);
    return TRI_ATTN_ERR_OOM;
  }
  CUDA_TRY(cudaMalloc(&h->ws, bytes));
  h->ws_bytes = bytes;
  return TRI_ATTN_OK;
}

EventPair& timing_slot(tri_attn_handle* h, int kernel) {
  int& used = h->ev_used[kernel];
  auto& vec = h->ev[kernel];
  if (used == static_cast<int>(vec.size())) {
    EventPair p;
    cudaEventCreate(&p.a);
    cudaEventCreate(&p.b);
    vec.push_back(p);
  }
  return vec[used++];
}

struct Timer {
  tri_attn_handle* h;
  cudaStream_t st;
  bool on;
  EventPair* p = nullptr;
  Timer(tri_attn_handle* h_, cudaStream_t s, bool on_, int kernel) : h(h_), st(s), on(on_) {
    if (on) {
      p = &timing_slot(h, kernel);
      cudaEventRecord(p->a, st);
    }
  }
  ~Timer() {
    if (on) cudaEventRecord(p->b, st);
  }
};

bool ranges_overlap(const void* a, const void* b, size_t bytes) {
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + bytes && y < x + bytes;
}

// A row slab of a starting-node block (bf16): Z and out hold problem rows
// row0 .. row0+nrows-1.  Phase 0 writes the slab's logit-bias rows to bias_io
// ([H][nrows][ld]); phase 1 runs the block on the slab with bias_io as the
// whole problem's bias ([H][N][ld]).
struct RowSlab {
  int row0, nrows, phase;
  void* bias_io;
};

// Optional per-chunk hook: at most max_rows problem rows per chunk (0 = no
// cap), and after(r0, nr) called once each chunk's output rows r0..r0+nr-1
// are enqueued (after its gate_out launch, on the call's stream).
struct ChunkHook {
  int max_rows = 0;
  std::function<int(int, int)> after;
  // bf16, unchunked calls only: the projection runs in launches of
  // proj_split_rows rows, each preceded by before_proj(r0, nr) (which may make
  // the stream wait for those rows' input)
  int proj_split_rows = 0;
  std::function<int(int, int)> before_proj;
};

int forward_impl(tri_attn_handle* h, const void* Z, int N, const uint8_t* mask, int orient,
                 void* out, cudaStream_t st, unsigned flags, const RowSlab* slab = nullptr,
                 const ChunkHook* hook = nullptr) {
  const tri_attn_dtype dt = h->dtype;
  const bool timed = (flags & TRI_ATTN_FLAG_TIME_KERNELS) != 0;
  const int ld = ld_bias_for(N);
  const int rbeg = slab ? slab->row0 : 0;           // problem rows of this call
  const int rend = slab ? slab->row0 + slab->nrows : N;
  const int zrows = rend - rbeg;                     // rows Z and out hold

  // rows per chunk under the workspace limit
  const size_t full = layout_for(dt, N, zrows).total;
  int rows = zrows;
  if (full > h->ws_limit) {
    const size_t fixed = bias_bytes(dt, N) + 6 * 256;
    if (h->ws_limit <= fixed) return TRI_ATTN_ERR_OOM;
    size_t fit = (h->ws_limit - fixed) / row_bytes(dt, N);
    fit = fit / tri::attn::kRows * tri::attn::kRows;
    if (fit < static_cast<size_t>(tri::attn::kRows)) return TRI_ATTN_ERR_OOM;
    rows = static_cast<int>(std::min<size_t>(fit, static_cast<size_t>(zrows)));
  }
  if (hook && hook->max_rows > 0 && hook->max_rows < rows) rows = hook->max_rows;
  const bool chunked = rows < zrows;
  const Layout L = layout_for(dt, N, rows);
  int rc = ensure_workspace(h, L.total, (flags & TRI_ATTN_FLAG_DEBUG_FAIL_ALLOC) != 0);
  if (rc != TRI_ATTN_OK) {
    h->q = h->k = h->v = h->g = h->o = h->bias = nullptr;  // the old workspace is gone
    h->rows_last = 0;
    return rc;
  }
  char* ws = static_cast<char*>(h->ws);
  h->q = ws + L.q;
  h->k = ws + L.k;
  h->v = ws + L.v;
  h->g = L.has_g ? ws + L.g : nullptr;
  h->o = ws + L.o;
  h->bias = (slab && slab->phase == 1) ? slab->bias_io : static_cast<void*>(ws + L.bias);
  h->ld_bias = ld;
  TA_LOG("forward N=%d orient=%d dtype=%d rows/chunk=%d ws=%zu", N, orient, static_cast<int>(dt),
         rows, L.total);

  if (dt == TRI_ATTN_F32) {
    const float* Zf = static_cast<const float*>(Z);
    float* outf = static_cast<float*>(out);
    const int pad = ld - N;
    if (pad > 0) {
      const long long tot = static_cast<long long>(kHeads) * N * pad;
      tri::f32::bias_pad_kernel<<<static_cast<unsigned>((tot + 255) / 256), 256, 0, st>>>(
          static_cast<float*>(h->bias), N, ld);
    }
    auto proj = [&](int row0, int nrows, int wq, int wb) {
      tri::ProjArgsF32 a{};
      a.Z = Zf;
      a.mask = mask;
      a.N = N;
      a.orient = orient;
      a.row0 = row0;
      a.rows = nrows;
      a.write_qkvg = wq;
      a.write_bias = wb;
      a.w_qkvg = static_cast<const float*>(h->w_qkvg);
      a.w_b = h->w_b;
      a.gamma = h->gamma;
      a.beta = h->beta;
      a.b_g = h->b_g;
      a.eps = h->eps;
      a.q_scale = h->q_scale;
      a.Q = static_cast<float*>(h->q);
      a.K = static_cast<float*>(h->k);
      a.V = static_cast<float*>(h->v);
      a.G = static_cast<float*>(h->g);
      a.bias = static_cast<float*>(h->bias);
      a.ld_bias = ld;
      const long long pairs = static_cast<long long>(nrows) * N;
      Timer tm(h, st, timed, 0);
      tri::f32::ln_proj_kernel<<<static_cast<unsigned>((pairs + tri::f32::kProjThreads - 1) /
                                                        tri::f32::kProjThreads),
                                 tri::f32::kProjThreads, 0, st>>>(a);
    };
    if (chunked) proj(0, N, 0, 1);
    for (int r0 = 0; r0 < N; r0 += rows) {
      const int nr = std::min(rows, N - r0);
      proj(r0, nr, 1, chunked ? 0 : 1);
      {
        tri::AttnArgsF32 a{};
        a.Q = static_cast<const float*>(h->q);
        a.K = static_cast<const float*>(h->k);
        a.V = static_cast<const float*>(h->v);
        a.bias = static_cast<const float*>(h->bias);
        a.O = static_cast<float*>(h->o);
        a.N = N;
        a.rows = nr;
        a.ld_bias = ld;
        const long long tot = static_cast<long long>(nr) * kHeads * N;
        Timer tm(h, st, timed, 1);
        tri::f32::attn_kernel<<<static_cast<unsigned>((tot + 127) / 128), 128, 0, st>>>(a);
      }
      {
        tri::GateArgsF32 a{};
        a.Z = Zf;
        a.O = static_cast<const float*>(h->o);
        a.G = static_cast<const float*>(h->g);
        a.w_o = static_cast<const float*>(h->w_o);
        a.b_o = h->b_o;
        a.out = outf;
        a.N = N;
        a.orient = orient;
        a.row0 = r0;
        a.rows = nr;
        const long long pairs = static_cast<long long>(nr) * N;
        Timer tm(h, st, timed, 2);
        tri::f32::gate_out_kernel<<<static_cast<unsigned>((pairs + tri::f32::kProjThreads - 1) /
                                                          tri::f32::kProjThreads),
                                    tri::f32::kProjThreads, 0, st>>>(a);
      }
      if (hook && hook->after) {
        CUDA_TRY(cudaGetLastError());
        const int hrc = hook->after(r0, nr);
        if (hrc != TRI_ATTN_OK) return hrc;
      }
    }
    h->rows_last = std::min(rows, N - (N - 1) / rows * rows);
    CUDA_TRY(cudaGetLastError());
    return TRI_ATTN_OK;
  }

  // ------------------------------------------------------------ bf16 path
  rc = set_kernel_attrs();
  if (rc != TRI_ATTN_OK) return rc;
  const bf16* Zb = static_cast<const bf16*>(Z);
  bf16* outb = static_cast<bf16*>(out);
  const int jtiles = (N + 127) / 128;
  auto proj = [&](int row0, int nrows, int wq, int wb, int out_off = 0) {
    const size_t off = static_cast<size_t>(out_off) * kHeads * N * kD;  // rows into Q/K/V
    tri::ProjArgs a{};
    a.Z = Zb;
    a.mask = mask;
    a.N = N;
    a.orient = orient;
    a.row0 = row0;
    a.rows = nrows;
    a.write_qkv = wq;
    a.write_bias = wb;
    a.w_img = static_cast<const uint8_t*>(h->w_qkvg);
    a.w_b = h->w_b;
    a.gamma = h->gamma;
    a.beta = h->beta;
    a.eps = h->eps;
    a.q_scale = h->q_scale;
    a.Q = static_cast<bf16*>(h->q) + off;
    a.K = static_cast<bf16*>(h->k) + off;
    a.V = static_cast<bf16*>(h->v) + off;
    a.bias = static_cast<bf16*>(slab && slab->phase == 0 ? slab->bias_io : h->bias);
    a.ld_bias = ld;
    a.z_row0 = rbeg;
    a.bias_row0 = slab && slab->phase == 0 ? rbeg : 0;
    a.bias_rows = slab && slab->phase == 0 ? zrows : N;
    a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL_PROJ) ? 1 : 0;
    a.status = h->status;
    const long long ntiles = static_cast<long long>(nrows) * jtiles;
    const unsigned grid = static_cast<unsigned>(
        std::min<long long>((ntiles + tri::plp::kGroupsPerCta - 1) / tri::plp::kGroupsPerCta, h->num_sms));
    // Z in boxes of 64 channels x 128 pairs: along j (starting node) or, through
    // the swapped view, along the rows of Z (ending node)
    CUtensorMap mz;
    const uint32_t zb1 = orient == 0 ? 128u : 1u, zb2 = orient == 0 ? 1u : 128u;
    if (!make_map_3d(&mz, Zb, kCz, N, zrows, kCz * 2, static_cast<uint64_t>(N) * kCz * 2, 64, zb1,
                     CU_TENSOR_MAP_SWIZZLE_128B, zb2))
      return cudaErrorInvalidValue;
    Timer tm(h, st, timed, 0);
    tri::plp::pair_ln_proj<<<grid, tri::plp::kThreads, tri::plp::kSmemBytes, st>>>(mz, a);
    return cudaGetLastError();
  };
  if (slab && slab->phase == 0) {  // the slab's bias rows only
    CUDA_TRY(proj(rbeg, zrows, 0, 1));
    CUDA_TRY(cudaGetLastError());
    return TRI_ATTN_OK;
  }
  const bool own_bias = slab == nullptr;
  if (chunked && own_bias) CUDA_TRY(proj(0, N, 0, 1));
  for (int r0 = rbeg; r0 < rend; r0 += rows) {
    const int nr = std::min(rows, rend - r0);
    if (!chunked && own_bias && hook && hook->before_proj && hook->proj_split_rows > 0) {
      for (int p0 = r0; p0 < r0 + nr; p0 += hook->proj_split_rows) {
        const int pn = std::min(hook->proj_split_rows, r0 + nr - p0);
        const int hrc = hook->before_proj(p0, pn);
        if (hrc != TRI_ATTN_OK) return hrc;
        CUDA_TRY(proj(p0, pn, 1, 1, p0 - r0));
      }
    } else {
      CUDA_TRY(proj(r0, nr, 1, (chunked || !own_bias) ? 0 : 1));
    }
    {
      CUtensorMap mq, mk, mv, mb;
      const uint64_t rh = static_cast<uint64_t>(nr) * kHeads;
      const uint64_t row_stride = static_cast<uint64_t>(N) * kD * 2;
      bool okm = make_map_3d(&mq, h->q, kD, N, rh, kD * 2, row_stride, kD, tri::attn::kBJ,
                             CU_TENSOR_MAP_SWIZZLE_64B) &&
                 make_map_3d(&mk, h->k, kD, N, rh, kD * 2, row_stride, kD, tri::attn::kBK,
                             CU_TENSOR_MAP_SWIZZLE_64B) &&
                 make_map_3d(&mv, h->v, kD, N, rh, kD * 2, row_stride, kD, tri::attn::kBK,
                             CU_TENSOR_MAP_SWIZZLE_64B) &&
                 make_map_3d(&mb, h->bias, ld, N, kHeads, static_cast<uint64_t>(ld) * 2,
                             static_cast<uint64_t>(N) * ld * 2, tri::attn::kBK, tri::attn::kBJ,
                             CU_TENSOR_MAP_SWIZZLE_128B);
      if (!okm) return TRI_ATTN_ERR_CUDA;
      tri::AttnArgs a{};
      a.O = static_cast<bf16*>(h->o);
      a.N = N;
      a.rows = nr;
      a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL) ? 1 : 0;
      a.status = h->status;
      dim3 grid(jtiles, (nr + tri::attn::kRows - 1) / tri::attn::kRows, kHeads);
      Timer tm(h, st, timed, 1);
      tri::attn::tri_attn_fwd<<<grid, tri::attn::kThreads, tri::attn::kSmemBytes, st>>>(mq, mk, mv, mb,
                                                                                 a);
      CUDA_TRY(cudaGetLastError());
    }
    {
      // o: this chunk's workspace (head-major); z, out: the pair tensor, boxes of 128 pairs
      // along j (starting node) or, through the swapped view, along the rows of Z
      CUtensorMap mo, mz, mout;
      const uint64_t rowb = static_cast<uint64_t>(N) * kCz * 2;
      const uint32_t zb1 = orient == 0 ? 128u : 1u, zb2 = orient == 0 ? 1u : 128u;
      bool okm =
          make_map_3d(&mo, h->o, kD, N, static_cast<uint64_t>(nr) * kHeads, kD * 2,
                      static_cast<uint64_t>(N) * kD * 2, kD, 128, CU_TENSOR_MAP_SWIZZLE_64B) &&
          make_map_3d(&mz, Zb, kCz, N, zrows, kCz * 2, rowb, 64, zb1, CU_TENSOR_MAP_SWIZZLE_128B,
                      zb2) &&
          make_map_3d(&mout, outb, kCz, N, zrows, kCz * 2, rowb, 64, zb1,
                      CU_TENSOR_MAP_SWIZZLE_128B, zb2);
      if (!okm) return TRI_ATTN_ERR_CUDA;
      tri::GateArgs a{};
      a.Z = Zb;
      a.O = static_cast<const bf16*>(h->o);
      a.wo_img = static_cast<const uint8_t*>(h->w_o);
      a.wg_img = static_cast<const uint8_t*>(h->w_g);
      a.b_o = h->b_o;
      a.b_g = h->b_g;
      a.gamma = h->gamma;
      a.beta = h->beta;
      a.eps = h->eps;
      a.out = outb;
      a.N = N;
      a.orient = orient;
      a.row0 = r0;
      a.rows = nr;
      a.z_row0 = rbeg;
      a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL_GATE) ? 1 : 0;
      a.status = h->status;
      const long long ntiles = static_cast<long long>(nr) * jtiles;
      const unsigned grid = static_cast<unsigned>(std::min<long long>(ntiles, h->num_sms));
      Timer tm(h, st, timed, 2);
      tri::gout::gate_out<<<grid, tri::gout::kThreads, tri::gout::kSmemBytes, st>>>(mo, mz, mout, a);
      CUDA_TRY(cudaGetLastError());
    }
    if (hook && hook->after) {
      const int hrc = hook->after(r0, nr);
      if (hrc != TRI_ATTN_OK) return hrc;
    }
  }
  h->rows_last = zrows - (zrows - 1) / rows * rows;
  CUDA_TRY(cudaGetLastError());
  return TRI_ATTN_OK;
}

int read_status(tri_attn_handle* h, cudaStream_t st) {
  int s = 0;
  CUDA_TRY(cudaMemcpyAsync(&s, h->status, sizeof(int), cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (s != 0) CUDA_TRY(cudaMemsetAsync(h->status, 0, sizeof(int), st));
  CUDA_TRY(cudaStreamSynchronize(st));
  return s;
}

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return TRI_ATTN_ERR_NO_DEVICE;
  }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return TRI_ATTN_ERR_NO_DEVICE;
  }
  return major == 10 ? TRI_ATTN_OK : TRI_ATTN_ERR_NO_DEVICE;
}

}  // namespace

extern "C" {

const char* tri_attn_status_string(int code) {
  switch (code) {
    case TRI_ATTN_OK: return "ok";
    case TRI_ATTN_ERR_INVALID_ARG: return "invalid argument";
    case TRI_ATTN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case TRI_ATTN_ERR_ALIAS: return "out partially overlaps Z";
    case TRI_ATTN_ERR_OOM: return "out of memory";
    case TRI_ATTN_ERR_CUDA: return "CUDA error";
    case TRI_ATTN_ERR_TIMEOUT: return "device wait timed out";
    case TRI_ATTN_ERR_NO_DEVICE: return "no sm_100 device";
    default: return "unknown status";
  }
}

size_t tri_attn_workspace_bytes(tri_attn_dtype dtype, int N) {
  if (N < 1 || (dtype != TRI_ATTN_F32 && dtype != TRI_ATTN_BF16)) return 0;
  return layout_for(dtype, N, N).total;
}

int tri_attn_create(const tri_attn_params* p, tri_attn_handle** out) {
  if (!p || !out) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->dtype != TRI_ATTN_F32 && p->dtype != TRI_ATTN_BF16) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->c_z != kCz || p->n_heads != kHeads || p->head_dim != kD) return TRI_ATTN_ERR_UNSUPPORTED;
  if (!p->ln_gamma || !p->ln_beta || !p->w_q || !p->w_k || !p->w_v || !p->w_g || !p->w_b ||
      !p->w_o)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (!(p->ln_eps >= 0.f) || !std::isfinite(p->ln_eps)) return TRI_ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;

  tri_attn_handle* h = new (std::nothrow) tri_attn_handle();
  if (!h) return TRI_ATTN_ERR_OOM;
  auto fail = [&](int code) {
    tri_attn_destroy(h);
    return code;
  };
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) !=
          cudaSuccess) {
    cudaGetLastError();
    return fail(TRI_ATTN_ERR_CUDA);
  }
  h->dtype = p->dtype;
  h->eps = p->ln_eps;
  h->q_scale = tri::kLog2e / std::sqrt(static_cast<float>(kD));

  std::vector<float> wq, wk, wv, wg, wb, wo, gamma, beta, bg, bo;
  const tri_attn_dtype dt = p->dtype;
  if ((rc = copy_to_host_f32(p->w_q, kHD * kCz, dt, wq, 0.f)) ||
      (rc = copy_to_host_f32(p->w_k, kHD * kCz, dt, wk, 0.f)) ||
      (rc = copy_to_host_f32(p->w_v, kHD * kCz, dt, wv, 0.f)) ||
      (rc = copy_to_host_f32(p->w_g, kHD * kCz, dt, wg, 0.f)) ||
      (rc = copy_to_host_f32(p->w_b, kHeads * kCz, dt, wb, 0.f)) ||
      (rc = copy_to_host_f32(p->w_o, kCz * kHD, dt, wo, 0.f)) ||
      (rc = copy_to_host_f32(p->ln_gamma, kCz, dt, gamma, 1.f)) ||
      (rc = copy_to_host_f32(p->ln_beta, kCz, dt, beta, 0.f)) ||
      (rc = copy_to_host_f32(p->b_g, kHD, dt, bg, 0.f)) ||
      (rc = copy_to_host_f32(p->b_o, kCz, dt, bo, 0.f)))
    return fail(rc);
  for (float& x : wb) x *= tri::kLog2e;

  if (dt == TRI_ATTN_BF16) {
    // [Wq; Wk; Wv] as 384 K-major rows, Wg / 2 and Wo / 2 as 128 K-major rows each,
    // all in the shared-memory image the tcgen05 B operand reads (bf16 values kept
    // exactly: halving a bf16 number is exact).  gate_out works with
    // t = (Wg x + bg) / 2 and a = 2 g o = (1 + tanh t) o, so the halves cancel.
    std::vector<uint16_t> w384(384 * 128), wg128(128 * 128), w128(128 * 128), img;
    const std::vector<float>* parts[3] = {&wq, &wk, &wv};
    for (int part = 0; part < 3; ++part)
      for (int n = 0; n < kHD; ++n)
        for (int c = 0; c < kCz; ++c)
          w384[(part * kHD + n) * 128 + c] = f32_to_bf16_bits((*parts[part])[n * kCz + c]);
    for (int n = 0; n < kHD; ++n)
      for (int c = 0; c < kCz; ++c) wg128[n * 128 + c] = f32_to_bf16_bits(0.5f * wg[n * kCz + c]);
    for (int n = 0; n < kCz; ++n)
      for (int c = 0; c < kHD; ++c) w128[n * 128 + c] = f32_to_bf16_bits(0.5f * wo[n * kHD + c]);
    pack_kmajor_sw128(w384, 384, img);
    if ((rc = upload(img, &h->w_qkvg))) return fail(rc);
    pack_kmajor_sw128(wg128, 128, img);
    if ((rc = upload(img, &h->w_g))) return fail(rc);
    pack_kmajor_sw128(w128, 128, img);
    if ((rc = upload(img, &h->w_o))) return fail(rc);
  } else {
    std::vector<float> w512(512 * 128);
    std::memcpy(&w512[0], wq.data(), kHD * kCz * 4);
    std::memcpy(&w512[kHD * kCz], wk.data(), kHD * kCz * 4);
    std::memcpy(&w512[2 * kHD * kCz], wv.data(), kHD * kCz * 4);
    std::memcpy(&w512[3 * kHD * kCz], wg.data(), kHD * kCz * 4);
    if ((rc = upload(w512, &h->w_qkvg))) return fail(rc);
    if ((rc = upload(wo, &h->w_o))) return fail(rc);
  }
  // the handle owns each buffer as soon as it is allocated, so a failure part
  // way through is cleaned up by tri_attn_destroy
  auto upload_to = [&](const std::vector<float>& v, float** field) {
    void* t = nullptr;
    const int r = upload(v, &t);
    *field = static_cast<float*>(t);
    return r;
  };
  if ((rc = upload_to(wb, &h->w_b)) || (rc = upload_to(gamma, &h->gamma)) ||
      (rc = upload_to(beta, &h->beta)) || (rc = upload_to(bg, &h->b_g)) ||
      (rc = upload_to(bo, &h->b_o)))
    return fail(rc);
  if (cudaMalloc(&h->status, sizeof(int)) != cudaSuccess) return fail(TRI_ATTN_ERR_OOM);
  if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return fail(TRI_ATTN_ERR_CUDA);
  *out = h;
  return TRI_ATTN_OK;
}

int tri_attn_forward(tri_attn_handle* h, const void* Z, int N, const uint8_t* mask,
                     tri_attn_orientation orientation, void* out, void* stream, unsigned flags) {
  if (!h || !Z || !out || N < 1) return TRI_ATTN_ERR_INVALID_ARG;
  if (orientation != TRI_ATTN_STARTING && orientation != TRI_ATTN_ENDING)
    return TRI_ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Z) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
    return TRI_ATTN_ERR_INVALID_ARG;
  if (N > 46340) return TRI_ATTN_ERR_UNSUPPORTED;  // N*N pairs must fit in int32 per row index math
  const size_t bytes = static_cast<size_t>(N) * N * kCz * esize(h->dtype);
  if (Z != out && ranges_overlap(Z, out, bytes)) return TRI_ATTN_ERR_ALIAS;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = forward_impl(h, Z, N, mask, static_cast<int>(orientation), out, st, flags);
  if (rc != TRI_ATTN_OK) return rc;
  if (flags & TRI_ATTN_FLAG_SYNC) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return TRI_ATTN_ERR_CUDA;
    return read_status(h, st);
  }
  return TRI_ATTN_OK;
}

namespace {
// Shared checks of the two row-slab entry points.
int check_rows_args(tri_attn_handle* h, const void* Z_rows, int N, int row0, int nrows,
                    const void* bias, const void* out_rows) {
  if (!h || !Z_rows || !bias || N < 1 || row0 < 0 || nrows < 1 || row0 > N - nrows)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (h->dtype != TRI_ATTN_BF16) return TRI_ATTN_ERR_UNSUPPORTED;
  if (N > 46340) return TRI_ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(Z_rows) & 15) || (reinterpret_cast<uintptr_t>(bias) & 15) ||
      (out_rows && (reinterpret_cast<uintptr_t>(out_rows) & 15)))
    return TRI_ATTN_ERR_INVALID_ARG;
  return TRI_ATTN_OK;
}

int finish_call(tri_attn_handle* h, cudaStream_t st, unsigned flags) {
  if (flags & TRI_ATTN_FLAG_SYNC) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return TRI_ATTN_ERR_CUDA;
    return read_status(h, st);
  }
  return TRI_ATTN_OK;
}
}  // namespace

int tri_attn_bias_ld(int N) { return N < 1 ? 0 : ld_bias_for(N); }

int tri_attn_rows_bias(tri_attn_handle* h, const void* Z_rows, int N, int row0, int nrows,
                       const uint8_t* mask, void* bias_rows, void* stream, unsigned flags) {
  int rc = check_rows_args(h, Z_rows, N, row0, nrows, bias_rows, nullptr);
  if (rc != TRI_ATTN_OK) return rc;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const RowSlab slab{row0, nrows, 0, bias_rows};
  rc = forward_impl(h, Z_rows, N, mask, TRI_ATTN_STARTING, nullptr, st, flags, &slab);
  if (rc != TRI_ATTN_OK) return rc;
  return finish_call(h, st, flags);
}

int tri_attn_rows_forward(tri_attn_handle* h, const void* Z_rows, int N, int row0, int nrows,
                          const uint8_t* mask, const void* bias_all, void* out_rows,
                          void* stream, unsigned flags) {
  int rc = check_rows_args(h, Z_rows, N, row0, nrows, bias_all, out_rows);
  if (rc != TRI_ATTN_OK) return rc;
  if (!out_rows) return TRI_ATTN_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(nrows) * N * kCz * 2;
  if (Z_rows != out_rows && ranges_overlap(Z_rows, out_rows, bytes)) return TRI_ATTN_ERR_ALIAS;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const RowSlab slab{row0, nrows, 1, const_cast<void*>(bias_all)};
  rc = forward_impl(h, Z_rows, N, mask, TRI_ATTN_STARTING, out_rows, st, flags, &slab);
  if (rc != TRI_ATTN_OK) return rc;
  return finish_call(h, st, flags);
}

}  // extern "C"

namespace {

// Wait for every upload and download of the host-buffer entry points.
int host_drain(tri_attn_handle* h) {
  const cudaError_t a = h->copy_in ? cudaStreamSynchronize(h->copy_in) : cudaSuccess;
  const cudaError_t b = h->copy_out ? cudaStreamSynchronize(h->copy_out) : cudaSuccess;
  for (bool& p : h->slot_pending) p = false;
  return a == cudaSuccess && b == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

// The host-buffer forward, enqueued on three streams: uploads on copy_in, the
// blocks on `st`, downloads on copy_out, ordered by events.  `slot` picks the
// device staging buffer; the upload into it waits for the slot's previous
// download.  Returns once everything is enqueued.
int host_enqueue(tri_attn_handle* h, const void* Z_host, int N, const uint8_t* mask_host,
                 const int* orientations, int n_orientations, void* out_host, cudaStream_t st,
                 unsigned flags, int slot) {
  const size_t bytes = static_cast<size_t>(N) * N * kCz * esize(h->dtype);
  if (!h->copy_in) CUDA_TRY(cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking));
  if (!h->copy_out) CUDA_TRY(cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking));
  if (!h->chunk_ev) CUDA_TRY(cudaEventCreateWithFlags(&h->chunk_ev, cudaEventDisableTiming));
  if (!h->up_ev) CUDA_TRY(cudaEventCreateWithFlags(&h->up_ev, cudaEventDisableTiming));
  for (int k = 0; k < tri_attn_handle::kRing; ++k)
    if (!h->slot_free[k])
      CUDA_TRY(cudaEventCreateWithFlags(&h->slot_free[k], cudaEventDisableTiming));
  if (h->stage_bytes < bytes) {
    // a larger problem: every staging buffer is reallocated once nothing uses it
    const int rc = host_drain(h);
    if (rc != TRI_ATTN_OK) return rc;
    CUDA_TRY(cudaStreamSynchronize(st));
    for (void*& b : h->stage) {
      if (b) cudaFree(b);
      b = nullptr;
    }
    h->stage_bytes = bytes;
  }
  if (!h->stage[slot]) {
    const cudaError_t e = cudaMalloc(&h->stage[slot], h->stage_bytes);
    if (e != cudaSuccess) {
      h->stage[slot] = nullptr;
      return e == cudaErrorMemoryAllocation ? TRI_ATTN_ERR_OOM : TRI_ATTN_ERR_CUDA;
    }
  }
  char* stage = static_cast<char*>(h->stage[slot]);
  const uint8_t* dmask = nullptr;
  if (mask_host) {
    // on `st`: ordered after the previous call's blocks, which read the buffer
    if (h->stage_mask_bytes < static_cast<size_t>(N)) {
      CUDA_TRY(cudaStreamSynchronize(st));
      if (h->stage_mask) cudaFree(h->stage_mask);
      h->stage_mask = nullptr;
      h->stage_mask_bytes = 0;
      CUDA_TRY(cudaMalloc(&h->stage_mask, static_cast<size_t>(N)));
      h->stage_mask_bytes = N;
    }
    CUDA_TRY(cudaMemcpyAsync(h->stage_mask, mask_host, N, cudaMemcpyHostToDevice, st));
    dmask = h->stage_mask;
  }
  // the slot's previous download must be complete before the upload overwrites it
  if (h->slot_pending[slot]) CUDA_TRY(cudaStreamWaitEvent(h->copy_in, h->slot_free[slot], 0));
  const size_t es = esize(h->dtype), pair_b = kCz * es, row_b = static_cast<size_t>(N) * pair_b;
  // With two or more blocks and an unchunked bf16 first block, Z goes up in
  // kInRanges pieces (rows of Z when the first block is a starting node,
  // columns when it is an ending node), and the first block's projection of
  // each piece starts as soon as that piece has arrived; everything after the
  // projection needs the whole bias and waits for all pieces.
  const bool pipelined_in = n_orientations >= 2 && h->dtype == TRI_ATTN_BF16 &&
                            layout_for(h->dtype, N, N).total <= h->ws_limit &&
                            N >= tri_attn_handle::kInRanges;
  const int in_split = (N + tri_attn_handle::kInRanges - 1) / tri_attn_handle::kInRanges;
  if (pipelined_in) {
    const int first = orientations[0];
    for (int c = 0; c < tri_attn_handle::kInRanges; ++c) {
      if (!h->in_ev[c]) CUDA_TRY(cudaEventCreateWithFlags(&h->in_ev[c], cudaEventDisableTiming));
      const int r0 = c * in_split, nr = std::min(in_split, N - r0);
      if (nr <= 0) continue;
      const char* src = static_cast<const char*>(Z_host);
      if (first == TRI_ATTN_STARTING) {
        CUDA_TRY(cudaMemcpyAsync(stage + r0 * row_b, src + r0 * row_b, nr * row_b,
                                 cudaMemcpyHostToDevice, h->copy_in));
      } else {  // columns r0 .. r0+nr-1 of every row
        CUDA_TRY(cudaMemcpy2DAsync(stage + r0 * pair_b, row_b, src + r0 * pair_b, row_b,
                                   nr * pair_b, static_cast<size_t>(N), cudaMemcpyHostToDevice,
                                   h->copy_in));
      }
      CUDA_TRY(cudaEventRecord(h->in_ev[c], h->copy_in));
    }
  } else {
    CUDA_TRY(cudaMemcpyAsync(stage, Z_host, bytes, cudaMemcpyHostToDevice, h->copy_in));
    CUDA_TRY(cudaEventRecord(h->up_ev, h->copy_in));
    CUDA_TRY(cudaStreamWaitEvent(st, h->up_ev, 0));
  }
  if (n_orientations == 0) {
    CUDA_TRY(cudaStreamWaitEvent(h->copy_out, h->up_ev, 0));
    CUDA_TRY(cudaMemcpyAsync(out_host, stage, bytes, cudaMemcpyDeviceToHost, h->copy_out));
    CUDA_TRY(cudaEventRecord(h->slot_free[slot], h->copy_out));
    h->slot_pending[slot] = true;
    return TRI_ATTN_OK;
  }
  for (int t = 0; t + 1 < n_orientations; ++t) {
    ChunkHook in_hook;
    if (t == 0 && pipelined_in) {
      in_hook.proj_split_rows = in_split;
      in_hook.before_proj = [&](int r0, int) -> int {
        CUDA_TRY(cudaStreamWaitEvent(st, h->in_ev[r0 / in_split], 0));
        return TRI_ATTN_OK;
      };
    }
    const int rc = forward_impl(h, stage, N, dmask, orientations[t], stage, st,
                                flags & ~TRI_ATTN_FLAG_SYNC, nullptr,
                                (t == 0 && pipelined_in) ? &in_hook : nullptr);
    if (rc != TRI_ATTN_OK) return rc;
  }
  // The last block runs in row chunks (about 8), and each chunk's output goes
  // back to the host on copy_out as soon as its gate_out has run, while the
  // later chunks compute: a chunk's output region (rows of Z for the starting
  // node, columns for the ending node) is final once written, and no later
  // chunk reads or writes it.
  const int last = orientations[n_orientations - 1];
  ChunkHook hook;
  hook.max_rows = std::max(tri::attn::kRows,
                           ((N + 7) / 8 + tri::attn::kRows - 1) / tri::attn::kRows * tri::attn::kRows);
  hook.after = [&](int r0, int nr) -> int {
    CUDA_TRY(cudaEventRecord(h->chunk_ev, st));
    CUDA_TRY(cudaStreamWaitEvent(h->copy_out, h->chunk_ev, 0));
    char* dst = static_cast<char*>(out_host);
    if (last == TRI_ATTN_STARTING) {
      CUDA_TRY(cudaMemcpyAsync(dst + r0 * row_b, stage + r0 * row_b, nr * row_b,
                               cudaMemcpyDeviceToHost, h->copy_out));
    } else {  // columns r0 .. r0+nr-1 of every row
      CUDA_TRY(cudaMemcpy2DAsync(dst + r0 * pair_b, row_b, stage + r0 * pair_b, row_b,
                                 nr * pair_b, static_cast<size_t>(N), cudaMemcpyDeviceToHost,
                                 h->copy_out));
    }
    return TRI_ATTN_OK;
  };
  const int rc = forward_impl(h, stage, N, dmask, last, stage, st, flags & ~TRI_ATTN_FLAG_SYNC,
                              nullptr, &hook);
  if (rc != TRI_ATTN_OK) return rc;
  CUDA_TRY(cudaEventRecord(h->slot_free[slot], h->copy_out));
  h->slot_pending[slot] = true;
  return TRI_ATTN_OK;
}

int host_check(tri_attn_handle* h, const void* Z_host, int N, const int* orientations,
               int n_orientations, const void* out_host) {
  if (!h || !Z_host || !out_host || N < 1 || n_orientations < 0 ||
      (n_orientations > 0 && !orientations))
    return TRI_ATTN_ERR_INVALID_ARG;
  for (int t = 0; t < n_orientations; ++t)
    if (orientations[t] != TRI_ATTN_STARTING && orientations[t] != TRI_ATTN_ENDING)
      return TRI_ATTN_ERR_INVALID_ARG;
  if (N > 46340) return TRI_ATTN_ERR_UNSUPPORTED;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  return TRI_ATTN_OK;
}

}  // namespace

extern "C" {

int tri_attn_forward_host(tri_attn_handle* h, const void* Z_host, int N, const uint8_t* mask_host,
                          const int* orientations, int n_orientations, void* out_host,
                          void* stream, unsigned flags) {
  int rc = host_check(h, Z_host, N, orientations, n_orientations, out_host);
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = host_enqueue(h, Z_host, N, mask_host, orientations, n_orientations, out_host, st, flags,
                    0);
  const int rd = host_drain(h);
  if (rc != TRI_ATTN_OK) {
    cudaStreamSynchronize(st);
    return rc;
  }
  if (rd != TRI_ATTN_OK) return rd;
  CUDA_TRY(cudaStreamSynchronize(st));
  return read_status(h, st);
}

int tri_attn_forward_host_async(tri_attn_handle* h, const void* Z_host, int N,
                                const uint8_t* mask_host, const int* orientations,
                                int n_orientations, void* out_host, void* stream,
                                unsigned flags) {
  int rc = host_check(h, Z_host, N, orientations, n_orientations, out_host);
  if (rc != TRI_ATTN_OK) return rc;
  const int slot = static_cast<int>(h->ring_next % tri_attn_handle::kRing);
  rc = host_enqueue(h, Z_host, N, mask_host, orientations, n_orientations, out_host,
                    static_cast<cudaStream_t>(stream), flags, slot);
  if (rc == TRI_ATTN_OK) ++h->ring_next;
  return rc;
}

int tri_attn_host_wait(tri_attn_handle* h) {
  if (!h) return TRI_ATTN_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  const int rc = host_drain(h);
  if (rc != TRI_ATTN_OK) return rc;
  // every download follows the blocks that produced it, so the status word is
  // final once copy_out has drained
  return read_status(h, h->copy_out ? h->copy_out : nullptr);
}

int tri_attn_get_status(tri_attn_handle* h, void* stream) {
  if (!h) return TRI_ATTN_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  return read_status(h, static_cast<cudaStream_t>(stream));
}

int tri_attn_kernel_times(tri_attn_handle* h, float ms[3], int launches[3]) {
  if (!h || !ms) return TRI_ATTN_ERR_INVALID_ARG;
  for (int k = 0; k < 3; ++k) {
    float tot = 0.f;
    for (int u = 0; u < h->ev_used[k]; ++u) {
      float t = 0.f;
      CUDA_TRY(cudaEventSynchronize(h->ev[k][u].b));
      CUDA_TRY(cudaEventElapsedTime(&t, h->ev[k][u].a, h->ev[k][u].b));
      tot += t;
    }
    ms[k] = tot;
    if (launches) launches[k] = h->ev_used[k];
    h->ev_used[k] = 0;
  }
  return TRI_ATTN_OK;
}

int tri_attn_set_workspace_limit(tri_attn_handle* h, size_t bytes) {
  if (!h) return TRI_ATTN_ERR_INVALID_ARG;
  h->ws_limit = bytes ? bytes : kDefaultWorkspaceLimit;
  return TRI_ATTN_OK;
}

int tri_attn_debug_workspace(tri_attn_handle* h, void** q, void** k, void** v, void** g,
                             void** bias, void** o, int* ld_bias, int* rows) {
  if (!h) return TRI_ATTN_ERR_INVALID_ARG;
  if (q) *q = h->q;
  if (k) *k = h->k;
  if (v) *v = h->v;
  if (g) *g = h->g;
  if (bias) *bias = h->bias;
  if (o) *o = h->o;
  if (ld_bias) *ld_bias = h->ld_bias;
  if (rows) *rows = h->rows_last;
  return TRI_ATTN_OK;
}

int tri_attn_destroy(tri_attn_handle* h) {
  if (!h) return TRI_ATTN_OK;
  cudaSetDevice(h->device);
  if (h->copy_in) cudaStreamSynchronize(h->copy_in);
  if (h->copy_out) cudaStreamSynchronize(h->copy_out);
  void* ptrs[] = {h->w_qkvg, h->w_g,  h->w_o,      h->w_b,      h->gamma,    h->beta,
                  h->b_g,    h->b_o,  h->status,   h->ws,       h->stage[0], h->stage[1],
                  h->stage[2], h->stage_mask};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  for (auto& vec : h->ev)
    for (auto& p : vec) {
      if (p.a) cudaEventDestroy(p.a);
      if (p.b) cudaEventDestroy(p.b);
    }
  if (h->chunk_ev) cudaEventDestroy(h->chunk_ev);
  if (h->up_ev) cudaEventDestroy(h->up_ev);
  for (cudaEvent_t e : h->in_ev)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : h->slot_free)
    if (e) cudaEventDestroy(e);
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  delete h;
  return TRI_ATTN_OK;
}

}  // extern "C"

// ===================================================================== no-alloc
// Entry point for callers that cannot allocate device memory (see
// tri_attn_forward_noalloc in tri_attn.h).  Everything the block needs beyond the
// caller's own buffers lives in one file-scope device array: the packed weight
// images, the fp32 parameters, the device status word and the workspace.  The
// existing kernels run on it unchanged, in row chunks sized to the array.
namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr size_t kNaWImg = 0;                                // [Wq; Wk; Wv]: 384 x 128 bf16 image
constexpr size_t kNaWgImg = kNaWImg + 384 * 128 * 2;         // Wg: 128 x 128 bf16 image
constexpr size_t kNaWoImg = kNaWgImg + 128 * 128 * 2;        // Wo: 128 x 128 bf16 image
constexpr size_t kNaWb = kNaWoImg + 128 * 128 * 2;           // fp32 [H][c_z] x log2(e)
constexpr size_t kNaGamma = kNaWb + kHeads * kCz * 4;
constexpr size_t kNaBeta = kNaGamma + kCz * 4;
constexpr size_t kNaBg = kNaBeta + kCz * 4;
constexpr size_t kNaBo = kNaBg + kHD * 4;
constexpr size_t kNaStatus = kNaBo + kCz * 4;
constexpr size_t kNaWs = (kNaStatus + 256 + 1023) / 1024 * 1024;  // workspace: the rest
constexpr int kNaMaxDevices = 64;

// Device memory of the library itself: present on every GPU that loads it,
// until the process exits.  In host code this name is only a stand-in; the
// device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kNaMaxDevices] = {};

// Byte offset of element (n, k) in the K-major, 128-byte-swizzled image of a
// bf16 operand with `rows` rows of 128 elements (same layout as
// pack_kmajor_sw128 above).
__device__ __forceinline__ size_t sw128_offset(int rows, int n, int k) {
  const int slab = k / 64, c = (k % 64) / 8, e = k % 8;
  return static_cast<size_t>(slab) * rows * 128 + static_cast<size_t>(n) * 128 +
         ((c ^ (n & 7)) * 16) + e * 2;
}

// Repack the caller's bf16 weights into the scratch array, on the stream.
__global__ void pack_weights_noalloc(const bf16* wq, const bf16* wk, const bf16* wv,
                                     const bf16* wg, const bf16* wo, const bf16* wb,
                                     const bf16* gamma, const bf16* beta, const bf16* bg,
                                     const bf16* bo, unsigned char* scratch) {
  const int n_w = 384 * 128, n_wg = 128 * 128, n_wo = 128 * 128, n_wb = kHeads * kCz;
  const int total = n_w + n_wg + n_wo + n_wb + 4 * kCz;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += gridDim.x * blockDim.x) {
    if (idx < n_w) {
      const int n = idx / 128, k = idx % 128, part = n / kHD, nn = n % kHD;
      const bf16* src = part == 0 ? wq : part == 1 ? wk : wv;
      *reinterpret_cast<bf16*>(scratch + kNaWImg + sw128_offset(384, n, k)) = src[nn * kCz + k];
    } else if (idx < n_w + n_wg) {
      const int t = idx - n_w, n = t / 128, k = t % 128;
      *reinterpret_cast<bf16*>(scratch + kNaWgImg + sw128_offset(128, n, k)) =
          __float2bfloat16(0.5f * __bfloat162float(wg[n * kCz + k]));  // exact
    } else if (idx < n_w + n_wg + n_wo) {
      const int t = idx - n_w - n_wg, n = t / 128, k = t % 128;
      *reinterpret_cast<bf16*>(scratch + kNaWoImg + sw128_offset(128, n, k)) =
          __float2bfloat16(0.5f * __bfloat162float(wo[n * kHD + k]));  // exact
    } else if (idx < n_w + n_wg + n_wo + n_wb) {
      const int t = idx - n_w - n_wg - n_wo;
      reinterpret_cast<float*>(scratch + kNaWb)[t] = __bfloat162float(wb[t]) * tri::kLog2e;
    } else {
      const int t = idx - n_w - n_wg - n_wo - n_wb, which = t / kCz, c = t % kCz;
      if (which == 0) reinterpret_cast<float*>(scratch + kNaGamma)[c] = __bfloat162float(gamma[c]);
      if (which == 1) reinterpret_cast<float*>(scratch + kNaBeta)[c] = __bfloat162float(beta[c]);
      if (which == 2)
        reinterpret_cast<float*>(scratch + kNaBg)[c] = bg ? __bfloat162float(bg[c]) : 0.f;
      if (which == 3)
        reinterpret_cast<float*>(scratch + kNaBo)[c] = bo ? __bfloat162float(bo[c]) : 0.f;
    }
  }
}

// Scratch a forward of size N needs: the weights, the whole bias and at least one
// chunk of rows (the attention kernel's row group).
size_t noalloc_required(int N) {
  return kNaWs + bias_bytes(TRI_ATTN_BF16, N) + 6 * 256 +
         static_cast<size_t>(tri::attn::kRows) * row_bytes(TRI_ATTN_BF16, N);
}

}  // namespace

extern "C" int tri_attn_forward_noalloc(const tri_attn_params* p, const void* Z, int N,
                                        const uint8_t* mask, tri_attn_orientation orientation,
                                        void* out, void* stream, unsigned flags) {
  if (!p || !Z || !out || N < 1) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->dtype != TRI_ATTN_BF16) return TRI_ATTN_ERR_UNSUPPORTED;
  if (p->c_z != kCz || p->n_heads != kHeads || p->head_dim != kD) return TRI_ATTN_ERR_UNSUPPORTED;
  if (!p->ln_gamma || !p->ln_beta || !p->w_q || !p->w_k || !p->w_v || !p->w_g || !p->w_b ||
      !p->w_o)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (!(p->ln_eps >= 0.f) || !std::isfinite(p->ln_eps)) return TRI_ATTN_ERR_INVALID_ARG;
  if (orientation != TRI_ATTN_STARTING && orientation != TRI_ATTN_ENDING)
    return TRI_ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Z) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
    return TRI_ATTN_ERR_INVALID_ARG;
  if (N > 46340 || noalloc_required(N) > kNoallocScratchBytes) {
    TA_LOG("tri_attn_forward_noalloc: N=%d needs %zu bytes of scratch, the static array holds %zu",
           N, noalloc_required(N), kNoallocScratchBytes);
    return TRI_ATTN_ERR_UNSUPPORTED;
  }
  const size_t bytes = static_cast<size_t>(N) * N * kCz * 2;
  if (Z != out && ranges_overlap(Z, out, bytes)) return TRI_ATTN_ERR_ALIAS;
  int rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNaMaxDevices) return TRI_ATTN_ERR_UNSUPPORTED;

  // set-up, once per device, with that device current
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
      void* ptr = nullptr;
      CUDA_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
      g_noalloc_addr[dev] = ptr;
    }
    base = g_noalloc_addr[dev];
  }
  unsigned char* scratch = static_cast<unsigned char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // the array keeps the previous call's contents: the status word must start at 0
  CUDA_TRY(cudaMemsetAsync(scratch + kNaStatus, 0, sizeof(int), st));
  pack_weights_noalloc<<<128, 256, 0, st>>>(
      static_cast<const bf16*>(p->w_q), static_cast<const bf16*>(p->w_k),
      static_cast<const bf16*>(p->w_v), static_cast<const bf16*>(p->w_g),
      static_cast<const bf16*>(p->w_o), static_cast<const bf16*>(p->w_b),
      static_cast<const bf16*>(p->ln_gamma), static_cast<const bf16*>(p->ln_beta),
      static_cast<const bf16*>(p->b_g), static_cast<const bf16*>(p->b_o), scratch);
  CUDA_TRY(cudaGetLastError());

  // a handle on the stack whose buffers all point into the scratch array, so the
  // forward below never reaches cudaMalloc
  tri_attn_handle hh;
  hh.device = dev;
  CUDA_TRY(cudaDeviceGetAttribute(&hh.num_sms, cudaDevAttrMultiProcessorCount, dev));
  hh.dtype = TRI_ATTN_BF16;
  hh.eps = p->ln_eps;
  hh.q_scale = tri::kLog2e / std::sqrt(static_cast<float>(kD));
  hh.w_qkvg = scratch + kNaWImg;
  hh.w_g = scratch + kNaWgImg;
  hh.w_o = scratch + kNaWoImg;
  hh.w_b = reinterpret_cast<float*>(scratch + kNaWb);
  hh.gamma = reinterpret_cast<float*>(scratch + kNaGamma);
  hh.beta = reinterpret_cast<float*>(scratch + kNaBeta);
  hh.b_g = reinterpret_cast<float*>(scratch + kNaBg);
  hh.b_o = reinterpret_cast<float*>(scratch + kNaBo);
  hh.status = reinterpret_cast<int*>(scratch + kNaStatus);
  hh.ws = scratch + kNaWs;
  hh.ws_bytes = kNoallocScratchBytes - kNaWs;
  hh.ws_limit = hh.ws_bytes;
  rc = forward_impl(&hh, Z, N, mask, static_cast<int>(orientation), out, st,
                    flags & TRI_ATTN_FLAG_SYNC);
  if (rc == TRI_ATTN_OK && (flags & TRI_ATTN_FLAG_SYNC)) {
    int s = 0;
    CUDA_TRY(cudaMemcpyAsync(&s, hh.status, sizeof(int), cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    rc = s;
  }
  hh.ws = nullptr;  // nothing in hh is owned: the handle is never destroyed
  return rc;
}

// ------------------------------------------------------------------ backward
// The backward pass of the attention core (attn_bwd.cuh): row statistics, then
// dQ, dK/dV and the bias gradient, four launches on the caller's stream.

extern "C" size_t tri_attn_attention_backward_workspace_bytes(int rows, int N) {
  if (rows < 1 || N < 1) return 0;
  return 2 * static_cast<size_t>(rows) * tri::kHeads * N * sizeof(float);
}

extern "C" int tri_attn_attention_forward(const float* Q, const float* K, const float* V,
                                          const float* bias, const uint8_t* mask, int rows,
                                          int N, float* O, float* lse, void* stream,
                                          unsigned flags) {
  const void* vec[] = {Q, K, V, O};
  for (const void* ptr : vec)
    if (!ptr || reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return TRI_ATTN_ERR_INVALID_ARG;
  if (!bias || !lse || rows < 1 || N < 1) return TRI_ATTN_ERR_INVALID_ARG;
  if (rows > 65535 || N > 46340) return TRI_ATTN_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  tri::bwd::BwdArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.B = bias;
  a.mask = mask;
  a.lse = lse;
  a.O = O;
  a.rows = rows;
  a.N = N;
  const unsigned tiles = static_cast<unsigned>((N + tri::bwd::kThreadsRow - 1) / tri::bwd::kThreadsRow);
  tri::bwd::bwd_stats<<<dim3(tiles, static_cast<unsigned>(rows), tri::kHeads),
                        tri::bwd::kThreadsRow, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  if (flags & TRI_ATTN_FLAG_SYNC) CUDA_TRY(cudaStreamSynchronize(st));
  return TRI_ATTN_OK;
}

extern "C" int tri_attn_attention_backward(const float* Q, const float* K, const float* V,
                                           const float* bias, const uint8_t* mask,
                                           const float* dO, int rows, int N, float* dQ,
                                           float* dK, float* dV, float* dbias, void* workspace,
                                           size_t workspace_bytes, void* stream,
                                           unsigned flags) {
  const void* vec[] = {Q, K, V, dO, dQ, dK, dV, workspace};
  for (const void* ptr : vec)
    if (!ptr || reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return TRI_ATTN_ERR_INVALID_ARG;
  if (!bias || !dbias || rows < 1 || N < 1) return TRI_ATTN_ERR_INVALID_ARG;
  // indices stay within 64-bit element offsets; grids within their limits
  if (rows > 65535 || N > 46340) return TRI_ATTN_ERR_UNSUPPORTED;
  if (workspace_bytes < tri_attn_attention_backward_workspace_bytes(rows, N))
    return TRI_ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  tri::bwd::BwdArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.B = bias;
  a.dO = dO;
  a.mask = mask;
  a.dQ = dQ;
  a.dK = dK;
  a.dV = dV;
  a.dB = dbias;
  a.lse = static_cast<float*>(workspace);
  a.D = a.lse + static_cast<size_t>(rows) * tri::kHeads * N;
  a.rows = rows;
  a.N = N;
  const unsigned tiles = static_cast<unsigned>((N + tri::bwd::kThreadsRow - 1) / tri::bwd::kThreadsRow);
  const dim3 grid_rows(tiles, static_cast<unsigned>(rows), tri::kHeads);
  tri::bwd::bwd_stats<<<grid_rows, tri::bwd::kThreadsRow, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  tri::bwd::bwd_dq<<<grid_rows, tri::bwd::kThreadsRow, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  tri::bwd::bwd_dkdv<<<grid_rows, tri::bwd::kDkdvThreads, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  const unsigned blocks = static_cast<unsigned>((N + tri::bwd::kBlk - 1) / tri::bwd::kBlk);
  tri::bwd::bwd_dbias<<<dim3(blocks, blocks, tri::kHeads), tri::bwd::kBlkThreads, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  if (flags & TRI_ATTN_FLAG_SYNC) CUDA_TRY(cudaStreamSynchronize(st));
  return TRI_ATTN_OK;
}

// ------------------------------------------------------------------ bf16 attention core
namespace {

struct CoreWs {
  int* status = nullptr;
  bf16 *qs = nullptr, *b2 = nullptr, *b2T = nullptr;
  float *nlse2 = nullptr, *nD = nullptr;
};

// Workspace of the bf16 core calls: the device status word, Qs [rows][H][N][d]
// bf16, b2 and b2T [H][N][ld] bf16, -lse2 and -D [rows][H][ld] fp32 (ld = N
// rounded up to 128), each part 256-byte aligned.  Returns the bytes needed;
// fills *w when base is set.
size_t core_ws_layout(int rows, int N, void* base, CoreWs* w) {
  const size_t ld = static_cast<size_t>(tri::bwdtc::padded_ld(N));
  const size_t rh = static_cast<size_t>(rows) * tri::kHeads;
  const size_t parts[6] = {sizeof(int), rh * N * tri::kD * 2, tri::kHeads * N * ld * 2,
                           tri::kHeads * N * ld * 2, rh * ld * 4, rh * ld * 4};
  size_t off[6], total = 0;
  for (int p = 0; p < 6; ++p) {
    off[p] = total;
    total = align_up(total + parts[p], 256);
  }
  if (base != nullptr && w != nullptr) {
    char* b = static_cast<char*>(base);
    w->status = reinterpret_cast<int*>(b + off[0]);
    w->qs = reinterpret_cast<bf16*>(b + off[1]);
    w->b2 = reinterpret_cast<bf16*>(b + off[2]);
    w->b2T = reinterpret_cast<bf16*>(b + off[3]);
    w->nlse2 = reinterpret_cast<float*>(b + off[4]);
    w->nD = reinterpret_cast<float*>(b + off[5]);
  }
  return total;
}

// [rows][H][N][d] bf16 operand, boxes of `box` rows x 32 (64-byte swizzle)
bool operand_map(CUtensorMap* m, const void* p, int rows, int N, uint32_t box) {
  return make_map_3d(m, p, tri::kD, N, static_cast<uint64_t>(rows) * tri::kHeads, tri::kD * 2,
                     static_cast<uint64_t>(N) * tri::kD * 2, tri::kD, box,
                     CU_TENSOR_MAP_SWIZZLE_64B);
}

// [H][N][ld] bf16 bias, boxes of 128 rows x 64 columns (128-byte swizzle)
bool bias_map(CUtensorMap* m, const void* p, int N, int ld) {
  return make_map_3d(m, p, ld, N, tri::kHeads, static_cast<uint64_t>(ld) * 2,
                     static_cast<uint64_t>(N) * ld * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
}

int core_args_ok(const void* const* aligned16, int n, const void* bias, int rows, int N,
                 void* workspace, size_t workspace_bytes) {
  for (int i = 0; i < n; ++i)
    if (!aligned16[i] || reinterpret_cast<uintptr_t>(aligned16[i]) % 16 != 0)
      return TRI_ATTN_ERR_INVALID_ARG;
  if (!bias || rows < 1 || N < 1) return TRI_ATTN_ERR_INVALID_ARG;
  if (rows > 65535 || N > 46340) return TRI_ATTN_ERR_UNSUPPORTED;
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 16 != 0 ||
      workspace_bytes < core_ws_layout(rows, N, nullptr, nullptr))
    return TRI_ATTN_ERR_INVALID_ARG;
  return TRI_ATTN_OK;
}

// Clear the status word; Qs, b2 (and b2T when asked) from the caller's operands
int core_prep(const void* Q, const void* bias, const uint8_t* mask, int rows, int N,
              const CoreWs& w, bool transpose, cudaStream_t st) {
  CUDA_TRY(cudaMemsetAsync(w.status, 0, sizeof(int), st));
  const int ld = tri::bwdtc::padded_ld(N);
  const long long n8 = static_cast<long long>(rows) * tri::kHeads * N * tri::kD / 8;
  const int blocks = static_cast<int>(std::min<long long>((n8 + 255) / 256, 148 * 16));
  tri::bwdtc::prep_q<<<blocks, 256, 0, st>>>(static_cast<const bf16*>(Q), w.qs, n8);
  CUDA_TRY(cudaGetLastError());
  tri::bwdtc::prep_bias<<<dim3(ld / 32, ld / 32, tri::kHeads), dim3(32, 8), 0, st>>>(
      static_cast<const bf16*>(bias), mask, N, ld, w.b2, transpose ? w.b2T : nullptr);
  CUDA_TRY(cudaGetLastError());
  return TRI_ATTN_OK;
}

// With TRI_ATTN_FLAG_SYNC: wait for the call and return its device status.
int core_finish(const CoreWs& w, cudaStream_t st, unsigned flags) {
  if (!(flags & TRI_ATTN_FLAG_SYNC)) return TRI_ATTN_OK;
  int s = 0;
  CUDA_TRY(cudaMemcpyAsync(&s, w.status, sizeof(int), cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  return s;
}

}  // namespace

extern "C" size_t tri_attn_attention_bf16_workspace_bytes(int rows, int N) {
  if (rows < 1 || N < 1) return 0;
  return core_ws_layout(rows, N, nullptr, nullptr);
}

extern "C" int tri_attn_attention_forward_bf16(const void* Q, const void* K, const void* V,
                                               const void* bias, const uint8_t* mask, int rows,
                                               int N, void* O, float* lse, void* workspace,
                                               size_t workspace_bytes, void* stream,
                                               unsigned flags) {
  const void* vec[] = {Q, K, V, O};
  int rc = core_args_ok(vec, 4, bias, rows, N, workspace, workspace_bytes);
  if (rc != TRI_ATTN_OK) return rc;
  if (lse && reinterpret_cast<uintptr_t>(lse) % 4 != 0) return TRI_ATTN_ERR_INVALID_ARG;
  rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;
  rc = set_kernel_attrs();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CoreWs w;
  core_ws_layout(rows, N, workspace, &w);
  rc = core_prep(Q, bias, mask, rows, N, w, false, st);
  if (rc != TRI_ATTN_OK) return rc;
  const int ld = tri::bwdtc::padded_ld(N);
  CUtensorMap mq, mk, mv, mb;
  if (!operand_map(&mq, w.qs, rows, N, tri::attn::kBJ) ||
      !operand_map(&mk, K, rows, N, tri::attn::kBK) ||
      !operand_map(&mv, V, rows, N, tri::attn::kBK) || !bias_map(&mb, w.b2, N, ld))
    return TRI_ATTN_ERR_CUDA;
  tri::AttnArgs a{};
  a.O = static_cast<bf16*>(O);
  a.lse = lse;
  a.N = N;
  a.rows = rows;
  a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL) ? 1 : 0;
  a.status = w.status;
  const dim3 grid((N + tri::attn::kBJ - 1) / tri::attn::kBJ,
                  (rows + tri::attn::kRows - 1) / tri::attn::kRows, tri::kHeads);
  tri::attn::tri_attn_fwd<<<grid, tri::attn::kThreads, tri::attn::kSmemBytes, st>>>(mq, mk, mv,
                                                                                 mb, a);
  CUDA_TRY(cudaGetLastError());
  return core_finish(w, st, flags);
}

extern "C" int tri_attn_attention_backward_bf16(const void* Q, const void* K, const void* V,
                                                const void* bias, const uint8_t* mask,
                                                const void* O, const float* lse, const void* dO,
                                                int rows, int N, float* dQ, float* dK, float* dV,
                                                float* dbias, void* workspace,
                                                size_t workspace_bytes, void* stream,
                                                unsigned flags) {
  const void* vec[] = {Q, K, V, O, dO, dQ, dK, dV, dbias};
  int rc = core_args_ok(vec, 9, bias, rows, N, workspace, workspace_bytes);
  if (rc != TRI_ATTN_OK) return rc;
  if (!lse || reinterpret_cast<uintptr_t>(lse) % 4 != 0) return TRI_ATTN_ERR_INVALID_ARG;
  rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;
  rc = set_kernel_attrs();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CoreWs w;
  core_ws_layout(rows, N, workspace, &w);
  rc = core_prep(Q, bias, mask, rows, N, w, true, st);
  if (rc != TRI_ATTN_OK) return rc;
  const int ld = tri::bwdtc::padded_ld(N);
  {
    const long long rh = static_cast<long long>(rows) * tri::kHeads;
    const int blocks = static_cast<int>(std::min<long long>((rh * ld + 255) / 256, 148 * 16));
    tri::bwdtc::prep_rows<<<blocks, 256, 0, st>>>(static_cast<const bf16*>(O),
                                                  static_cast<const bf16*>(dO), lse, rh, N, ld,
                                                  w.nlse2, w.nD);
    CUDA_TRY(cudaGetLastError());
  }
  CUtensorMap q128, o128, k128, v128, q64, o64, k64, v64, mb, mbT;
  if (!operand_map(&q128, w.qs, rows, N, 128) || !operand_map(&o128, dO, rows, N, 128) ||
      !operand_map(&k128, K, rows, N, 128) || !operand_map(&v128, V, rows, N, 128) ||
      !operand_map(&q64, w.qs, rows, N, 64) || !operand_map(&o64, dO, rows, N, 64) ||
      !operand_map(&k64, K, rows, N, 64) || !operand_map(&v64, V, rows, N, 64) ||
      !bias_map(&mb, w.b2, N, ld) || !bias_map(&mbT, w.b2T, N, ld))
    return TRI_ATTN_ERR_CUDA;
  namespace bt = tri::bwdtc;
  bt::RowsArgs ra{};
  ra.nlse2 = w.nlse2;
  ra.nD = w.nD;
  ra.N = N;
  ra.rows = rows;
  ra.ld = ld;
  ra.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL) ? 1 : 0;
  ra.status = w.status;
  const unsigned mtiles = static_cast<unsigned>((N + bt::kTM - 1) / bt::kTM);
  {
    using L = bt::RowsLayout<bt::kDQ>;
    ra.out1 = dQ;
    ra.out2 = nullptr;
    const dim3 grid(mtiles, (rows + L::kR - 1) / L::kR, tri::kHeads);
    bt::bwd_rows<bt::kDQ><<<grid, L::kThreads, L::kSmemBytes, st>>>(q128, o128, k64, v64, mb, ra);
    CUDA_TRY(cudaGetLastError());
  }
  {
    using L = bt::RowsLayout<bt::kDKDV>;
    ra.out1 = dK;
    ra.out2 = dV;
    const dim3 grid(mtiles, (rows + L::kR - 1) / L::kR, tri::kHeads);
    bt::bwd_rows<bt::kDKDV><<<grid, L::kThreads, L::kSmemBytes, st>>>(k128, v128, q64, o64, mbT,
                                                                       ra);
    CUDA_TRY(cudaGetLastError());
  }
  {
    bt::DbiasArgs da{};
    da.nlse2 = w.nlse2;
    da.nD = w.nD;
    da.dB = dbias;
    da.N = N;
    da.rows = rows;
    da.ld = ld;
    da.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL) ? 1 : 0;
    da.status = w.status;
    const dim3 grid((N + bt::kTN - 1) / bt::kTN, mtiles, tri::kHeads);
    bt::bwd_dbias_tc<<<grid, bt::kDbThreads, bt::kDbSmemBytes, st>>>(q128, o128, k64, v64, mb, da);
    CUDA_TRY(cudaGetLastError());
  }
  return core_finish(w, st, flags);
}

// ------------------------------------------------------------------ block-level calls
// The three kernels of the block on caller-owned tensors, for a distributed
// driver that moves the intermediate tensors between devices itself (the 2D
// grid: K/V column blocks passed round a ring, partial outputs merged by
// their log-sum-exp).  A block of pairs is [rows][cols][c_z], taken as a
// starting-node problem whose rows are its rows and whose keys are its columns.
namespace {

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_block_handle(tri_attn_handle* h, int rows, int cols) {
  if (!h || rows < 1 || cols < 1) return TRI_ATTN_ERR_INVALID_ARG;
  if (h->dtype != TRI_ATTN_BF16) return TRI_ATTN_ERR_UNSUPPORTED;
  if (rows > 65535 || cols > 46340) return TRI_ATTN_ERR_UNSUPPORTED;
  return TRI_ATTN_OK;
}

}  // namespace

extern "C" int tri_attn_block_project(tri_attn_handle* h, const void* Z, int rows, int cols,
                                      const uint8_t* mask, void* Q, void* K, void* V, void* bias,
                                      void* stream, unsigned flags) {
  int rc = check_block_handle(h, rows, cols);
  if (rc != TRI_ATTN_OK) return rc;
  if (!aligned16(Z) || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(bias))
    return TRI_ATTN_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  rc = set_kernel_attrs();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  tri::ProjArgs a{};
  a.Z = static_cast<const bf16*>(Z);
  a.mask = mask;
  a.N = cols;
  a.orient = 0;
  a.row0 = 0;
  a.rows = rows;
  a.write_qkv = 1;
  a.write_bias = 1;
  a.w_img = static_cast<const uint8_t*>(h->w_qkvg);
  a.w_b = h->w_b;
  a.gamma = h->gamma;
  a.beta = h->beta;
  a.eps = h->eps;
  a.q_scale = h->q_scale;
  a.Q = static_cast<bf16*>(Q);
  a.K = static_cast<bf16*>(K);
  a.V = static_cast<bf16*>(V);
  a.bias = static_cast<bf16*>(bias);
  a.ld_bias = ld_bias_for(cols);
  a.z_row0 = 0;
  a.bias_row0 = 0;
  a.bias_rows = rows;
  a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL_PROJ) ? 1 : 0;
  a.status = h->status;
  const long long ntiles = static_cast<long long>(rows) * ((cols + 127) / 128);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(
      (ntiles + tri::plp::kGroupsPerCta - 1) / tri::plp::kGroupsPerCta, h->num_sms));
  CUtensorMap mz;
  if (!make_map_3d(&mz, Z, kCz, cols, rows, kCz * 2, static_cast<uint64_t>(cols) * kCz * 2, 64,
                   128, CU_TENSOR_MAP_SWIZZLE_128B, 1))
    return TRI_ATTN_ERR_CUDA;
  tri::plp::pair_ln_proj<<<grid, tri::plp::kThreads, tri::plp::kSmemBytes, st>>>(mz, a);
  CUDA_TRY(cudaGetLastError());
  return finish_call(h, st, flags);
}

extern "C" int tri_attn_block_attend(tri_attn_handle* h, const void* Q, const void* K,
                                     const void* V, const void* bias, int ld_bias, int rows,
                                     int n, void* O, float* lse, void* stream, unsigned flags) {
  int rc = check_block_handle(h, rows, n);
  if (rc != TRI_ATTN_OK) return rc;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(bias) || !aligned16(O) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) || ld_bias < ld_bias_for(n) ||
      ld_bias % 8 != 0)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  rc = set_kernel_attrs();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap mq, mk, mv, mb;
  const uint64_t rh = static_cast<uint64_t>(rows) * kHeads;
  const uint64_t row_stride = static_cast<uint64_t>(n) * kD * 2;
  if (!make_map_3d(&mq, Q, kD, n, rh, kD * 2, row_stride, kD, tri::attn::kBJ,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_3d(&mk, K, kD, n, rh, kD * 2, row_stride, kD, tri::attn::kBK,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_3d(&mv, V, kD, n, rh, kD * 2, row_stride, kD, tri::attn::kBK,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_3d(&mb, bias, ld_bias, n, kHeads, static_cast<uint64_t>(ld_bias) * 2,
                   static_cast<uint64_t>(n) * ld_bias * 2, tri::attn::kBK, tri::attn::kBJ,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return TRI_ATTN_ERR_CUDA;
  tri::AttnArgs a{};
  a.O = static_cast<bf16*>(O);
  a.lse = lse;
  a.N = n;
  a.rows = rows;
  a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL) ? 1 : 0;
  a.status = h->status;
  const dim3 grid((n + tri::attn::kBJ - 1) / tri::attn::kBJ,
                  (rows + tri::attn::kRows - 1) / tri::attn::kRows, kHeads);
  tri::attn::tri_attn_fwd<<<grid, tri::attn::kThreads, tri::attn::kSmemBytes, st>>>(mq, mk, mv,
                                                                                 mb, a);
  CUDA_TRY(cudaGetLastError());
  return finish_call(h, st, flags);
}

extern "C" int tri_attn_block_gate(tri_attn_handle* h, const void* Z, int rows, int cols,
                                   const void* O, void* out, void* stream, unsigned flags) {
  int rc = check_block_handle(h, rows, cols);
  if (rc != TRI_ATTN_OK) return rc;
  if (!aligned16(Z) || !aligned16(O) || !aligned16(out)) return TRI_ATTN_ERR_INVALID_ARG;
  {
    // out may be Z itself; any other overlap is rejected
    const size_t bytes = static_cast<size_t>(rows) * cols * kCz * 2;
    const char* z0 = static_cast<const char*>(Z);
    const char* o0 = static_cast<const char*>(out);
    if (o0 != z0 && o0 < z0 + bytes && z0 < o0 + bytes) return TRI_ATTN_ERR_ALIAS;
  }
  if (cudaSetDevice(h->device) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  rc = set_kernel_attrs();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap mo, mz, mout;
  const uint64_t rowb = static_cast<uint64_t>(cols) * kCz * 2;
  if (!make_map_3d(&mo, O, kD, cols, static_cast<uint64_t>(rows) * kHeads, kD * 2,
                   static_cast<uint64_t>(cols) * kD * 2, kD, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_3d(&mz, Z, kCz, cols, rows, kCz * 2, rowb, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B,
                   1) ||
      !make_map_3d(&mout, out, kCz, cols, rows, kCz * 2, rowb, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B, 1))
    return TRI_ATTN_ERR_CUDA;
  tri::GateArgs a{};
  a.Z = static_cast<const bf16*>(Z);
  a.O = static_cast<const bf16*>(O);
  a.wo_img = static_cast<const uint8_t*>(h->w_o);
  a.wg_img = static_cast<const uint8_t*>(h->w_g);
  a.b_o = h->b_o;
  a.b_g = h->b_g;
  a.gamma = h->gamma;
  a.beta = h->beta;
  a.eps = h->eps;
  a.out = static_cast<bf16*>(out);
  a.N = cols;
  a.orient = 0;
  a.row0 = 0;
  a.rows = rows;
  a.z_row0 = 0;
  a.debug_stall = (flags & TRI_ATTN_FLAG_DEBUG_STALL_GATE) ? 1 : 0;
  a.status = h->status;
  const long long ntiles = static_cast<long long>(rows) * ((cols + 127) / 128);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(ntiles, h->num_sms));
  tri::gout::gate_out<<<grid, tri::gout::kThreads, tri::gout::kSmemBytes, st>>>(mo, mz, mout, a);
  CUDA_TRY(cudaGetLastError());
  return finish_call(h, st, flags);
}

extern "C" int tri_attn_merge_partial(float* O_acc, float* lse_acc, const void* O_part,
                                      const float* lse_part, long long count, int first,
                                      void* O_out, void* stream, unsigned flags) {
  if (!aligned16(O_acc) || !aligned16(O_part) || !lse_acc || !lse_part || count < 1 ||
      (O_out && !aligned16(O_out)) || (reinterpret_cast<uintptr_t>(lse_acc) & 3) ||
      (reinterpret_cast<uintptr_t>(lse_part) & 3))
    return TRI_ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != TRI_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  tri::merge::MergeArgs a{};
  a.o_acc = O_acc;
  a.lse_acc = lse_acc;
  a.o_part = static_cast<const bf16*>(O_part);
  a.lse_part = lse_part;
  a.o_out = static_cast<bf16*>(O_out);
  a.count = count;
  a.first = first ? 1 : 0;
  const long long blocks = (count + tri::merge::kThreads - 1) / tri::merge::kThreads;
  if (blocks > 0x7fffffffLL) return TRI_ATTN_ERR_UNSUPPORTED;
  tri::merge::merge_partial<<<static_cast<unsigned>(blocks), tri::merge::kThreads, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  if (flags & TRI_ATTN_FLAG_SYNC) CUDA_TRY(cudaStreamSynchronize(st));
  return TRI_ATTN_OK;
}
