// merge.cuh — merging attention outputs computed over disjoint key blocks.
//
// When the keys of a query are split into blocks (the 2D grid of the
// Design-CP technical summary, §Metodología 1: K/V column blocks passed round a
// ring of devices), each block c gives the softmax over its own keys: o_c
// (normalised within the block) and lse_c = log sum_{k in c} exp(s_k).  The
// softmax over the union is then
//   lse = log sum_c exp(lse_c),   o = sum_c exp(lse_c - lse) o_c,
// evaluated two at a time as the blocks arrive, with the running maximum
// subtracted so that no exponential overflows.  A block whose every key is
// masked has lse_c = +inf by the forward kernel's convention (an empty sum)
// and weight 0; if every block is empty, o = 0 and lse = +inf.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace merge {

constexpr int kThreads = 256;

struct MergeArgs {
  float* o_acc;            // [count][d] fp32, running merged output
  float* lse_acc;          // [count] natural log, running
  const __nv_bfloat16* o_part;  // [count][d] bf16, the new block's output
  const float* lse_part;   // [count]
  __nv_bfloat16* o_out;    // [count][d] bf16 copy of the merged output, or nullptr
  long long count;
  int first;               // the accumulator holds nothing yet
};

// One thread per query (its 32 channels).
__global__ void __launch_bounds__(kThreads) merge_partial(const MergeArgs a) {
  const long long q = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x;
  if (q >= a.count) return;
  const float l2 = a.lse_part[q];
  const float l1 = a.first ? INFINITY : a.lse_acc[q];
  const bool e1 = l1 == INFINITY, e2 = l2 == INFINITY;  // empty blocks
  float w1 = 0.f, w2 = 0.f, lse = INFINITY;
  if (!(e1 && e2)) {
    const float m = e1 ? l2 : (e2 ? l1 : fmaxf(l1, l2));
    w1 = e1 ? 0.f : expf(l1 - m);
    w2 = e2 ? 0.f : expf(l2 - m);
    lse = m + logf(w1 + w2);
    const float inv = 1.0f / (w1 + w2);
    w1 *= inv;
    w2 *= inv;
  }
  float4* acc = reinterpret_cast<float4*>(a.o_acc + q * kD);
  const uint4* part = reinterpret_cast<const uint4*>(a.o_part + q * kD);
#pragma unroll
  for (int c = 0; c < kD / 8; ++c) {
    const uint4 pv = part[c];
    const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
    float r[8];
    const float4 o1a = a.first ? make_float4(0.f, 0.f, 0.f, 0.f) : acc[2 * c];
    const float4 o1b = a.first ? make_float4(0.f, 0.f, 0.f, 0.f) : acc[2 * c + 1];
    const float o1[8] = {o1a.x, o1a.y, o1a.z, o1a.w, o1b.x, o1b.y, o1b.z, o1b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      r[2 * e] = w1 * o1[2 * e] + w2 * bf16lo_to_f32(pw[e]);
      r[2 * e + 1] = w1 * o1[2 * e + 1] + w2 * bf16hi_to_f32(pw[e]);
    }
    acc[2 * c] = make_float4(r[0], r[1], r[2], r[3]);
    acc[2 * c + 1] = make_float4(r[4], r[5], r[6], r[7]);
    if (a.o_out != nullptr) {
      uint4 ov;
      ov.x = pack_bf16x2(r[0], r[1]);
      ov.y = pack_bf16x2(r[2], r[3]);
      ov.z = pack_bf16x2(r[4], r[5]);
      ov.w = pack_bf16x2(r[6], r[7]);
      reinterpret_cast<uint4*>(a.o_out + q * kD)[c] = ov;
    }
  }
  a.lse_acc[q] = lse;
}

}  // namespace merge
}  // namespace tri
