// kernels_f32.cuh — fp32 path (SIMT FFMA) of the three steps of the block.
//
// Used for fp32 handles, where the result must match an fp64 evaluation to
// 1e-4 absolute: tf32 tensor-core arithmetic (10-bit mantissa) cannot meet
// that, so the contractions run as ordinary fp32 fused multiply-adds.
// Workspace semantics are those of the bf16 path (q pre-scaled by
// log2(e)/sqrt(d), logit bias pre-scaled by log2(e), exponentials in base 2).
#pragma once

#include "common.cuh"

namespace tri {
namespace f32 {

constexpr int kProjThreads = 64;

// LayerNorm + Q/K/V/gate/bias projections, one thread per pair.
__global__ void __launch_bounds__(kProjThreads) ln_proj_kernel(ProjArgsF32 a) {
  __shared__ float xs[kProjThreads][kCz + 1];
  const int t = threadIdx.x;
  const long long pair = static_cast<long long>(blockIdx.x) * kProjThreads + t;
  const long long total = static_cast<long long>(a.rows) * a.N;
  const bool valid = pair < total;
  const int r = valid ? static_cast<int>(pair / a.N) : 0;
  const int j = valid ? static_cast<int>(pair % a.N) : 0;
  const int i = a.row0 + r;
  float* x = xs[t];
  if (valid) {
    const float* z = a.Z + pair_offset(a.orient, a.N, i, j);
    float mu = 0.f;
    for (int c = 0; c < kCz; ++c) mu += z[c];
    mu *= (1.0f / kCz);
    float var = 0.f;
    for (int c = 0; c < kCz; ++c) {
      const float dz = z[c] - mu;
      var += dz * dz;
    }
    var *= (1.0f / kCz);
    const float rstd = 1.0f / sqrtf(var + a.eps);
    for (int c = 0; c < kCz; ++c) x[c] = (z[c] - mu) * rstd * a.gamma[c] + a.beta[c];
  }
  if (!valid) return;
  const bool key_valid = a.mask == nullptr || a.mask[j] != 0;
  if (a.write_bias) {
    for (int h = 0; h < kHeads; ++h) {
      float acc = 0.f;
      for (int c = 0; c < kCz; ++c) acc += a.w_b[h * kCz + c] * x[c];
      a.bias[(static_cast<long long>(h) * a.N + i) * a.ld_bias + j] =
          key_valid ? acc : -INFINITY;
    }
  }
  if (!a.write_qkvg) return;
  for (int o = 0; o < 4 * kHD; ++o) {
    const float* w = a.w_qkvg + static_cast<long long>(o) * kCz;
    float acc = 0.f;
    for (int c = 0; c < kCz; ++c) acc += w[c] * x[c];
    const int part = o / kHD, ch = o % kHD, h = ch / kD, e = ch % kD;
    const long long qkv_idx = ((static_cast<long long>(r) * kHeads + h) * a.N + j) * kD + e;
    if (part == 0) a.Q[qkv_idx] = acc * a.q_scale;
    else if (part == 1) a.K[qkv_idx] = acc;
    else if (part == 2) a.V[qkv_idx] = acc;
    else a.G[qkv_idx] = 1.0f / (1.0f + expf(-(acc + a.b_g[ch])));
  }
}

// Bias padding columns j in [N, ld_bias) of every row and head: -inf.
__global__ void bias_pad_kernel(float* bias, int N, int ld_bias) {
  const int pad = ld_bias - N;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(kHeads) * N * pad;
  if (pad <= 0 || idx >= total) return;
  const long long hr = idx / pad;
  bias[hr * ld_bias + N + idx % pad] = -INFINITY;
}

// Online-softmax attention, one thread per (row, head, query).
__global__ void attn_kernel(AttnArgsF32 a) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(a.rows) * kHeads * a.N;
  if (tid >= total) return;
  const int j = static_cast<int>(tid % a.N);
  const long long rh = tid / a.N;  // r * H + h
  const int h = static_cast<int>(rh % kHeads);
  const float* q = a.Q + (rh * a.N + j) * kD;
  const float* kb = a.K + rh * a.N * kD;
  const float* vb = a.V + rh * a.N * kD;
  const float* brow = a.bias + (static_cast<long long>(h) * a.N + j) * a.ld_bias;
  float qr[kD], o[kD];
#pragma unroll
  for (int c = 0; c < kD; ++c) {
    qr[c] = q[c];
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int k = 0; k < a.N; ++k) {
    const float b = brow[k];
    if (b == -INFINITY) continue;  // masked key
    const float* kr = kb + static_cast<long long>(k) * kD;
    float s = b;
#pragma unroll
    for (int c = 0; c < kD; ++c) s += qr[c] * kr[c];
    const float mn = fmaxf(m, s);
    const float corr = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    const float p = exp2f(s - mn);
    l = l * corr + p;
    const float* vr = vb + static_cast<long long>(k) * kD;
#pragma unroll
    for (int c = 0; c < kD; ++c) o[c] = o[c] * corr + p * vr[c];
    m = mn;
  }
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  float* out = a.O + (rh * a.N + j) * kD;
#pragma unroll
  for (int c = 0; c < kD; ++c) out[c] = o[c] * inv;
}

// Gate, output projection and residual, one thread per pair.
__global__ void __launch_bounds__(kProjThreads) gate_out_kernel(GateArgsF32 a) {
  __shared__ float gs[kProjThreads][kHD + 1];
  const int t = threadIdx.x;
  const long long pair = static_cast<long long>(blockIdx.x) * kProjThreads + t;
  const long long total = static_cast<long long>(a.rows) * a.N;
  if (pair >= total) return;
  const int r = static_cast<int>(pair / a.N);
  const int j = static_cast<int>(pair % a.N);
  const int i = a.row0 + r;
  float* go = gs[t];
  for (int ch = 0; ch < kHD; ++ch) {
    const int h = ch / kD, e = ch % kD;
    const long long idx = ((static_cast<long long>(r) * kHeads + h) * a.N + j) * kD + e;
    go[ch] = a.O[idx] * a.G[idx];
  }
  const long long off = pair_offset(a.orient, a.N, i, j);
  const float* z = a.Z + off;
  float* out = a.out + off;
  for (int c = 0; c < kCz; ++c) {
    const float* w = a.w_o + static_cast<long long>(c) * kHD;
    float acc = a.b_o[c];
    for (int t2 = 0; t2 < kHD; ++t2) acc += w[t2] * go[t2];
    out[c] = z[c] + acc;  // z[c] is read before out[c] is written (in-place safe)
  }
}

}  // namespace f32
}  // namespace tri
