// attn_bwd.cuh — backward pass of the attention core, fp32 (SIMT FFMA).
//
// For the starting-node core over R problem rows (the ending node is the same
// computation on the transposed problem), head h, query j and key k of row r:
//   s_jk = q_j . k_k / sqrt(d) + B[h][j][k]   over unmasked keys k
//   p_jk = softmax_k(s_j.),  o_j = sum_k p_jk v_k
// and, given dO = d loss / d o, the chain rule through each softmax row:
//   D_j   = dO_j . o_j = sum_k p_jk (dO_j . v_k)
//   ds_jk = p_jk (dO_j . v_k - D_j)
//   dQ_j  = sum_k ds_jk k_k / sqrt(d),   dK_k = sum_j ds_jk q_j / sqrt(d),
//   dV_k  = sum_j p_jk dO_j,             dB[h][j][k] = sum_r ds_jk (over rows).
// p is recomputed from the row statistics instead of being stored: an R x N x N
// x H probability tensor would not fit (58 GB at N = 1536).  Four kernels:
//   bwd_stats   thread = query: one pass over the keys with a running maximum
//               gives LSE_j = log sum_k exp(s_jk) and D_j (alone, with o written
//               out, it is also the forward of the core);
//   bwd_dq      thread = query: dQ_j, keys streamed through shared memory;
//   bwd_dkdv    thread = key: dK_k and dV_k, queries streamed through shared
//               memory;
//   bwd_dbias   a CTA owns a 64 x 64 (j, k) block of one head and sums ds over
//               all rows in registers, so the bias gradient is written once,
//               with no atomics (deterministic).
// Every product is an fp32 fused multiply-add; exponentials use expf.
#pragma once

#include "common.cuh"

namespace tri {
namespace bwd {

struct BwdArgs {
  const float *Q, *K, *V, *B, *dO;  // [rows][H][N][d]; B: [H][N][N]; dO may be null (forward)
  const uint8_t* mask;              // [N] or nullptr
  float *dQ, *dK, *dV, *dB;         // like Q, K, V and B
  float *lse, *D;                   // [rows][H][N] scratch (D unused without dO)
  float* O;                         // [rows][H][N][d]: o written here when not null
  int rows, N;
};

constexpr float kScale = 0.17677669529663687f;  // 1 / sqrt(32)
constexpr int kThreadsRow = 128;  // bwd_stats, bwd_dq: queries per CTA; bwd_dkdv: keys per CTA
constexpr int kTileK = 32;        // keys per shared-memory tile (bwd_stats, bwd_dq)
constexpr int kTileJ = 32;        // queries per shared-memory tile (bwd_dkdv)
constexpr int kBlk = 64;          // bwd_dbias: (j, k) block edge
constexpr int kBlkThreads = 256;  // bwd_dbias: each thread a 4 x 4 sub-block
constexpr int kTr = kBlk + 4;     // row pitch of the transposed tiles of bwd_dbias

__device__ __forceinline__ bool key_ok(const BwdArgs& a, int k) {
  return k < a.N && (a.mask == nullptr || a.mask[k] != 0);
}

__device__ __forceinline__ void load_vec(const float* src, float (&x)[kD]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int c = 0; c < kD / 4; ++c) {
    const float4 v = __ldg(s4 + c);
    x[4 * c] = v.x;
    x[4 * c + 1] = v.y;
    x[4 * c + 2] = v.z;
    x[4 * c + 3] = v.w;
  }
}

// Stage rows k0 .. k0+n-1 of a [N][d] block into tile[n][d] (zeros past N).
template <int n, int nthreads>
__device__ __forceinline__ void stage_rows(const float* blk, int k0, int N, float (*tile)[kD]) {
  for (int idx = threadIdx.x; idx < n * kD / 4; idx += nthreads) {
    const int kk = idx / (kD / 4), c4 = idx % (kD / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (k0 + kk < N) v = __ldg(reinterpret_cast<const float4*>(blk + (k0 + kk) * kD) + c4);
    reinterpret_cast<float4*>(tile[kk])[c4] = v;
  }
}

// ------------------------------------------------------------------ bwd_stats
__global__ void __launch_bounds__(kThreadsRow, 4) bwd_stats(BwdArgs a) {
  __shared__ float sK[kTileK][kD], sV[kTileK][kD];
  __shared__ float sB[kThreadsRow][kTileK + 1];
  __shared__ unsigned char sM[kTileK];
  const int h = blockIdx.z, r = blockIdx.y, j0 = blockIdx.x * kThreadsRow, t = threadIdx.x;
  const int j = j0 + t;
  const bool jv = j < a.N;
  const long long blk = (static_cast<long long>(r) * kHeads + h) * a.N;  // row-head block
  float q[kD], o[kD];
#pragma unroll
  for (int c = 0; c < kD; ++c) q[c] = o[c] = 0.f;
  if (jv) load_vec(a.Q + (blk + j) * kD, q);
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < a.N; k0 += kTileK) {
    __syncthreads();
    stage_rows<kTileK, kThreadsRow>(a.K + blk * kD, k0, a.N, sK);
    stage_rows<kTileK, kThreadsRow>(a.V + blk * kD, k0, a.N, sV);
    for (int idx = t; idx < kThreadsRow * kTileK; idx += kThreadsRow) {
      const int jj = idx / kTileK, kk = idx % kTileK;
      sB[jj][kk] = (j0 + jj < a.N && k0 + kk < a.N)
                       ? __ldg(a.B + (static_cast<long long>(h) * a.N + j0 + jj) * a.N + k0 + kk)
                       : 0.f;
    }
    if (t < kTileK) sM[t] = key_ok(a, k0 + t) ? 1 : 0;
    __syncthreads();
    if (!jv) continue;
    float s[kTileK];
    float tmax = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < kTileK; ++kk) {
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < kD; ++c) dot = fmaf(q[c], sK[kk][c], dot);
      s[kk] = sM[kk] ? fmaf(dot, kScale, sB[t][kk]) : -INFINITY;
      tmax = fmaxf(tmax, s[kk]);
    }
    if (tmax == -INFINITY) continue;  // every key of this tile masked
    const float mn = fmaxf(m, tmax);
    const float corr = m == -INFINITY ? 0.f : expf(m - mn);
    l *= corr;
#pragma unroll
    for (int c = 0; c < kD; ++c) o[c] *= corr;
#pragma unroll
    for (int kk = 0; kk < kTileK; ++kk) {
      const float p = expf(s[kk] - mn);  // 0 at masked keys
      l += p;
#pragma unroll
      for (int c = 0; c < kD; ++c) o[c] = fmaf(p, sV[kk][c], o[c]);
    }
    m = mn;
  }
  if (!jv) return;
  // a query with every key masked: LSE = +inf makes every p exactly 0
  a.lse[blk + j] = l > 0.f ? m + logf(l) : INFINITY;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  if (a.O) {  // the forward: o = O / l
    float4* dst = reinterpret_cast<float4*>(a.O + (blk + j) * kD);
#pragma unroll
    for (int c = 0; c < kD / 4; ++c)
      dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv,
                           o[4 * c + 3] * inv);
  }
  if (a.dO) {
    float g[kD];
    load_vec(a.dO + (blk + j) * kD, g);
    float dd = 0.f;
#pragma unroll
    for (int c = 0; c < kD; ++c) dd = fmaf(g[c], o[c], dd);
    a.D[blk + j] = dd * inv;
  }
}

// --------------------------------------------------------------------- bwd_dq
__global__ void __launch_bounds__(kThreadsRow) bwd_dq(BwdArgs a) {
  __shared__ float sK[kTileK][kD], sV[kTileK][kD];
  __shared__ float sB[kThreadsRow][kTileK + 1];
  __shared__ unsigned char sM[kTileK];
  const int h = blockIdx.z, r = blockIdx.y, j0 = blockIdx.x * kThreadsRow, t = threadIdx.x;
  const int j = j0 + t;
  const bool jv = j < a.N;
  const long long blk = (static_cast<long long>(r) * kHeads + h) * a.N;
  float q[kD], g[kD], dq[kD];
#pragma unroll
  for (int c = 0; c < kD; ++c) q[c] = g[c] = dq[c] = 0.f;
  float lse = INFINITY, Dj = 0.f;
  if (jv) {
    load_vec(a.Q + (blk + j) * kD, q);
    load_vec(a.dO + (blk + j) * kD, g);
    lse = a.lse[blk + j];
    Dj = a.D[blk + j];
  }
  for (int k0 = 0; k0 < a.N; k0 += kTileK) {
    __syncthreads();
    stage_rows<kTileK, kThreadsRow>(a.K + blk * kD, k0, a.N, sK);
    stage_rows<kTileK, kThreadsRow>(a.V + blk * kD, k0, a.N, sV);
    for (int idx = t; idx < kThreadsRow * kTileK; idx += kThreadsRow) {
      const int jj = idx / kTileK, kk = idx % kTileK;
      sB[jj][kk] = (j0 + jj < a.N && k0 + kk < a.N)
                       ? __ldg(a.B + (static_cast<long long>(h) * a.N + j0 + jj) * a.N + k0 + kk)
                       : 0.f;
    }
    if (t < kTileK) sM[t] = key_ok(a, k0 + t) ? 1 : 0;
    __syncthreads();
    if (!jv || lse == INFINITY) continue;
#pragma unroll 4
    for (int kk = 0; kk < kTileK; ++kk) {
      if (!sM[kk]) continue;
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < kD; ++c) {
        dot = fmaf(q[c], sK[kk][c], dot);
        dp = fmaf(g[c], sV[kk][c], dp);
      }
      const float p = expf(fmaf(dot, kScale, sB[t][kk]) - lse);
      const float ds = p * (dp - Dj);
#pragma unroll
      for (int c = 0; c < kD; ++c) dq[c] = fmaf(ds, sK[kk][c], dq[c]);
    }
  }
  if (!jv) return;
  float4* dst = reinterpret_cast<float4*>(a.dQ + (blk + j) * kD);
#pragma unroll
  for (int c = 0; c < kD / 4; ++c)
    dst[c] = make_float4(dq[4 * c] * kScale, dq[4 * c + 1] * kScale, dq[4 * c + 2] * kScale,
                         dq[4 * c + 3] * kScale);
}

// ------------------------------------------------------------------- bwd_dkdv
constexpr int kDkdvThreads = kThreadsRow;  // one thread per key
__global__ void __launch_bounds__(kDkdvThreads) bwd_dkdv(BwdArgs a) {
  __shared__ float sQ[kTileJ][kD], sG[kTileJ][kD];
  __shared__ float sB[kTileJ][kThreadsRow];
  __shared__ float sL[kTileJ], sDj[kTileJ];
  const int h = blockIdx.z, r = blockIdx.y, k0 = blockIdx.x * kThreadsRow, t = threadIdx.x;
  const int k = k0 + t;
  const bool kv = key_ok(a, k);  // a masked key gets p = 0 from every query
  const long long blk = (static_cast<long long>(r) * kHeads + h) * a.N;
  float kk_[kD], vv[kD], dk[kD], dv[kD];
#pragma unroll
  for (int c = 0; c < kD; ++c) kk_[c] = vv[c] = dk[c] = dv[c] = 0.f;
  if (kv) {
    load_vec(a.K + (blk + k) * kD, kk_);
    load_vec(a.V + (blk + k) * kD, vv);
  }
  for (int q0 = 0; q0 < a.N; q0 += kTileJ) {
    __syncthreads();
    stage_rows<kTileJ, kThreadsRow>(a.Q + blk * kD, q0, a.N, sQ);
    stage_rows<kTileJ, kThreadsRow>(a.dO + blk * kD, q0, a.N, sG);
    for (int idx = t; idx < kTileJ * kThreadsRow; idx += kThreadsRow) {
      const int jj = idx / kThreadsRow, kq = idx % kThreadsRow;
      sB[jj][kq] = (q0 + jj < a.N && k0 + kq < a.N)
                       ? __ldg(a.B + (static_cast<long long>(h) * a.N + q0 + jj) * a.N + k0 + kq)
                       : 0.f;
    }
    if (t < kTileJ) {
      const bool jv = q0 + t < a.N;
      sL[t] = jv ? a.lse[blk + q0 + t] : INFINITY;  // p = 0 past N
      sDj[t] = jv ? a.D[blk + q0 + t] : 0.f;
    }
    __syncthreads();
    if (!kv) continue;
#pragma unroll 2
    for (int jj = 0; jj < kTileJ; ++jj) {
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < kD; ++c) {
        dot = fmaf(sQ[jj][c], kk_[c], dot);
        dp = fmaf(sG[jj][c], vv[c], dp);
      }
      const float p = expf(fmaf(dot, kScale, sB[jj][t]) - sL[jj]);
      const float ds = p * (dp - sDj[jj]);
#pragma unroll
      for (int c = 0; c < kD; ++c) {
        dk[c] = fmaf(ds, sQ[jj][c], dk[c]);
        dv[c] = fmaf(p, sG[jj][c], dv[c]);
      }
    }
  }
  if (k >= a.N) return;
  float4* dK = reinterpret_cast<float4*>(a.dK + (blk + k) * kD);
  float4* dV = reinterpret_cast<float4*>(a.dV + (blk + k) * kD);
#pragma unroll
  for (int c = 0; c < kD / 4; ++c) {
    dK[c] = make_float4(dk[4 * c] * kScale, dk[4 * c + 1] * kScale, dk[4 * c + 2] * kScale,
                        dk[4 * c + 3] * kScale);
    dV[c] = make_float4(dv[4 * c], dv[4 * c + 1], dv[4 * c + 2], dv[4 * c + 3]);
  }
}

// ------------------------------------------------------------------ bwd_dbias
// CTA = head h, queries j0 .. j0+63, keys k0 .. k0+63; thread = a 4 x 4 block
// (queries j0 + 4 (t / 16) + a, keys k0 + 4 (t % 16) + b).  Per row, the
// row's q, dO, k, v rows of the block are staged transposed ([c][row], pitch
// kTr) so that a thread reads its four rows' channel c as one float4.
__global__ void __launch_bounds__(kBlkThreads, 2) bwd_dbias(BwdArgs a) {
  __shared__ __align__(16) float sQ[kD][kTr], sG[kD][kTr], sK[kD][kTr], sV[kD][kTr];
  __shared__ float sL[kBlk], sDj[kBlk];
  const int h = blockIdx.z, j0 = blockIdx.y * kBlk, k0 = blockIdx.x * kBlk, t = threadIdx.x;
  const int ja = 4 * (t / 16), kb = 4 * (t % 16);
  float bias[4][4], acc[4][4];
  bool kvalid[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) kvalid[b] = key_ok(a, k0 + kb + b);
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + ja + x, k = k0 + kb + b;
      bias[x][b] = (j < a.N && k < a.N) ? __ldg(a.B + (static_cast<long long>(h) * a.N + j) * a.N + k)
                                        : 0.f;
      acc[x][b] = 0.f;
    }
  for (int r = 0; r < a.rows; ++r) {
    const long long blk = (static_cast<long long>(r) * kHeads + h) * a.N;
    __syncthreads();
    for (int idx = t; idx < kBlk * kD; idx += kBlkThreads) {
      const int row = idx / kD, c = idx % kD;
      const bool jin = j0 + row < a.N, kin = k0 + row < a.N;
      sQ[c][row] = jin ? __ldg(a.Q + (blk + j0 + row) * kD + c) : 0.f;
      sG[c][row] = jin ? __ldg(a.dO + (blk + j0 + row) * kD + c) : 0.f;
      sK[c][row] = kin ? __ldg(a.K + (blk + k0 + row) * kD + c) : 0.f;
      sV[c][row] = kin ? __ldg(a.V + (blk + k0 + row) * kD + c) : 0.f;
    }
    if (t < kBlk) {
      const bool jin = j0 + t < a.N;
      sL[t] = jin ? a.lse[blk + j0 + t] : INFINITY;
      sDj[t] = jin ? a.D[blk + j0 + t] : 0.f;
    }
    __syncthreads();
    float dot[4][4], dp[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int b = 0; b < 4; ++b) dot[x][b] = dp[x][b] = 0.f;
#pragma unroll 8
    for (int c = 0; c < kD; ++c) {
      const float4 q4 = *reinterpret_cast<const float4*>(&sQ[c][ja]);
      const float4 g4 = *reinterpret_cast<const float4*>(&sG[c][ja]);
      const float4 k4 = *reinterpret_cast<const float4*>(&sK[c][kb]);
      const float4 v4 = *reinterpret_cast<const float4*>(&sV[c][kb]);
      const float qx[4] = {q4.x, q4.y, q4.z, q4.w}, gx[4] = {g4.x, g4.y, g4.z, g4.w};
      const float kx[4] = {k4.x, k4.y, k4.z, k4.w}, vx[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          dot[x][b] = fmaf(qx[x], kx[b], dot[x][b]);
          dp[x][b] = fmaf(gx[x], vx[b], dp[x][b]);
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float lse = sL[ja + x], Dj = sDj[ja + x];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float p = kvalid[b] ? expf(fmaf(dot[x][b], kScale, bias[x][b]) - lse) : 0.f;
        acc[x][b] = fmaf(p, dp[x][b] - Dj, acc[x][b]);
      }
    }
  }
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + ja + x, k = k0 + kb + b;
      if (j < a.N && k < a.N) a.dB[(static_cast<long long>(h) * a.N + j) * a.N + k] = acc[x][b];
    }
}

}  // namespace bwd
}  // namespace tri
