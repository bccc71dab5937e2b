// tri_attn_fwd.cuh — flash-style pair-biased triangle attention on tcgen05.
//
// Problem (per problem row i, head h, in the canonical starting-node frame;
// the ending-node block runs the same kernel on the swapped view produced by
// pair_ln_proj):
//     o_ij = sum_k softmax_k( q_ij . k_ik + b_h(j, k) ) v_ik
// with q already scaled by log2(e)/sqrt(d) and b by log2(e), so the softmax is
// taken in base 2.  Scores are never written to memory: each CTA walks the keys
// in tiles of 64 with an online softmax (the on-chip counterpart of the ring
// attention with K/V blocks arriving one by one, Design-CP technical summary,
// §Metodología 1).
//
// CTA work unit: 4 rows i (i0..i0+3) x 128 queries j (j0..j0+127) x one head.
// The 4 rows share every bias tile b_h(j0.., k-tile), which is loaded once per
// CTA; K and V differ per row.
//
// Warp roles (576 threads):
//   warps 4r..4r+3  softmax group r = row i0+r (thread = query j = TMEM lane j)
//   warp 16         TMA producer: Q once; per key tile K, V of the 4 rows + the bias tile
//   warp 17         MMA issuer (one thread): S_r = Q_r K_r^T (M=128, N=64, K=32),
//                   O_r += P_r V_r (M=128, N=32, K=64, P read from TMEM)
// TMEM (512 columns): S_r/P_r at columns 64r (fp32 scores, bf16 P aliased over
// the first 32 columns), O_r at 256 + 32r.
// Pipeline: 3 shared-memory stages of {K[4][64][32], V[4][64][32], bias[128][64]}.
// The four softmax groups interleave with the tensor core: while a group turns
// its S into P, the MMA warp runs the other groups' PV and next QK.
//
// The exponentials are the binding resource (the special-function unit does 16
// per clock per SM, against 8192 MMA flops; at d = 32 each score needs one
// exponential per 128 flops).  A compile-time fraction of them (kEmuEvery) is
// evaluated on the FMA pipe instead: 2^x = 2^n * 2^f with n = round(x) (Cody-Waite
// range reduction, n obtained by the 1.5 * 2^23 rounding constant) and 2^f, |f| <= 1/2,
// from a degree-3 polynomial fitted here for minimal relative error (7.5e-5, below
// the 2^-9 of the bf16 P it feeds); 2^n is applied by adding n to the exponent
// field of the polynomial value.
//
// Online softmax per (row, query): the running offset m is raised only when a
// tile's maximum exceeds it by more than kTau (log2 units), so the O rescale in
// TMEM is rare; p = 2^(s - m) is then at most 2^kTau.  The offset starts at a
// finite floor so fully-masked tiles (bias -inf) give p = 0, never NaN.  A row
// whose keys are all masked ends with l = 0 and writes o = 0.
//
// Every mbarrier wait is bounded (sm100.cuh); on expiry the CTA records
// TRI_ATTN_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace attn {

constexpr int kBJ = 128;          // queries per CTA
constexpr int kBK = 64;           // keys per step
constexpr int kRows = 4;          // problem rows per CTA
constexpr int kGroups = 4;        // softmax warpgroups, one row each
constexpr int kStages = 3;
// 18 warps: 16 softmax + producer + MMA issuer.  Five of them share one SM
// sub-partition (16K registers), which caps the kernel at 96 registers per thread.
constexpr int kThreads = (4 * kGroups + 2) * 32;
constexpr int kProducerWarp = 4 * kGroups;
constexpr int kMmaWarp = 4 * kGroups + 1;
#ifndef TRI_ATTN_EMU_EVERY
#define TRI_ATTN_EMU_EVERY 0
#endif
constexpr int kEmuEvery = TRI_ATTN_EMU_EVERY;  // every kEmuEvery-th pair of scores: FMA exp2
constexpr float kTau = 8.0f;
constexpr float kFloor = -1.0e30f;

constexpr uint32_t kQTileBytes = kBJ * kD * 2;          // 8192 (128 rows x 64 B)
constexpr uint32_t kKVTileBytes = kBK * kD * 2;         // 4096 (64 rows x 64 B)
constexpr uint32_t kBiasTileBytes = kBJ * kBK * 2;      // 16384 (128 rows x 128 B)
constexpr uint32_t kStageK = 0;
constexpr uint32_t kStageV = kRows * kKVTileBytes;      // 16384
constexpr uint32_t kStageB = 2 * kRows * kKVTileBytes;  // 32768
constexpr uint32_t kStageBytes = kStageB + kBiasTileBytes;  // 49152
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemStages = kRows * kQTileBytes;       // 32768
constexpr uint32_t kSmemBar = kSmemStages + kStages * kStageBytes;
constexpr uint32_t kNumBars = 1 + 2 * kStages + 2 * kGroups + 2;
constexpr uint32_t kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // + 64 r
constexpr uint32_t kColO = 256;    // + 32 r

struct Maps {
  CUtensorMap q, k, v, bias;
};

__global__ void __launch_bounds__(kThreads, 1)
    tri_attn_fwd(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
           const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_b,
           const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* q_full = bars;
  uint64_t* st_full = bars + 1;
  uint64_t* st_empty = st_full + kStages;
  uint64_t* s_full = st_empty + kStages;
  uint64_t* p_full = s_full + kGroups;
  uint64_t* o_full = p_full + kGroups;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int jt = blockIdx.x;
  const int ig = blockIdx.y;          // group of kRows problem rows
  const int h = blockIdx.z;
  const int j0 = jt * kBJ;
  const int T = (a.N + kBK - 1) / kBK;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1 + kGroups * 4);  // MMA commit + one arrive per softmax warp
    }
    for (int g = 0; g < kGroups; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], 4);
    }
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_b);
      int last_issued[kStages];
      for (int s = 0; s < kStages; ++s) last_issued[s] = -1;
      mbar_arrive_expect_tx(q_full, kRows * kQTileBytes);
      for (int r = 0; r < kRows; ++r)
        tma_load_3d(smem + kSmemQ + r * kQTileBytes, &map_q, q_full, 0, j0,
                    (ig * kRows + r) * kHeads + h);
      const bool stall = a.debug_stall && jt == 0 && ig == 0 && h == 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % kStages;
        if (t >= kStages) {
          if (!mbar_wait(&st_empty[s], ((t / kStages) - 1) & 1, abort_flag)) {
            *abort_flag = 1;
            report_status(a.status, kStatusTimeout);
            break;
          }
        }
        if (stall && t == 0) continue;  // fault injection: stage 0 is never filled
        uint8_t* st = smem + kSmemStages + s * kStageBytes;
        mbar_arrive_expect_tx(&st_full[s], kStageBytes);
        for (int r = 0; r < kRows; ++r) {
          const int c2 = (ig * kRows + r) * kHeads + h;
          tma_load_3d(st + kStageK + r * kKVTileBytes, &map_k, &st_full[s], 0, t * kBK, c2);
          tma_load_3d(st + kStageV + r * kKVTileBytes, &map_v, &st_full[s], 0, t * kBK, c2);
        }
        tma_load_3d(st + kStageB, &map_b, &st_full[s], t * kBK, j0, h);
        last_issued[s] = t;
      }
      // never leave a copy in flight into this CTA's shared memory
      if (!mbar_wait(q_full, 0, nullptr)) report_status(a.status, kStatusTimeout);
      for (int s = 0; s < kStages; ++s)
        if (last_issued[s] >= 0 && !mbar_wait(&st_full[s], (last_issued[s] / kStages) & 1, nullptr))
          report_status(a.status, kStatusTimeout);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBK, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kD, true);
      const uint32_t sQ = smem_u32(smem + kSmemQ);
      const uint32_t sSt = smem_u32(smem + kSmemStages);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      bool issued = false;
      auto issue_pv = [&](int r, int tt) {
        const uint32_t sV = sSt + (tt % kStages) * kStageBytes + kStageV;
#pragma unroll
        for (int kc = 0; kc < kBK / 16; ++kc) {
          const uint64_t bd = smem_desc(sV + r * kKVTileBytes + kc * 1024, 512, kSwizzle64B);
          mma_ts(tmem + kColO + 32 * r, tmem + kColS + 64 * r + kc * 8, bd, kIdescPV,
                 (tt > 0 || kc > 0) ? 1u : 0u);
        }
      };
      for (int t = 0; ok && t < T; ++t) {
        const int s = t % kStages;
        if (!(ok = mbar_wait(&st_full[s], (t / kStages) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t sK = sSt + s * kStageBytes + kStageK;
        for (int g = 0; g < kGroups; ++g) {
          if (t > 0) {
            if (!(ok = mbar_wait(&p_full[g], (t - 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(g, t - 1);
          }
#pragma unroll
          for (int kc = 0; kc < kD / 16; ++kc) {
            const uint64_t ad = smem_desc(sQ + g * kQTileBytes + kc * 32, 512, kSwizzle64B);
            const uint64_t bd = smem_desc(sK + g * kKVTileBytes + kc * 32, 512, kSwizzle64B);
            mma_ss(tmem + kColS + 64 * g, ad, bd, kIdescQK, kc > 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit(&s_full[g]);
        }
        if (!ok) break;
        if (t > 0) mma_commit(&st_empty[(t - 1) % kStages]);
      }
      if (ok) {
        for (int g = 0; g < kGroups; ++g) {
          if (!(ok = mbar_wait(&p_full[g], (T - 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(g, T - 1);
        }
      }
      if (ok) {
        mma_commit(o_full);
        mma_commit(&st_empty[(T - 1) % kStages]);
      } else {
        *abort_flag = 1;
        report_status(a.status, kStatusTimeout);
        if (issued) {  // wait until no MMA of this CTA is in flight
          mma_commit(drain);
          mbar_wait(drain, 0, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp < kProducerWarp) {
    // ------------------------------------------------------------ softmax
    const int g = warp >> 2;              // softmax group = row of the CTA
    const int quad = warp & 3;            // TMEM lane quadrant
    const int jl = quad * 32 + lane;      // query within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t colS = tmem + lane_base + kColS + 64 * g;
    const uint32_t colO = tmem + lane_base + kColO + 32 * g;
    float m_used = kFloor;
    float l_sum = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % kStages;
      bool w = mbar_wait(&s_full[g], t & 1, abort_flag);
      w = w && mbar_wait(&st_full[s], (t / kStages) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // x = s + b (base-2 logits) in two 32-key halves; tile maximum over four
      // independent chains.  The bias row jl of this key tile is 64 bf16 in a
      // 128-byte swizzled row: 16-byte chunk c sits at position c ^ (jl % 8).
      const uint8_t* brow = smem + kSmemStages + s * kStageBytes + kStageB + jl * 128;
      float2 x[32];
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sr[32];
        tmem_ld32(colS + 32 * half, sr);
        uint32_t bw[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v =
              *reinterpret_cast<const uint4*>(brow + (((half * 4 + c) ^ (jl & 7)) << 4));
          bw[4 * c] = v.x;
          bw[4 * c + 1] = v.y;
          bw[4 * c + 2] = v.z;
          bw[4 * c + 3] = v.w;
        }
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float2& xe = x[half * 16 + e];
          xe = __fadd2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                          make_float2(bf16lo_to_f32(bw[e]), bf16hi_to_f32(bw[e])));
          mx[e & 3] = fmax3(mx[e & 3], xe.x, xe.y);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&st_empty[s]);  // this warp is done with the bias tile
      const float tmax = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      // lazy rescale: raise the offset only when the tile max exceeds it by > kTau
      const bool need = tmax > m_used + kTau;
      float scale = 1.0f;
      if (need) {
        scale = ex2_approx(m_used - tmax);
        l_sum *= scale;
        m_used = tmax;
      }
      if (t > 0 && __any_sync(0xffffffffu, need)) {
        uint32_t ov[32];
        tmem_ld32(colO, ov);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * scale);
        tmem_st32(colO, ov);
      }
      const float2 neg_m = make_float2(-m_used, -m_used);
      float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int quarter = 0; quarter < 4; ++quarter) {
        uint32_t pk[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = quarter * 8 + q;
          const float2 dlt = __fadd2_rn(x[e], neg_m);
          float2 p;
          if (kEmuEvery > 0 && (e % (kEmuEvery > 0 ? kEmuEvery : 1)) == kEmuEvery - 1) {
            p = exp2_poly2(dlt);
          } else {
            p = make_float2(ex2_approx(dlt.x), ex2_approx(dlt.y));
          }
          acc[e & 1] = __fadd2_rn(acc[e & 1], p);
          pk[q] = pack_bf16x2(p.x, p.y);
        }
        tmem_st8(colS + 8 * quarter, pk);
      }
      const float2 a = __fadd2_rn(acc[0], acc[1]);
      l_sum += a.x + a.y;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[g]);
    }
    // ---- epilogue: o = O / l
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int j = j0 + jl;
      const int row = ig * kRows + g;
      uint32_t ov[32];
      tmem_ld32(colO, ov);
      tmem_ld_wait();
      if (row < a.rows && j < a.N) {
        const float inv = l_sum > 0.f ? 1.0f / l_sum : 0.f;
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(
            a.O + ((static_cast<long long>(row) * kHeads + h) * a.N + j) * kD);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    } else if (lane == 0) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn
}  // namespace tri
