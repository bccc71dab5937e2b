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
// CTA work unit: 3 rows i (i0..i0+2) x 128 queries j (j0..j0+127) x one head.
// The 3 rows share every bias tile b_h(j0.., k-tile), which is loaded once per
// CTA; K and V differ per row.
//
// Warp roles (512 threads, four warps per SM sub-partition, so up to 128
// registers per thread):
//   warps 4r..4r+3  softmax group r = row i0+r (thread = query j = TMEM lane j)
//   warp 12         TMA producer: Q once; per key tile K, V of the 3 rows + the bias tile
//   warp 13+r       MMA issuer of row r (one thread): S_r = Q_r K_r^T (M=128, N=64,
//                   K=32) and O_r += P_r V_r (M=128, N=32, K=64, P read from TMEM)
// One issuing thread per row keeps each issuer's instruction stream short (it
// shares a sub-partition with three softmax warps, and the tensor core waits
// on it) and lets a row's MMAs go ahead without waiting for the other rows.
// TMEM (512 columns): per row two S/P buffers of 64 columns at 128r and 128r+64
// (fp32 scores; bf16 P aliased over the first 32 columns of its buffer), O_r at
// 384 + 32r.
//
// Scheduling.  With two S buffers per row the scores of key tile t+1 are
// computed while the softmax works on tile t: as soon as P(t) is written, the
// MMA issuer runs PV(t) and then QK(t+2) into the buffer P(t) occupied, so a
// softmax group finds its next S ready when it finishes the current one and the
// tensor core (which spends ~50 cycles on each of these small MMAs) runs
// alongside the exponentials instead of between them.  4 shared-memory stages
// of {K[3][64][32], V[3][64][32], bias[128][64]} cover the tile in PV, the one
// in the softmax, the one in QK and the one being loaded.
//
// Exponentials: 16 per clock per SM on the special-function unit, one per
// score, which makes that unit the kernel's ceiling at head width 32; one
// pair in four is evaluated on the FMA pipe instead (exp2_poly2: Cody-Waite
// reduction and a degree-3 polynomial fitted to 7.5e-5 relative error, far
// below the bf16 rounding of P): with the bias added by a mixed-precision add
// (one instruction per score) that share measured fastest (5.21 ms at
// N = 1536 against 5.34 with one pair in eight and 5.37 with none).
//
// Online softmax per (row, query): the running offset m is raised only when a
// tile's maximum exceeds it by more than kTau (log2 units), so O is rarely
// rescaled in TMEM (then only after the previous PV has completed, which the
// commit of the QK issued right after it signals); p = 2^(s - m) is at most 2^kTau.  The offset starts
// at a finite floor so fully-masked tiles (bias -3e38) give p = 0, never NaN;
// a row whose keys are all masked ends with l = 0 and writes o = 0 (and, when
// asked for, lse = +inf).
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
constexpr int kRows = 3;          // problem rows per CTA
constexpr int kGroups = kRows;    // softmax warpgroups, one row each
constexpr int kStages = 4;
constexpr int kThreads = (4 * kGroups + 1 + kGroups) * 32;
constexpr int kProducerWarp = 4 * kGroups;
constexpr int kMmaWarp0 = 4 * kGroups + 1;  // MMA warp of row g: kMmaWarp0 + g
constexpr float kTau = 8.0f;
constexpr float kFloor = -1.0e30f;

constexpr uint32_t kQTileBytes = kBJ * kD * 2;          // 8192 (128 rows x 64 B)
constexpr uint32_t kKVTileBytes = kBK * kD * 2;         // 4096 (64 rows x 64 B)
constexpr uint32_t kBiasTileBytes = kBJ * kBK * 2;      // 16384 (128 rows x 128 B)
constexpr uint32_t kStageK = 0;
constexpr uint32_t kStageV = kRows * kKVTileBytes;      // 12288
constexpr uint32_t kStageB = 2 * kRows * kKVTileBytes;  // 24576 (1024-aligned)
constexpr uint32_t kStageBytes = kStageB + kBiasTileBytes;  // 40960
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemStages = kRows * kQTileBytes;       // 24576
constexpr uint32_t kSmemBar = kSmemStages + kStages * kStageBytes;
// q_full, st_full[S], st_empty[S], s_full[R][2], p_full[R][2], o_ready[R], o_full[R], drain[R]
constexpr uint32_t kNumBars = 1 + 2 * kStages + 2 * kGroups + 2 * kGroups + 3 * kGroups;
constexpr uint32_t kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // + 128 r + 64 b
constexpr uint32_t kColO = 384;    // + 32 r
static_assert(kStageB % 1024 == 0 && kStageBytes % 1024 == 0 && kSmemStages % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");

__global__ void __launch_bounds__(kThreads, 1)
    tri_attn_fwd(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_b,
                 const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* q_full = bars;
  uint64_t* st_full = q_full + 1;
  uint64_t* st_empty = st_full + kStages;
  uint64_t* s_full = st_empty + kStages;   // [g][buffer]
  // p_full is per buffer as well: S(t+1) can be ready before every warp of the
  // group has written P(t), so one warp may arrive for tile t+1 while another
  // still works on tile t; with a single barrier that early arrival would count
  // towards tile t's phase.
  uint64_t* p_full = s_full + 2 * kGroups;  // [g][buffer]
  uint64_t* o_ready = p_full + 2 * kGroups;  // [g]: PV(T-2) of row g complete
  uint64_t* o_full = o_ready + kGroups;      // [g]: every MMA of row g complete
  uint64_t* drain = o_full + kGroups;        // [g]
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
      mbar_init(&st_empty[s], kGroups + kGroups * 4);  // one commit per MMA warp, one arrive per softmax warp
    }
    for (int g = 0; g < kGroups; ++g) {
      mbar_init(&s_full[2 * g], 1);
      mbar_init(&s_full[2 * g + 1], 1);
      mbar_init(&p_full[2 * g], 4);
      mbar_init(&p_full[2 * g + 1], 4);
      mbar_init(&o_ready[g], 1);
      mbar_init(&o_full[g], 1);
      mbar_init(&drain[g], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp0) {
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
      mbar_arrive_expect_tx(q_full, kRows * kQTileBytes);
      for (int r = 0; r < kRows; ++r)
        tma_load_3d(smem + kSmemQ + r * kQTileBytes, &map_q, q_full, 0, j0,
                    (ig * kRows + r) * kHeads + h);
      const bool stall = a.debug_stall && jt == 0 && ig == 0 && h == 0;
      int t_end = 0;  // steps 0..t_end-1 were attempted
      for (int t = 0; t < T; ++t) {
        const int s = t % kStages;
        if (t >= kStages) {
          if (!mbar_wait(&st_empty[s], ((t / kStages) - 1) & 1, abort_flag)) {
            *abort_flag = 1;
            report_status(a.status, kStatusTimeout);
            break;
          }
        }
        t_end = t + 1;
        if (stall && t == 0) continue;  // fault injection: stage 0 is never filled
        uint8_t* st = smem + kSmemStages + s * kStageBytes;
        mbar_arrive_expect_tx(&st_full[s], kStageBytes);
        for (int r = 0; r < kRows; ++r) {
          const int c2 = (ig * kRows + r) * kHeads + h;
          tma_load_3d(st + kStageK + r * kKVTileBytes, &map_k, &st_full[s], 0, t * kBK, c2);
          tma_load_3d(st + kStageV + r * kKVTileBytes, &map_v, &st_full[s], 0, t * kBK, c2);
        }
        tma_load_3d(st + kStageB, &map_b, &st_full[s], t * kBK, j0, h);
      }
      // never leave a copy in flight into this CTA's shared memory: wait for the
      // last step issued into each stage
      if (!mbar_wait(q_full, 0, nullptr)) report_status(a.status, kStatusTimeout);
      for (int s = 0; s < kStages; ++s) {
        int last = -1;
        for (int t = s; t < t_end; t += kStages)
          if (!(stall && t == 0)) last = t;
        if (last >= 0 && !mbar_wait(&st_full[s], (last / kStages) & 1, nullptr))
          report_status(a.status, kStatusTimeout);
      }
    }
    __syncwarp();
  } else if (warp >= kMmaWarp0) {
    // ------------------------------------------------------------ MMA issuer of row g
    const int g = warp - kMmaWarp0;
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBK, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kD, true);
      // Descriptors of the Q tiles and of the stage area.  Operands are reached
      // by adding (byte offset >> 4) to the start-address field in the low word
      // (every offset stays inside shared memory, so the 14-bit field never
      // carries into the rest).  The tile loop below is unrolled over the
      // kStages stages so that stage, S buffer, barrier parities and operand
      // offsets are compile-time constants: this thread's instruction issue is
      // on the critical path of its row.
      const uint64_t dQ = smem_desc(smem_u32(smem + kSmemQ), 512, kSwizzle64B);
      const uint64_t dSt = smem_desc(smem_u32(smem + kSmemStages), 512, kSwizzle64B);
      const uint32_t q_lo = static_cast<uint32_t>(dQ), st_lo = static_cast<uint32_t>(dSt);
      const uint64_t q_hi = dQ & 0xFFFFFFFF00000000ull, st_hi = dSt & 0xFFFFFFFF00000000ull;
      auto qdesc = [&](uint32_t off) { return q_hi | (q_lo + (off >> 4)); };
      auto sdesc = [&](uint32_t off) { return st_hi | (st_lo + (off >> 4)); };
      // S(g) = Q_g K_g^T from stage `st` into S buffer `b` of row g
      auto issue_qk = [&](int st, int b) {
        const uint32_t dS = tmem + kColS + 128 * g + 64 * b;
#pragma unroll
        for (int kc = 0; kc < kD / 16; ++kc)
          mma_ss(dS, qdesc(g * kQTileBytes + kc * 32),
                 sdesc(st * kStageBytes + kStageK + g * kKVTileBytes + kc * 32), kIdescQK,
                 kc > 0 ? 1u : 0u);
        mma_commit(&s_full[2 * g + b]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag);
      bool issued = false;
      // prologue: the scores of the first two key tiles (stages 0 and 1, phase 0)
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!ok || t >= T) break;
        if (!(ok = mbar_wait(&st_full[t], 0, abort_flag))) break;
        tc_fence_after();
        issue_qk(t, t);
        issued = true;
      }
      for (int base = 0; ok && base < T; base += kStages) {
        const uint32_t ph = (base / kStages) & 1;  // phase of the stage barriers this round
#pragma unroll
        for (int s = 0; s < kStages; ++s) {
          const int t = base + s;
          if (!ok || t >= T) break;
          const int b = s & 1;                           // S buffer t % 2
          const uint32_t pb = (s >> 1) & 1;              // (t / 2) % 2
          const int s2 = (s + 2) % kStages;              // stage of tile t+2
          const uint32_t ph2 = s + 2 < kStages ? ph : ph ^ 1u;
          {
            if (!(ok = mbar_wait(&p_full[2 * g + b], pb, abort_flag))) break;
            tc_fence_after();
            // O_g += P_g(t) V_g(t), P read from S buffer t % 2
            const uint32_t aP = tmem + kColS + 128 * g + 64 * b;
#pragma unroll
            for (int kc = 0; kc < kBK / 16; ++kc)
              mma_ts(tmem + kColO + 32 * g, aP + kc * 8,
                     sdesc(s * kStageBytes + kStageV + g * kKVTileBytes + kc * 1024), kIdescPV,
                     (t > 0 || kc > 0) ? 1u : 0u);
            // QK(t+2) into the buffer P(t) occupied (issued after the PV that
            // reads it); its commit also tells the softmax that PV(t) is
            // complete.  After the last QK, o_ready carries that signal.
            if (t + 2 < T) {
              if (!(ok = mbar_wait(&st_full[s2], ph2, abort_flag))) break;
              tc_fence_after();
              issue_qk(s2, b);
            } else if (t + 2 == T) {
              mma_commit(&o_ready[g]);
            }
            mma_commit(&st_empty[s]);  // this row's MMAs on stage s
          }
        }
      }
      if (ok) {
        mma_commit(&o_full[g]);
      } else {
        *abort_flag = 1;
        report_status(a.status, kStatusTimeout);
        if (issued) {  // wait until no MMA of this warp is in flight
          mma_commit(&drain[g]);
          mbar_wait(&drain[g], 0, nullptr);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int g = warp >> 2;              // softmax group = row of the CTA
    const int quad = warp & 3;            // TMEM lane quadrant
    const int jl = quad * 32 + lane;      // query within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t colO = tmem + lane_base + kColO + 32 * g;
    float m_used = kFloor;
    float l_sum = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % kStages;
      const uint32_t colS = tmem + lane_base + kColS + 128 * g + 64 * (t & 1);
      bool w = mbar_wait(&s_full[2 * g + (t & 1)], (t >> 1) & 1, abort_flag);
      w = w && mbar_wait(&st_full[s], (t / kStages) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // x = s + b (base-2 logits); tile maximum over four independent chains.
      // The bias row jl of this key tile is 64 bf16 in a 128-byte swizzled row:
      // 16-byte chunk c sits at position c ^ (jl % 8).
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
        tmem_regs_ready(sr);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // s + b with the bf16 bias as the operand of a mixed-precision add (no
          // separate widening of the bias)
          float2& xe = x[half * 16 + e];
          xe = add_bf16x2_f32x2(bw[e],
                                make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])));
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
        // O may only be touched once PV(t-1) has completed: the MMA warp issues
        // QK(t+1) right after PV(t-1) (commit covers both), and after PV(T-2)
        // commits o_ready instead
        uint64_t* pv_done = t + 1 < T ? &s_full[2 * g + ((t + 1) & 1)] : &o_ready[g];
        const uint32_t pv_parity = t + 1 < T ? ((t + 1) >> 1) & 1 : 0;
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done, pv_parity, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t ov[32];
        tmem_ld32(colO, ov);
        tmem_ld_wait();
        tmem_regs_ready(ov);
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
          // the last pair of every 4 on the FMA pipe (exp2_poly2), the rest on
          // the special-function unit, which is the busiest unit of the kernel
          const float2 p = (e % 4 == 3) ? exp2_poly2(dlt)
                                        : make_float2(ex2_approx(dlt.x), ex2_approx(dlt.y));
          acc[e & 1] = __fadd2_rn(acc[e & 1], p);
          pk[q] = pack_bf16x2(p.x, p.y);
        }
        tmem_st8(colS + 8 * quarter, pk);
      }
      const float2 asum = __fadd2_rn(acc[0], acc[1]);
      l_sum += asum.x + asum.y;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[2 * g + (t & 1)]);
    }
    // ---- epilogue: o = O / l
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_full[g], 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int j = j0 + jl;
      const int row = ig * kRows + g;
      uint32_t ov[32];
      tmem_ld32(colO, ov);
      tmem_ld_wait();
      tmem_regs_ready(ov);
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
        // the row's natural-log log-sum-exp, ln 2 * (m + log2 l), for a backward pass
        if (a.lse != nullptr)
          a.lse[(static_cast<long long>(row) * kHeads + h) * a.N + j] =
              l_sum > 0.f ? (m_used + __log2f(l_sum)) * 0.69314718055994531f : INFINITY;
      }
    } else if (lane == 0) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn
}  // namespace tri
