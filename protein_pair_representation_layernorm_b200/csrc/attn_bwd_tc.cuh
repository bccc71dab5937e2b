// attn_bwd_tc.cuh — backward pass of the attention core on the tensor cores
// (tcgen05, bf16 operands, fp32 accumulation), and the preparation kernels it
// shares with the bf16 core forward.
//
// The mathematics is that of attn_bwd.cuh (the fp32 SIMT form), written in base
// 2 as the forward kernel works.  Per problem row r, head h, query j and key k:
//   x_jk  = q_j . k_k * log2(e)/sqrt(d) + b_h(j, k) * log2(e)   (masked key: -3e38)
//   p_jk  = 2^(x_jk - lse2_j),  lse2_j = log2 sum_k 2^x_jk  (the forward's row statistic)
//   D_j   = dO_j . o_j,   ds_jk = p_jk (dO_j . v_k - D_j)
//   dQ_j  = sum_k ds_jk k_k / sqrt(d),   dK_k = sum_j ds_jk q_j / sqrt(d)
//   dV_k  = sum_j p_jk dO_j,             dB_h(j, k) = sum_r ds_jk.
// (the chain rule through each softmax row; the training context is the
// BioNeMo context-parallelism page's, "Descomposición de sistemas moleculares
// grandes").  Three tensor-core kernels recompute the scores and dP = dO V^T of
// their tiles from the forward's row statistics instead of storing p (an
// R x N x N x H tensor):
//   bwd_rows<kDQ>    CTA = 3 rows x 128 queries x head; walks the keys in tiles
//                    of 64: S = Qs K^T and dP = dO V^T (SS MMAs into TMEM), ds in
//                    the softmax threads (thread = query = TMEM lane), written
//                    back to TMEM as bf16, then dQ += ds K (TS MMA).
//   bwd_rows<kDKDV>  CTA = 2 rows x 128 keys x head; the same walk over the
//                    queries with the roles of queries and keys exchanged:
//                    S^T = K Qs^T, dP^T = V dO^T, thread = key, then
//                    dV += P^T dO and dK += ds^T Qs (two TS MMAs).  The per-query
//                    statistics of each tile come with its stage.  ds and P have
//                    TMEM columns of their own, so the scores of step t+1 are
//                    computed as soon as the threads hold those of step t in
//                    registers, and the gradient MMAs of step t run while they
//                    work on step t+1.
//   bwd_dbias_tc     CTA = (128 queries, 64 keys, head); walks every problem row,
//                    S and dP double-buffered in TMEM, and sums ds in registers:
//                    the bias gradient is written once per element (no atomics,
//                    so the result is deterministic).
// The operands: Qs = bf16(q * log2(e)/sqrt(d)) (the forward's scaled q), the
// caller's bf16 K, V and dO, the base-2 bias b2 (and its transpose for
// bwd_rows<kDKDV>) with the key mask and the padding folded in, and per query
// -lse2 and -D (negated so that the kernels add them), padded with -inf and 0.
// Every wait is bounded (sm100.cuh); on expiry a CTA records
// TRI_ATTN_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace bwdtc {

constexpr int kTM = 128;  // thread rows of a tile (queries; keys in bwd_rows<kDKDV>)
constexpr int kTN = 64;   // columns per step (keys; queries in bwd_rows<kDKDV>)
constexpr float kInvSqrtD = 0.17677669529663687f;  // 1 / sqrt(32)
constexpr float kLn2 = 0.69314718055994531f;

// Leading dimension of the padded bias and per-query buffers: a whole number of
// 128-wide tiles, so every copy of a tile stays inside its buffer.
__host__ __device__ constexpr int padded_ld(int N) { return (N + 127) / 128 * 128; }

// ------------------------------------------------------------------ preparation
// Qs = bf16(Q * log2(e) / sqrt(d)), 8 elements (16 bytes) per step.
__global__ void prep_q(const __nv_bfloat16* __restrict__ Q, __nv_bfloat16* __restrict__ Qs,
                       long long n8) {
  const float c = kLog2e * kInvSqrtD;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(Q)[i];
    uint4 w;
    w.x = pack_bf16x2(bf16lo_to_f32(v.x) * c, bf16hi_to_f32(v.x) * c);
    w.y = pack_bf16x2(bf16lo_to_f32(v.y) * c, bf16hi_to_f32(v.y) * c);
    w.z = pack_bf16x2(bf16lo_to_f32(v.z) * c, bf16hi_to_f32(v.z) * c);
    w.w = pack_bf16x2(bf16lo_to_f32(v.w) * c, bf16hi_to_f32(v.w) * c);
    reinterpret_cast<uint4*>(Qs)[i] = w;
  }
}

// b2[h][j][k] = bias[h][j][k] * log2(e) for an unmasked key k < N, the masked
// logit for a masked key and for the padding columns N <= k < ld; rows j < N.
// With b2T: b2T[h][k][j] = b2[h][j][k] for rows k < N and columns j < ld (the
// padding columns j >= N masked too).  Blocks of 32 x 8 threads, one 32 x 32
// (j, k) tile each, transposed through shared memory.
__global__ void prep_bias(const __nv_bfloat16* __restrict__ bias, const uint8_t* __restrict__ mask,
                          int N, int ld, __nv_bfloat16* __restrict__ b2,
                          __nv_bfloat16* __restrict__ b2T) {
  __shared__ float tile[32][33];
  const int h = blockIdx.z, k0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int jj = ty; jj < 32; jj += 8) {
    const int j = j0 + jj, k = k0 + tx;
    float v = kMaskedLogit;
    if (j < N && k < N && (mask == nullptr || mask[k] != 0))
      v = __bfloat162float(bias[(static_cast<long long>(h) * N + j) * N + k]) * kLog2e;
    tile[jj][tx] = v;
    if (j < N && k < ld) b2[(static_cast<long long>(h) * N + j) * ld + k] = __float2bfloat16(v);
  }
  if (b2T != nullptr) {
    __syncthreads();
    for (int kk = ty; kk < 32; kk += 8) {
      const int k = k0 + kk, j = j0 + tx;
      if (k < N && j < ld)
        b2T[(static_cast<long long>(h) * N + k) * ld + j] = __float2bfloat16(tile[tx][kk]);
    }
  }
}

// Per query of every (row, head): nlse2 = -lse * log2(e) and, with dO, nD =
// -(dO . o) in fp32; the padding queries N <= j < ld get -inf (probability 0)
// and 0.  lse = +inf (every key masked) gives -inf as well.
__global__ void prep_rows(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                          const float* __restrict__ lse, long long rh_count, int N, int ld,
                          float* __restrict__ nlse2, float* __restrict__ nD) {
  const long long total = rh_count * ld;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long rh = idx / ld;
    const int j = static_cast<int>(idx - rh * ld);
    if (j < N) {
      const long long q = rh * N + j;
      nlse2[idx] = -lse[q] * kLog2e;
      if (nD != nullptr) {
        const uint4* a = reinterpret_cast<const uint4*>(dO + q * kD);
        const uint4* b = reinterpret_cast<const uint4*>(O + q * kD);
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < kD / 8; ++c) {
          const uint4 x = a[c], y = b[c];
          const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc = fmaf(bf16lo_to_f32(xs[e]), bf16lo_to_f32(ys[e]), acc);
            acc = fmaf(bf16hi_to_f32(xs[e]), bf16hi_to_f32(ys[e]), acc);
          }
        }
        nD[idx] = -acc;
      }
    } else {
      nlse2[idx] = -INFINITY;
      if (nD != nullptr) nD[idx] = 0.f;
    }
  }
}

// ------------------------------------------------------------------ bwd_rows
enum Mode { kDQ = 0, kDKDV = 1 };

struct RowsArgs {
  const float* nlse2;  // [rows][H][ld]
  const float* nD;     // [rows][H][ld]
  float* out1;         // dQ (kDQ) or dK (kDKDV): [rows][H][N][d]
  float* out2;         // dV (kDKDV)
  int N, rows, ld;
  int debug_stall;     // fault injection: the producer of CTA 0 withholds its first stage
  int* status;
};

// A CTA: kR problem rows, 128 thread rows (queries for kDQ, keys for kDKDV).
// Fixed operands A1, A2 (128 x 32 each, per row): Qs and dO (kDQ), K and V
// (kDKDV).  A stage per step of 64 columns: the bias tile shared by the rows
// (128 x 64 bf16, 128-byte swizzle) and per row X1, X2 (64 x 32): K and V
// (kDQ), Qs and dO (kDKDV), plus for kDKDV the step's -lse2 and -D (64 fp32
// each).
// kDKDV (kEarly): 2 rows; TMEM per row S at +0, dP at +64, ds (bf16, 32
// columns) at +128, P (bf16) at +160, dK at +192, dV at +224.  ds and P have
// columns of their own, so the scores of step t+1 are computed while the warps
// still work on step t.
// kDQ: 3 rows; TMEM per row S at +0, dP at +64 (ds as bf16 over its first 32
// columns, each half written after it was read), dQ at +128; the scores of
// step t+1 follow the gradient MMA of step t (measured faster for dQ than 2
// rows with early scores: 1.02 against 1.09 ms per launch at N = 768).
template <int kMode>
struct RowsLayout {
  static constexpr bool kEarly = kMode == kDKDV;
  static constexpr int kR = kEarly ? 2 : 3;
  static constexpr int kRowCols = kEarly ? 256 : 160;
  static constexpr int kColDS = kEarly ? 128 : 64;
  static constexpr int kColP = 160;
  static constexpr int kColAcc = kEarly ? 192 : 128;
  static constexpr int kStages = 4;
  static constexpr int kProducerWarp = 4 * kR;
  static constexpr int kMmaWarp0 = 4 * kR + 1;  // MMA warp of row g: kMmaWarp0 + g
  static constexpr int kThreads = (4 * kR + 1 + kR) * 32;
  static constexpr uint32_t kATile = kTM * kD * 2;   // 8192
  static constexpr uint32_t kXTile = kTN * kD * 2;   // 4096
  static constexpr uint32_t kBTile = kTM * kTN * 2;  // 16384
  static constexpr uint32_t kVecBytes = kMode == kDKDV ? kTN * 4 : 0;
  static constexpr uint32_t kSmemA1 = 0;
  static constexpr uint32_t kSmemA2 = kR * kATile;
  static constexpr uint32_t kSmemStages = 2 * kR * kATile;
  static constexpr uint32_t kStB = 0;
  static constexpr uint32_t kStX1 = kBTile;
  static constexpr uint32_t kStX2 = kBTile + kR * kXTile;
  static constexpr uint32_t kStVec = kBTile + 2 * kR * kXTile;  // [row][nlse2, nD][64]
  static constexpr uint32_t kStageTx = kStVec + 2 * kR * kVecBytes;
  static constexpr uint32_t kStageBytes = (kStageTx + 1023) / 1024 * 1024;
  static constexpr uint32_t kSmemBar = kSmemStages + kStages * kStageBytes;
  // a_full, st_full[S], st_empty[S], s_full[R], s_read[R], ds_full[R], acc_done[R],
  // acc_full[R], drain[R]
  static constexpr uint32_t kNumBars = 1 + 2 * kStages + 6 * kR;
  static constexpr uint32_t kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;
  static_assert(kSmemStages % 1024 == 0 && kStageBytes % 1024 == 0 && kStX1 % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(kR * kRowCols <= 512, "TMEM");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

template <int kMode>
__global__ void __launch_bounds__(RowsLayout<kMode>::kThreads, 1)
    bwd_rows(const __grid_constant__ CUtensorMap map_a1, const __grid_constant__ CUtensorMap map_a2,
             const __grid_constant__ CUtensorMap map_x1, const __grid_constant__ CUtensorMap map_x2,
             const __grid_constant__ CUtensorMap map_b, const RowsArgs a) {
  using L = RowsLayout<kMode>;
  constexpr int kR = L::kR, kStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kSmemBar);
  uint64_t* a_full = bars;
  uint64_t* st_full = a_full + 1;
  uint64_t* st_empty = st_full + kStages;  // one commit per row's MMA warp
  uint64_t* s_full = st_empty + kStages;   // [g]: S(t) and dP(t) of row g in TMEM
  uint64_t* s_read = s_full + kR;          // [g]: the warps of row g hold S(t), dP(t) in registers
  uint64_t* ds_full = s_read + kR;         // [g]: ds(t) (and P(t)) of row g in TMEM
  uint64_t* acc_done = ds_full + kR;       // [g]: the gradient MMAs of step t have read ds(t), P(t)
  uint64_t* acc_full = acc_done + kR;      // [g]: every MMA of row g complete
  uint64_t* drain = acc_full + kR;         // [g]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kTM;  // first thread row of the tile
  const int rg = blockIdx.y;        // group of kR problem rows
  const int h = blockIdx.z;
  const int T = (a.N + kTN - 1) / kTN;

  if (tid == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], kR);
    }
    for (int g = 0; g < kR; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_read[g], 4);
      mbar_init(&ds_full[g], 4);
      mbar_init(&acc_done[g], 1);
      mbar_init(&acc_full[g], 1);
      mbar_init(&drain[g], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == L::kMmaWarp0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == L::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_a1);
      tma_prefetch_desc(&map_a2);
      tma_prefetch_desc(&map_x1);
      tma_prefetch_desc(&map_x2);
      tma_prefetch_desc(&map_b);
      mbar_arrive_expect_tx(a_full, 2 * kR * L::kATile);
      for (int r = 0; r < kR; ++r) {
        const int c2 = (rg * kR + r) * kHeads + h;
        tma_load_3d(smem + L::kSmemA1 + r * L::kATile, &map_a1, a_full, 0, m0, c2);
        tma_load_3d(smem + L::kSmemA2 + r * L::kATile, &map_a2, a_full, 0, m0, c2);
      }
      const bool stall = a.debug_stall && blockIdx.x == 0 && rg == 0 && h == 0;
      int t_end = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % kStages;
        if (t >= kStages && !mbar_wait(&st_empty[s], ((t / kStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          report_status(a.status, kStatusTimeout);
          break;
        }
        t_end = t + 1;
        if (stall && t == 0) continue;  // fault injection: stage 0 is never filled
        uint8_t* st = smem + L::kSmemStages + s * L::kStageBytes;
        mbar_arrive_expect_tx(&st_full[s], L::kStageTx);
        tma_load_3d(st + L::kStB, &map_b, &st_full[s], t * kTN, m0, h);
        for (int r = 0; r < kR; ++r) {
          const int c2 = (rg * kR + r) * kHeads + h;
          tma_load_3d(st + L::kStX1 + r * L::kXTile, &map_x1, &st_full[s], 0, t * kTN, c2);
          tma_load_3d(st + L::kStX2 + r * L::kXTile, &map_x2, &st_full[s], 0, t * kTN, c2);
          if constexpr (kMode == kDKDV) {
            // a row past the last one reads the last row's statistics (its
            // results are never stored; the copy stays inside the buffers)
            const int row = min(rg * kR + r, a.rows - 1);
            const long long off = (static_cast<long long>(row) * kHeads + h) * a.ld + t * kTN;
            bulk_load(st + L::kStVec + (2 * r) * L::kVecBytes, a.nlse2 + off, L::kVecBytes,
                      &st_full[s]);
            bulk_load(st + L::kStVec + (2 * r + 1) * L::kVecBytes, a.nD + off, L::kVecBytes,
                      &st_full[s]);
          }
        }
      }
      // never leave a copy in flight into this CTA's shared memory
      if (!mbar_wait(a_full, 0, nullptr)) report_status(a.status, kStatusTimeout);
      for (int s = 0; s < kStages; ++s) {
        int last = -1;
        for (int t = s; t < t_end; t += kStages)
          if (!(stall && t == 0)) last = t;
        if (last >= 0 && !mbar_wait(&st_full[s], (last / kStages) & 1, nullptr))
          report_status(a.status, kStatusTimeout);
      }
    }
    __syncwarp();
  } else if (warp >= L::kMmaWarp0) {
    // ------------------------------------------------------------ MMA issuer of row g
    const int g = warp - L::kMmaWarp0;
    if (lane == 0) {
      constexpr uint32_t kIdSS = idesc_bf16_f32(128, kTN, false);  // N = 64, B K-major
      constexpr uint32_t kIdTS = idesc_bf16_f32(128, kD, true);    // N = 32, B MN-major
      const uint64_t dA = smem_desc(smem_u32(smem), 512, kSwizzle64B);
      const uint64_t dSt = smem_desc(smem_u32(smem + L::kSmemStages), 512, kSwizzle64B);
      const uint32_t a_lo = static_cast<uint32_t>(dA), st_lo = static_cast<uint32_t>(dSt);
      const uint64_t a_hi = dA & 0xFFFFFFFF00000000ull, st_hi = dSt & 0xFFFFFFFF00000000ull;
      auto adesc = [&](uint32_t off) { return a_hi | (a_lo + (off >> 4)); };
      auto sdesc = [&](uint32_t off) { return st_hi | (st_lo + (off >> 4)); };
      const uint32_t tS = tmem + g * L::kRowCols, tDP = tS + 64;
      const uint32_t tDS = tS + L::kColDS, tP = tS + L::kColP, tAcc = tS + L::kColAcc;
      // S = A1 X1^T and dP = A2 X2^T of stage s (K = 32: two K = 16 steps each)
      auto issue_sdp = [&](int s) {
#pragma unroll
        for (int kc = 0; kc < kD / 16; ++kc)
          mma_ss(tS, adesc(L::kSmemA1 + g * L::kATile + kc * 32),
                 sdesc(s * L::kStageBytes + L::kStX1 + g * L::kXTile + kc * 32), kIdSS,
                 kc > 0 ? 1u : 0u);
#pragma unroll
        for (int kc = 0; kc < kD / 16; ++kc)
          mma_ss(tDP, adesc(L::kSmemA2 + g * L::kATile + kc * 32),
                 sdesc(s * L::kStageBytes + L::kStX2 + g * L::kXTile + kc * 32), kIdSS,
                 kc > 0 ? 1u : 0u);
        mma_commit(&s_full[g]);
      };
      // acc1 += ds X1 (dQ += ds K; dK += ds^T Qs) and, for kDKDV, acc2 += P X2
      // (dV += P^T dO): A from TMEM (64 bf16 columns = 32 TMEM columns, four
      // K = 16 steps), B the stage's X tile read MN-major
      auto issue_acc = [&](int s, bool first) {
#pragma unroll
        for (int kc = 0; kc < kTN / 16; ++kc)
          mma_ts(tAcc, tDS + kc * 8,
                 sdesc(s * L::kStageBytes + L::kStX1 + g * L::kXTile + kc * 1024), kIdTS,
                 (!first || kc > 0) ? 1u : 0u);
        if constexpr (kMode == kDKDV) {
#pragma unroll
          for (int kc = 0; kc < kTN / 16; ++kc)
            mma_ts(tAcc + 32, tP + kc * 8,
                   sdesc(s * L::kStageBytes + L::kStX2 + g * L::kXTile + kc * 1024), kIdTS,
                   (!first || kc > 0) ? 1u : 0u);
        }
        mma_commit(&acc_done[g]);
        mma_commit(&st_empty[s]);  // this row's MMAs on stage s
      };
      bool ok = mbar_wait(a_full, 0, abort_flag) && mbar_wait(&st_full[0], 0, abort_flag);
      bool issued = false;
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
        issued = true;
      }
      for (int t = 0; ok && t < T; ++t) {
        if constexpr (L::kEarly) {
          if (t + 1 < T) {
            // S(t+1), dP(t+1) as soon as the warps hold S(t), dP(t) in registers
            const int s1 = (t + 1) % kStages;
            if (!(ok = mbar_wait(&st_full[s1], ((t + 1) / kStages) & 1, abort_flag))) break;
            if (!(ok = mbar_wait(&s_read[g], t & 1, abort_flag))) break;
            tc_fence_after();
            issue_sdp(s1);
          }
          // the gradient products of step t once ds(t) (and P(t)) are in TMEM
          if (!(ok = mbar_wait(&ds_full[g], t & 1, abort_flag))) break;
          tc_fence_after();
          issue_acc(t % kStages, t == 0);
        } else {
          // the gradient product of step t reads ds(t) over dP's columns; S and
          // dP of step t+1 overwrite them after it (one thread's MMAs run in order)
          if (!(ok = mbar_wait(&ds_full[g], t & 1, abort_flag))) break;
          tc_fence_after();
          issue_acc(t % kStages, t == 0);
          if (t + 1 < T) {
            const int s1 = (t + 1) % kStages;
            if (!(ok = mbar_wait(&st_full[s1], ((t + 1) / kStages) & 1, abort_flag))) break;
            tc_fence_after();
            issue_sdp(s1);
          }
        }
      }
      if (ok) mma_commit(&acc_full[g]);
      if (!ok) {
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
    // ------------------------------------------------------------ softmax-gradient warps
    const int g = warp >> 2;            // row of the CTA
    const int quad = warp & 3;          // TMEM lane quadrant
    const int ml = quad * 32 + lane;    // thread row within the tile
    const int m = m0 + ml;
    const int row = rg * kR + g;
    const uint32_t tS = tmem + (static_cast<uint32_t>(quad * 32) << 16) + g * L::kRowCols;
    // kDQ: this query's statistics, fixed for the whole walk
    float nl = -INFINITY, nd = 0.f;
    if constexpr (kMode == kDQ) {
      if (row < a.rows && m < a.N) {
        const long long off = (static_cast<long long>(row) * kHeads + h) * a.ld + m;
        nl = a.nlse2[off];
        nd = a.nD[off];
      }
    }
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
      const uint8_t* st = smem + L::kSmemStages + s * L::kStageBytes;
      // bias row ml of the tile: 64 bf16 in a 128-byte swizzled row (16-byte
      // chunk c at position c ^ (ml % 8))
      const uint8_t* brow = st + L::kStB + ml * 128;
      const float* vl = reinterpret_cast<const float*>(st + L::kStVec + 2 * g * L::kVecBytes);
      const float* vd = reinterpret_cast<const float*>(st + L::kStVec + (2 * g + 1) * L::kVecBytes);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tS + 32 * half, sr);
        tmem_ld32(tS + 64 + 32 * half, dr);
        uint32_t bw[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(brow + (((half * 4 + c) ^ (ml & 7)) << 4));
          bw[4 * c] = v.x;
          bw[4 * c + 1] = v.y;
          bw[4 * c + 2] = v.z;
          bw[4 * c + 3] = v.w;
        }
        tmem_ld_wait();
        tmem_regs_ready(sr);
        tmem_regs_ready(dr);
        if (L::kEarly && half == 1) {
          // S(t) and dP(t) are in registers: the MMAs of step t+1 may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_read[g]);
        }
        uint32_t pds[16], pp[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float2 l2, d2;
          if constexpr (kMode == kDQ) {
            l2 = make_float2(nl, nl);
            d2 = make_float2(nd, nd);
          } else {
            l2 = *reinterpret_cast<const float2*>(vl + 32 * half + 2 * e);
            d2 = *reinterpret_cast<const float2*>(vd + 32 * half + 2 * e);
          }
          const float2 x = add_bf16x2_f32x2(
              bw[e], make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])));
          const float2 dl = __fadd2_rn(x, l2);
          // one pair in four on the FMA pipe, the rest on the exp2 unit
          const float2 p = (e % 4 == 3) ? exp2_poly2(dl)
                                        : make_float2(ex2_approx(dl.x), ex2_approx(dl.y));
          const float2 gd = __fadd2_rn(
              make_float2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])), d2);
          const float2 ds = __fmul2_rn(p, gd);
          pds[e] = pack_bf16x2(ds.x, ds.y);
          if constexpr (kMode == kDKDV) pp[e] = pack_bf16x2(p.x, p.y);
        }
        if (L::kEarly && half == 0 && t > 0) {
          // ds and P of step t-1 must have been read by its gradient MMAs
          if (!__all_sync(0xffffffffu, mbar_wait(&acc_done[g], (t - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st16(tS + L::kColDS + 16 * half, pds);
        if constexpr (kMode == kDKDV) tmem_st16(tS + L::kColP + 16 * half, pp);
      }
      if (!ok) break;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[g]);
    }
    // ---- epilogue: the accumulators to fp32 outputs
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[g], 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const bool live = row < a.rows && m < a.N;
      const long long orow = ((static_cast<long long>(row) * kHeads + h) * a.N + m) * kD;
      uint32_t v[32];
      tmem_ld32(tS + L::kColAcc, v);
      tmem_ld_wait();
      tmem_regs_ready(v);
      // dQ = (ds K) / sqrt(d);  dK = (ds^T Qs) / (log2(e)/sqrt(d) * sqrt(d)) = ln 2 (ds^T Qs)
      const float sc = kMode == kDQ ? kInvSqrtD : kLn2;
      if (live) {
        float4* dst = reinterpret_cast<float4*>(a.out1 + orow);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(__uint_as_float(v[4 * q]) * sc, __uint_as_float(v[4 * q + 1]) * sc,
                               __uint_as_float(v[4 * q + 2]) * sc, __uint_as_float(v[4 * q + 3]) * sc);
      }
      if constexpr (kMode == kDKDV) {
        tmem_ld32(tS + L::kColAcc + 32, v);
        tmem_ld_wait();
        tmem_regs_ready(v);
        if (live) {
          float4* dst = reinterpret_cast<float4*>(a.out2 + orow);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                 __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
      }
    } else if (lane == 0) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kMmaWarp0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ bwd_dbias_tc
struct DbiasArgs {
  const float* nlse2;  // [rows][H][ld]
  const float* nD;     // [rows][H][ld]
  float* dB;           // [H][N][N]
  int N, rows, ld;
  int debug_stall;     // fault injection: the producer of CTA 0 withholds its first stage
  int* status;
};

// A CTA: queries j0..j0+127, keys k0..k0+63, one head, every problem row.  The
// bias tile is loaded once; a stage per row holds Qs_r and dO_r (128 x 32), K_r
// and V_r (64 x 32) and the 128 queries' -lse2 and -D.  S and dP of row r go to
// TMEM buffer r % 2 (S at +0, dP at +64), so the MMAs of row r+1 run while the
// softmax-gradient warps work on row r.  Two CTAs share an SM.
constexpr int kDbStages = 3;
constexpr int kDbThreads = 192;  // warps 0-3 softmax gradient, 4 producer, 5 MMA issuer
constexpr int kDbProducerWarp = 4, kDbMmaWarp = 5;
constexpr uint32_t kDbATile = kTM * kD * 2;  // 8192
constexpr uint32_t kDbXTile = kTN * kD * 2;  // 4096
constexpr uint32_t kDbStQ = 0, kDbStO = kDbATile, kDbStK = 2 * kDbATile,
                   kDbStV = 2 * kDbATile + kDbXTile, kDbStVec = 2 * kDbATile + 2 * kDbXTile;
constexpr uint32_t kDbStageTx = kDbStVec + 2 * kTM * 4;  // 25600
constexpr uint32_t kDbStageBytes = (kDbStageTx + 1023) / 1024 * 1024;
constexpr uint32_t kDbSmemStages = kTM * kTN * 2;  // after the 16 KB bias tile
constexpr uint32_t kDbSmemBar = kDbSmemStages + kDbStages * kDbStageBytes;
// b_full, st_full[S], st_empty[S], s_full[2], s_free[2], drain
constexpr uint32_t kDbNumBars = 1 + 2 * kDbStages + 2 + 2 + 1;
constexpr uint32_t kDbSmemBytes = kDbSmemBar + kDbNumBars * 8 + 16 + 1024;
constexpr uint32_t kDbTmemCols = 256;
static_assert(kDbStageBytes % 1024 == 0 && kDbSmemStages % 1024 == 0, "tile alignment");
static_assert(2 * (kDbSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");

__global__ void __launch_bounds__(kDbThreads, 2)
    bwd_dbias_tc(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_o,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                 const __grid_constant__ CUtensorMap map_b, const DbiasArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDbSmemBar);
  uint64_t* b_full = bars;
  uint64_t* st_full = b_full + 1;
  uint64_t* st_empty = st_full + kDbStages;  // MMA commit + one arrive per softmax warp
  uint64_t* s_full = st_empty + kDbStages;   // [buffer]
  uint64_t* s_free = s_full + 2;             // [buffer]: the softmax warps have read it
  uint64_t* drain = s_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kDbNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.x * kTN, j0 = blockIdx.y * kTM, h = blockIdx.z;
  const int R = a.rows;

  if (tid == 0) {
    mbar_init(b_full, 1);
    for (int s = 0; s < kDbStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1 + 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kDbMmaWarp) {
    tmem_alloc(tmem_slot, kDbTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kDbProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_o);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_b);
      mbar_arrive_expect_tx(b_full, kTM * kTN * 2);
      tma_load_3d(smem, &map_b, b_full, k0, j0, h);
      const bool stall = a.debug_stall && blockIdx.x == 0 && blockIdx.y == 0 && h == 0;
      int r_end = 0;
      for (int r = 0; r < R; ++r) {
        const int s = r % kDbStages;
        if (r >= kDbStages && !mbar_wait(&st_empty[s], ((r / kDbStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          report_status(a.status, kStatusTimeout);
          break;
        }
        r_end = r + 1;
        if (stall && r == 0) continue;  // fault injection: stage 0 is never filled
        uint8_t* st = smem + kDbSmemStages + s * kDbStageBytes;
        const int c2 = r * kHeads + h;
        const long long voff = static_cast<long long>(c2) * a.ld + j0;
        mbar_arrive_expect_tx(&st_full[s], kDbStageTx);
        tma_load_3d(st + kDbStQ, &map_q, &st_full[s], 0, j0, c2);
        tma_load_3d(st + kDbStO, &map_o, &st_full[s], 0, j0, c2);
        tma_load_3d(st + kDbStK, &map_k, &st_full[s], 0, k0, c2);
        tma_load_3d(st + kDbStV, &map_v, &st_full[s], 0, k0, c2);
        bulk_load(st + kDbStVec, a.nlse2 + voff, kTM * 4, &st_full[s]);
        bulk_load(st + kDbStVec + kTM * 4, a.nD + voff, kTM * 4, &st_full[s]);
      }
      if (!mbar_wait(b_full, 0, nullptr)) report_status(a.status, kStatusTimeout);
      for (int s = 0; s < kDbStages; ++s) {
        int last = -1;
        for (int r = s; r < r_end; r += kDbStages)
          if (!(stall && r == 0)) last = r;
        if (last >= 0 && !mbar_wait(&st_full[s], (last / kDbStages) & 1, nullptr))
          report_status(a.status, kStatusTimeout);
      }
    }
    __syncwarp();
  } else if (warp == kDbMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdSS = idesc_bf16_f32(128, kTN, false);
      const uint64_t dSt = smem_desc(smem_u32(smem + kDbSmemStages), 512, kSwizzle64B);
      const uint32_t st_lo = static_cast<uint32_t>(dSt);
      const uint64_t st_hi = dSt & 0xFFFFFFFF00000000ull;
      auto sdesc = [&](uint32_t off) { return st_hi | (st_lo + (off >> 4)); };
      bool ok = true, issued = false;
      for (int r = 0; r < R; ++r) {
        const int s = r % kDbStages, b = r & 1;
        if (!(ok = mbar_wait(&st_full[s], (r / kDbStages) & 1, abort_flag))) break;
        if (r >= 2 && !(ok = mbar_wait(&s_free[b], ((r >> 1) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t base = s * kDbStageBytes;
        const uint32_t tS = tmem + 128 * b;
#pragma unroll
        for (int kc = 0; kc < kD / 16; ++kc)
          mma_ss(tS, sdesc(base + kDbStQ + kc * 32), sdesc(base + kDbStK + kc * 32), kIdSS,
                 kc > 0 ? 1u : 0u);
#pragma unroll
        for (int kc = 0; kc < kD / 16; ++kc)
          mma_ss(tS + 64, sdesc(base + kDbStO + kc * 32), sdesc(base + kDbStV + kc * 32), kIdSS,
                 kc > 0 ? 1u : 0u);
        mma_commit(&s_full[b]);
        mma_commit(&st_empty[s]);
        issued = true;
      }
      if (!ok) {
        *abort_flag = 1;
        report_status(a.status, kStatusTimeout);
      }
      if (issued) {  // no MMA of this CTA may be in flight when TMEM is freed
        mma_commit(drain);
        if (!mbar_wait(drain, 0, nullptr)) report_status(a.status, kStatusTimeout);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax-gradient warps
    const int jl = warp * 32 + lane;  // query within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint8_t* brow = smem + jl * 128;
    float2 acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = make_float2(0.f, 0.f);
    bool ok = __all_sync(0xffffffffu, mbar_wait(b_full, 0, abort_flag));
    for (int r = 0; ok && r < R; ++r) {
      const int s = r % kDbStages, b = r & 1;
      bool w = mbar_wait(&s_full[b], (r >> 1) & 1, abort_flag);
      w = w && mbar_wait(&st_full[s], (r / kDbStages) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t* st = smem + kDbSmemStages + s * kDbStageBytes;
      const float nl = reinterpret_cast<const float*>(st + kDbStVec)[jl];
      const float nd = reinterpret_cast<const float*>(st + kDbStVec + kTM * 4)[jl];
      __syncwarp();
      if (lane == 0) mbar_arrive(&st_empty[s]);  // this warp is done with the stage
      const float2 l2 = make_float2(nl, nl), d2 = make_float2(nd, nd);
      const uint32_t tS = tmem + lane_base + 128 * b;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tS + 32 * half, sr);
        tmem_ld32(tS + 64 + 32 * half, dr);
        uint32_t bw[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(brow + (((half * 4 + c) ^ (jl & 7)) << 4));
          bw[4 * c] = v.x;
          bw[4 * c + 1] = v.y;
          bw[4 * c + 2] = v.z;
          bw[4 * c + 3] = v.w;
        }
        tmem_ld_wait();
        tmem_regs_ready(sr);
        tmem_regs_ready(dr);
        if (half == 1) {
          // both halves of this buffer are in registers: the MMAs of row r+2 may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[b]);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x = add_bf16x2_f32x2(
              bw[e], make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])));
          const float2 dl = __fadd2_rn(x, l2);
          const float2 p = (e % 4 == 3) ? exp2_poly2(dl)
                                        : make_float2(ex2_approx(dl.x), ex2_approx(dl.y));
          const float2 gd = __fadd2_rn(
              make_float2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])), d2);
          acc[16 * half + e] = __ffma2_rn(p, gd, acc[16 * half + e]);
        }
      }
    }
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        report_status(a.status, kStatusTimeout);
      }
    } else {
      const int j = j0 + jl;
      if (j < a.N) {
        float* dst = a.dB + (static_cast<long long>(h) * a.N + j) * a.N + k0;
        if ((a.N & 3) == 0 && k0 + kTN <= a.N) {
#pragma unroll
          for (int q = 0; q < kTN / 4; ++q)
            reinterpret_cast<float4*>(dst)[q] =
                make_float4(acc[2 * q].x, acc[2 * q].y, acc[2 * q + 1].x, acc[2 * q + 1].y);
        } else {
#pragma unroll
          for (int e = 0; e < kTN / 2; ++e) {
            if (k0 + 2 * e < a.N) dst[2 * e] = acc[e].x;
            if (k0 + 2 * e + 1 < a.N) dst[2 * e + 1] = acc[e].y;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDbMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kDbTmemCols);
  }
}
}  // namespace bwdtc
}  // namespace tri
