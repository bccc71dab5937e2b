// pair_ln_proj.cuh — LayerNorm + fused Q/K/V/gate projection (tcgen05) + logit
// bias, bf16 pair representation.
//
// Persistent CTAs of two independent 128-thread groups.  Each group walks its
// own tiles of 128 pairs of one problem row (pairs (i, j0..j0+127)).  The tile of
// Z arrives by TMA straight into the group's MMA A buffer (K-major, 128-byte
// swizzle: two boxes of 64 channels; the ending-node block reads the swapped
// view, pair (i, j) = Z[j][i], as a box one pair wide and 128 pairs deep).
// Thread t of the group owns pair j0+t:
//   1. reads its 256-byte pair vector from the buffer,
//   2. LayerNorm in fp32 (mean, biased variance, rsqrt),
//   3. the per-head logit bias  Wb x  in fp32 (Wb pre-scaled by log2 e;
//      kMaskedLogit at masked keys and at the padding columns j >= N),
//   4. writes x as bf16 back in place, which makes the buffer the A operand.
// The next tile's TMA is issued as soon as the projection has consumed the
// buffer, so it overlaps the last epilogue.
// One thread of the group then issues the projection D = X W^T in two halves of
// N = 256 (q|k, then v|g), W = [Wq; Wk; Wv; Wg] resident in shared memory for the
// whole kernel, each half accumulating in fp32 in the group's 256 TMEM columns.
// Each thread reads back its TMEM lane; q (scaled by log2(e)/sqrt(d)), k, v and
// sigmoid(g + bg) are written head-major ([rows][H][N][d], bf16): each warp
// stages its 32 pairs' 64-byte rows of one head in shared memory and writes
// them with one TMA store (a contiguous 2 KB block).  While one group runs its MMAs the other normalises or
// stores, so the tensor core, the ALUs and HBM overlap.
//
// This is the HBM-bound step: per pair it reads 256 B and writes 1 KB + 8 B.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace plp {

constexpr int kGroupThreads = 128;
constexpr int kGroupsPerCta = 2;
constexpr int kThreads = kGroupThreads * kGroupsPerCta;
constexpr int kTileM = 128;
constexpr int kNOut = 4 * kHD;                       // q | k | v | g
constexpr uint32_t kWImgBytes = kNOut * kCz * 2;     // 131072
constexpr uint32_t kWAtomBytes = kNOut * 128;        // one 64-element K slab of W
constexpr uint32_t kATileBytes = kTileM * kCz * 2;   // 32768
constexpr uint32_t kAAtomBytes = kTileM * 128;       // 16384
constexpr uint32_t kSmemW = 0;
constexpr uint32_t kSmemA = kWImgBytes;                                  // + grp * kATileBytes
constexpr uint32_t kSmemPar = kSmemA + kGroupsPerCta * kATileBytes;     // fp32 params
constexpr uint32_t kParFloats = kHeads * kCz + 3 * kCz;                 // w_b, gamma, beta, b_g
constexpr uint32_t kSmemStg = kSmemPar + kParFloats * 4;               // per-warp store staging
constexpr uint32_t kStgBytes = 32 * 64;                                 // 32 pairs x 64 B
constexpr uint32_t kSmemBar = kSmemStg + (kThreads / 32) * kStgBytes;
constexpr uint32_t kSmemBytes = kSmemBar + 64 + 1024;                   // + alignment slack
static_assert(kGroupsPerCta * 2 * 8 + 8 + 8 <= 64, "barrier area");
constexpr uint32_t kTmemCols = 512;                                     // 256 per group

__global__ void __launch_bounds__(kThreads, 1)
    pair_ln_proj(const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_q,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                 const __grid_constant__ CUtensorMap map_g, const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_wb = reinterpret_cast<float*>(smem + kSmemPar);
  float* s_gamma = s_wb + kHeads * kCz;
  float* s_beta = s_gamma + kCz;
  float* s_bg = s_beta + kCz;
  uint64_t* w_bar = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* mma_bar = w_bar + 1;                // one per group
  uint64_t* z_full = mma_bar + kGroupsPerCta;   // one per group
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(z_full + kGroupsPerCta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int grp = tid / kGroupThreads;
  const int gt = tid % kGroupThreads;           // pair within the tile = TMEM lane
  const uint32_t bar_id = 1 + grp;
  const bool qkvg = a.write_qkvg != 0;
  uint8_t* sA = smem + kSmemA + grp * kATileBytes;

  for (int idx = tid; idx < kHeads * kCz; idx += kThreads) s_wb[idx] = a.w_b[idx];
  for (int idx = tid; idx < kCz; idx += kThreads) {
    s_gamma[idx] = a.gamma[idx];
    s_beta[idx] = a.beta[idx];
    s_bg[idx] = a.b_g[idx];
  }
  if (tid == 0) {
    mbar_init(w_bar, 1);
    for (int g = 0; g < kGroupsPerCta; ++g) {
      mbar_init(&mma_bar[g], 1);
      mbar_init(&z_full[g], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && qkvg) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot + static_cast<uint32_t>(grp * 256);
  if (tid == 0 && qkvg) {
    mbar_arrive_expect_tx(w_bar, kWImgBytes);
    for (uint32_t off = 0; off < kWImgBytes; off += 32768)
      bulk_load(smem + kSmemW + off, a.w_img + off, 32768, w_bar);
  }

  const int jtiles = (a.N + kTileM - 1) / kTileM;
  const long long ntiles = static_cast<long long>(a.rows) * jtiles;
  const long long stride = static_cast<long long>(gridDim.x) * kGroupsPerCta;
  const uint32_t sA_u32 = smem_u32(sA), sW_u32 = smem_u32(smem + kSmemW);
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, false);
  uint32_t mma_phase = 0;
  bool w_ready = false;
  const bool mma_thread = gt == 0;

  long long tile = static_cast<long long>(blockIdx.x) * kGroupsPerCta + grp;
  // TMA of a tile of Z into this group's A buffer
  auto issue_z = [&](long long t) {
    const int r = static_cast<int>(t / jtiles);
    const int j0 = static_cast<int>(t % jtiles) * kTileM;
    const int i = a.row0 + r;
    const int c1 = a.orient == 0 ? j0 : i, c2 = a.orient == 0 ? i - a.z_row0 : j0;
    mbar_arrive_expect_tx(&z_full[grp], kATileBytes);
    tma_load_3d(sA, &map_z, &z_full[grp], 0, c1, c2);
    tma_load_3d(sA + kAAtomBytes, &map_z, &z_full[grp], 64, c1, c2);
  };
  if (mma_thread) tma_prefetch_desc(&map_z);
  // fault injection: group 0 of CTA 0 never receives its first tile, so its
  // bounded wait below expires and the launch reports TRI_ATTN_ERR_TIMEOUT
  const bool stall = a.debug_stall && blockIdx.x == 0 && grp == 0;
  if (mma_thread && tile < ntiles && !stall) issue_z(tile);
  uint32_t z_phase = 0;
  bool z_pending = tile < ntiles && !stall;
  for (; tile < ntiles; tile += stride) {
    const int r = static_cast<int>(tile / jtiles);
    const int i = a.row0 + r;
    const int j = static_cast<int>(tile % jtiles) * kTileM + gt;
    const bool jv = j < a.N;

    if (!named_barrier_and(bar_id, kGroupThreads, mbar_wait(&z_full[grp], z_phase, abort_flag))) {
      if (gt == 0) report_status(a.status, kStatusTimeout);
      break;
    }
    z_phase ^= 1;
    z_pending = false;
    uint4 zr[16];
#pragma unroll
    for (int c = 0; c < 16; ++c)
      zr[c] = *reinterpret_cast<const uint4*>(sA + (c >> 3) * kAAtomBytes + gt * 128 +
                                              (((c & 7) ^ (gt & 7)) << 4));

    // ---- LayerNorm statistics in fp32: two passes over registers, packed
    // fp32x2 arithmetic on channel pairs, two independent accumulators each
    auto chan2 = [](uint32_t w) { return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w)); };
    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      acc[0] = __fadd2_rn(acc[0], chan2(zr[c].x));
      acc[1] = __fadd2_rn(acc[1], chan2(zr[c].y));
      acc[0] = __fadd2_rn(acc[0], chan2(zr[c].z));
      acc[1] = __fadd2_rn(acc[1], chan2(zr[c].w));
    }
    const float mu = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) * (1.0f / kCz);
    const float2 nmu = make_float2(-mu, -mu);
    acc[0] = acc[1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint32_t w[4] = {zr[c].x, zr[c].y, zr[c].z, zr[c].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 d = __fadd2_rn(chan2(w[e]), nmu);
        acc[e & 1] = __ffma2_rn(d, d, acc[e & 1]);
      }
    }
    const float var = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
    const float rstd = rsqrtf(var * (1.0f / kCz) + a.eps);
    const float2 rstd2 = make_float2(rstd, rstd);

    // ---- normalise, bias dot products, bf16 A tile (parameters read as float4,
    // arithmetic on channel pairs)
    float2 bacc[kHeads] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
    const float4* g4 = reinterpret_cast<const float4*>(s_gamma);
    const float4* b4 = reinterpret_cast<const float4*>(s_beta);
    const float4* w4 = reinterpret_cast<const float4*>(s_wb);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint32_t w[4] = {zr[c].x, zr[c].y, zr[c].z, zr[c].w};
      float2 xv[4];  // channels 8c .. 8c+7 as pairs
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        const float4 gm = g4[2 * c + hq], bt = b4[2 * c + hq];
        const float2 d0 = __fadd2_rn(chan2(w[2 * hq]), nmu);
        const float2 d1 = __fadd2_rn(chan2(w[2 * hq + 1]), nmu);
        xv[2 * hq] = __ffma2_rn(__fmul2_rn(d0, rstd2), make_float2(gm.x, gm.y),
                                make_float2(bt.x, bt.y));
        xv[2 * hq + 1] = __ffma2_rn(__fmul2_rn(d1, rstd2), make_float2(gm.z, gm.w),
                                    make_float2(bt.z, bt.w));
      }
#pragma unroll
      for (int h = 0; h < kHeads; ++h) {
        const float4 wa = w4[(h * kCz) / 4 + 2 * c], wb = w4[(h * kCz) / 4 + 2 * c + 1];
        float2 acc2 = bacc[h];
        acc2 = __ffma2_rn(make_float2(wa.x, wa.y), xv[0], acc2);
        acc2 = __ffma2_rn(make_float2(wa.z, wa.w), xv[1], acc2);
        acc2 = __ffma2_rn(make_float2(wb.x, wb.y), xv[2], acc2);
        acc2 = __ffma2_rn(make_float2(wb.z, wb.w), xv[3], acc2);
        bacc[h] = acc2;
      }
      if (qkvg) {
        // K-major, 128 B swizzle: row gt, 16-byte chunk (c % 8) of K-slab c / 8
        uint8_t* dst = sA + (c >> 3) * kAAtomBytes + gt * 128 + (((c & 7) ^ (gt & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pack_bf16x2(xv[0].x, xv[0].y), pack_bf16x2(xv[1].x, xv[1].y),
                       pack_bf16x2(xv[2].x, xv[2].y), pack_bf16x2(xv[3].x, xv[3].y));
      }
    }
    if (a.write_bias) {
      const bool key_valid = jv && (a.mask == nullptr || a.mask[j] != 0);
      if (j < a.ld_bias) {
#pragma unroll
        for (int h = 0; h < kHeads; ++h)
          a.bias[(static_cast<long long>(h) * a.bias_rows + (i - a.bias_row0)) * a.ld_bias + j] =
              __float2bfloat16_rn(key_valid ? bacc[h].x + bacc[h].y : kMaskedLogit);
      }
    }
    if (!qkvg) {
      // bias only: the buffer is free once every thread of the group has read it
      named_barrier_sync(bar_id, kGroupThreads);
      if (mma_thread && tile + stride < ntiles) {
        issue_z(tile + stride);
        z_pending = true;
      }
      continue;
    }

    fence_proxy_async_smem();
    tc_fence_before();
    named_barrier_sync(bar_id, kGroupThreads);
    tc_fence_after();

    bool ok = true;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      // ---- MMA: D[128 x 256] = X W[half*256 .. half*256+255]^T
      if (mma_thread) {
        bool ready = true;
        if (!w_ready) {
          ready = mbar_wait(w_bar, 0, abort_flag);
          w_ready = ready;
        }
        if (ready) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = smem_desc(sA_u32 + (kk >> 2) * kAAtomBytes + (kk & 3) * 32, 1024,
                                          kSwizzle128B);
            const uint64_t bd = smem_desc(
                sW_u32 + (kk >> 2) * kWAtomBytes + half * 256 * 128 + (kk & 3) * 32, 1024,
                kSwizzle128B);
            mma_ss(tmem, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&mma_bar[grp]);
        } else {
          *abort_flag = 1;
          report_status(a.status, kStatusTimeout);
        }
      }
      const bool done = mbar_wait(&mma_bar[grp], mma_phase, abort_flag);
      mma_phase ^= 1;
      if (!named_barrier_and(bar_id, kGroupThreads, done)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (half == 1 && mma_thread && tile + stride < ntiles) {
        issue_z(tile + stride);  // the A buffer has been consumed by both MMAs
        z_pending = true;
      }

      // ---- epilogue: TMEM lane gt -> two of q, k, v, g of pair j.  Each 32-column
      // chunk (one head of one output) of the warp's 32 pairs is 32 rows of 64 B,
      // contiguous in the head-major output: the warp stages it in shared memory
      // and writes it back with 512-byte coalesced stores.
      const int jw0 = static_cast<int>(tile % jtiles) * kTileM + (warp & 3) * 32;
      uint8_t* stg = smem + kSmemStg + warp * kStgBytes;
      uint32_t v[32], vn[32];
      tmem_ld32(tmem + lane_base, vn);
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = vn[e];
        if (cc + 1 < 8) tmem_ld32(tmem + lane_base + (cc + 1) * 32, vn);  // overlap the next load
        const int part = half * 2 + (cc >> 2), h = cc & 3;
        uint32_t pk[16];
        if (part < 3) {
          const float sc = part == 0 ? a.q_scale : 1.0f;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
        } else {
          // sigmoid(t) = 1/2 + tanh(t/2)/2: one special-function op per value
          const float4* bg4 = reinterpret_cast<const float4*>(s_bg + h * kD);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 bb = bg4[e4];
            const float t0 = __uint_as_float(v[4 * e4]) + bb.x;
            const float t1 = __uint_as_float(v[4 * e4 + 1]) + bb.y;
            const float t2 = __uint_as_float(v[4 * e4 + 2]) + bb.z;
            const float t3 = __uint_as_float(v[4 * e4 + 3]) + bb.w;
            pk[2 * e4] = pack_bf16x2(fmaf(0.5f, tanh_approx(0.5f * t0), 0.5f),
                                     fmaf(0.5f, tanh_approx(0.5f * t1), 0.5f));
            pk[2 * e4 + 1] = pack_bf16x2(fmaf(0.5f, tanh_approx(0.5f * t2), 0.5f),
                                         fmaf(0.5f, tanh_approx(0.5f * t3), 0.5f));
          }
        }
        // The staging buffer is the 64-byte-swizzled image of a 32 x 32 bf16 TMA
        // box (row = lane, 16-byte chunk q at position q ^ ((lane / 2) % 4), which
        // is also conflict-free); lane 0 stores it with one TMA store, which
        // clips the rows past N.  The previous chunk's store must have read the
        // buffer before it is rewritten.
        const int lane = gt & 31;
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(stg + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const CUtensorMap* m = part == 0 ? &map_q : part == 1 ? &map_k : part == 2 ? &map_v : &map_g;
          tma_store_3d(m, stg, 0, jw0, r * kHeads + h);
          bulk_commit();
        }
      }
      tc_fence_before();
      named_barrier_sync(bar_id, kGroupThreads);  // TMEM (and, after the second half, A) reused
      tc_fence_after();
    }
    if (!ok) {
      if (gt == 0) report_status(a.status, kStatusTimeout);
      break;
    }
  }

  // ---- teardown: no bulk copy may still be reading or writing this CTA's smem
  if ((gt & 31) == 0) bulk_wait_all();
  if (tid == 0 && qkvg && !w_ready) {
    if (!mbar_wait(w_bar, 0, nullptr)) report_status(a.status, kStatusTimeout);
  }
  if (mma_thread && z_pending) {
    if (!mbar_wait(&z_full[grp], z_phase, nullptr)) report_status(a.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && qkvg) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, kTmemCols);
  }
}

}  // namespace plp
}  // namespace tri
