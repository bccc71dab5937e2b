// gate_out.cuh — sigmoid gate, output projection (tcgen05) and residual add,
// bf16 pair representation.
//
// Persistent CTAs walk tiles of 128 pairs (i, j0..j0+127) of one problem row
// through a two-stage pipeline; two groups of four compute warps take the
// tiles in turn, group g always stage g, so that one group's LayerNorm and
// gate arithmetic overlaps the other's MMAs and stores.  A producer warp moves
// each tile in with TMA:
// o (4 head boxes of [128 pairs][32], 64-byte swizzle) and the residual z
// ([128][128], 128-byte swizzle; the ending-node block reads the swapped view,
// pair (i, j) = Z[j][i], as a box that is one pair wide and 128 pairs deep).
// The gate is recomputed here rather than read: g = sigmoid(Wg LayerNorm(z) +
// bg) needs only z, which this kernel reads anyway for the residual, so the
// projection kernel never writes a gate tensor and this kernel never reads one.
// Thread t of a group owns pair j0+t (TMEM lane t).  Both MMA A operands are
// built in TMEM (bf16 pairs, one lane per pair), so z stays untouched in
// shared memory until the residual add:
//   1. x = LayerNorm(z) in fp32 (mean, biased variance, rsqrt), stored to TMEM
//      as bf16;  one thread issues D_g = X Wg^T (8 tcgen05 MMAs, N = 128);
//   2. a = bf16(sigmoid(D_g + bg) * o), stored over D_g as it is read;
//      D_out = A Wo^T (8 MMAs) over X;
//   3. out = D_out + bo + z, written over z and stored with TMA (through the
//      swapped view again for the ending node).
// Wg and Wo stay resident in shared memory; each stage has its own two
// 128-column TMEM accumulators.  Every element of out is read (as z) and
// written by the same CTA, tile by tile, so out may alias Z.
//
// HBM-bound: per pair it reads 512 B (o, z) and writes 256 B.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace gout {

constexpr int kComputeThreads = 128;             // one group: a tile's 128 pairs
constexpr int kGroups = 2;
constexpr int kThreads = kGroups * kComputeThreads + 32;   // + producer warp
constexpr int kProducerWarp = 8;
constexpr int kTileM = 128;
constexpr int kStages = 2;
constexpr uint32_t kWBytes = kCz * kHD * 2;          // 32768: one 128 x 128 weight image
constexpr uint32_t kWAtomBytes = kCz * 128;          // 16384: one 64-element K slab of it
constexpr uint32_t kOHeadBytes = kTileM * kD * 2;    // 8192: [128 pairs][32] bf16
constexpr uint32_t kSlabBytes = kTileM * 128;        // 16384: [128 pairs][64] bf16
constexpr uint32_t kStO = 0;
constexpr uint32_t kStZ = kHeads * kOHeadBytes;      // 32768
constexpr uint32_t kStageBytes = kStZ + 2 * kSlabBytes;  // 65536
constexpr uint32_t kSmemWo = 0;
constexpr uint32_t kSmemWg = kWBytes;
constexpr uint32_t kSmemStages = 2 * kWBytes;
constexpr uint32_t kSmemPar = kSmemStages + kStages * kStageBytes;  // bo, bg, gamma, beta
constexpr uint32_t kSmemBar = kSmemPar + 4 * kCz * 4;
constexpr uint32_t kNumBars = 1 + 4 * kStages;   // w, full[S], empty[S], mma_g[S], mma_o[S]
constexpr uint32_t kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;
constexpr uint32_t kTmemCols = 512;  // per stage: D_g / A (128 columns), X / D_out (128)
static_assert(kStages == kGroups, "group g owns stage g");

// Nine warps: three share a sub-partition's 16K registers, so at most 168 each.
__global__ void __maxnreg__(168)
    gate_out(const __grid_constant__ CUtensorMap map_o, const __grid_constant__ CUtensorMap map_z,
             const __grid_constant__ CUtensorMap map_out, const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_bo = reinterpret_cast<float*>(smem + kSmemPar);
  float* s_bg = s_bo + kCz;
  float* s_gamma = s_bg + kCz;
  float* s_beta = s_gamma + kCz;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* w_bar = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + kStages;
  uint64_t* mma_g = empty + kStages;
  uint64_t* mma_o = mma_g + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int idx = tid; idx < kCz; idx += kThreads) {
    s_bo[idx] = a.b_o[idx];
    s_bg[idx] = a.b_g[idx];
    s_gamma[idx] = a.gamma[idx];
    s_beta[idx] = a.beta[idx];
  }
  if (tid == 0) {
    mbar_init(w_bar, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&mma_g[s], 1);
      mbar_init(&mma_o[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int jtiles = (a.N + kTileM - 1) / kTileM;
  const long long ntiles = static_cast<long long>(a.rows) * jtiles;
  // TMA coordinates of the z / out box of a tile: (channel, column, row) of Z
  auto zcoords = [&](long long tile, int& c1, int& c2) {
    const int r = static_cast<int>(tile / jtiles);
    const int j0 = static_cast<int>(tile % jtiles) * kTileM;
    const int i = a.row0 + r;
    if (a.orient == 0) {
      c1 = j0;
      c2 = i - a.z_row0;
    } else {
      c1 = i;
      c2 = j0;
    }
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_o);
      tma_prefetch_desc(&map_z);
      mbar_arrive_expect_tx(w_bar, 2 * kWBytes);
      bulk_load(smem + kSmemWo, a.wo_img, kWBytes, w_bar);
      bulk_load(smem + kSmemWg, a.wg_img, kWBytes, w_bar);
      // fault injection: CTA 0 never fills its first stage, so the compute
      // threads' bounded wait expires and the launch reports TRI_ATTN_ERR_TIMEOUT
      const bool stall = a.debug_stall && blockIdx.x == 0;
      long long n_issued = 0;
      for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++n_issued) {
        const int s = static_cast<int>(n_issued % kStages);
        if (n_issued >= kStages &&
            !mbar_wait(&empty[s], static_cast<uint32_t>((n_issued / kStages) - 1) & 1,
                       abort_flag)) {
          *abort_flag = 1;
          report_status(a.status, kStatusTimeout);
          break;
        }
        if (stall && n_issued == 0) continue;
        uint8_t* st = smem + kSmemStages + s * kStageBytes;
        const int r = static_cast<int>(tile / jtiles);
        const int j0 = static_cast<int>(tile % jtiles) * kTileM;
        int c1, c2;
        zcoords(tile, c1, c2);
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        for (int h = 0; h < kHeads; ++h)
          tma_load_3d(st + kStO + h * kOHeadBytes, &map_o, &full[s], 0, j0, r * kHeads + h);
        for (int slab = 0; slab < 2; ++slab)
          tma_load_3d(st + kStZ + slab * kSlabBytes, &map_z, &full[s], 64 * slab, c1, c2);
      }
      // never leave a copy in flight into this CTA's shared memory
      if (!mbar_wait(w_bar, 0, nullptr)) report_status(a.status, kStatusTimeout);
      for (long long n = n_issued - kStages; n < n_issued; ++n)
        if (n >= 0 && !(stall && n == 0) &&
            !mbar_wait(&full[n % kStages], static_cast<uint32_t>(n / kStages) & 1, nullptr))
          report_status(a.status, kStatusTimeout);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute
    const int grp = warp >> 2;              // = the stage this group works in
    const uint32_t bar_id = 1 + grp;
    const int gt = tid & (kComputeThreads - 1);  // pair within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sWo = smem_u32(smem + kSmemWo), sWg = smem_u32(smem + kSmemWg);
    // TMEM of the stage: D_g in columns 0..127 (then A, bf16 pairs, in 0..63);
    // X (bf16 pairs) in 128..191, then D_out in 128..255
    const uint32_t t_g = tmem + grp * 256, t_o = t_g + 128;
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);
    auto chan2 = [](uint32_t w) { return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w)); };
    bool w_ready = false, ok = true, stored = false;
    // D[128 x 128] = A (TMEM, bf16 pairs) W^T (W resident, K-major 128-byte
    // swizzle), issued by one thread
    auto issue = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t sW, uint64_t* bar) {
      bool ready = true;
      if (!w_ready) ready = w_ready = mbar_wait(w_bar, 0, abort_flag);
      if (ready) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd =
              smem_desc(sW + (kk >> 2) * kWAtomBytes + (kk & 3) * 32, 1024, kSwizzle128B);
          mma_ts(d_tmem, a_tmem + kk * 8, bd, kIdesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar);
      } else {
        *abort_flag = 1;
        report_status(a.status, kStatusTimeout);
      }
    };
    long long n = grp;  // the CTA's tile counter: tile n goes to stage n % kStages
    for (long long tile = blockIdx.x + grp * static_cast<long long>(gridDim.x); tile < ntiles;
         tile += kGroups * static_cast<long long>(gridDim.x), n += kGroups) {
      const int s = grp;
      const uint32_t ph = static_cast<uint32_t>(n / kStages) & 1;
      uint8_t* st = smem + kSmemStages + s * kStageBytes;
      // 16-byte chunk c (channels 8c .. 8c+7) of this thread's z row
      // bo, bg, gamma, beta (re-derived per tile: read where used, not kept in registers)
      const uint32_t par = opaque_u32(smem_u32(smem + kSmemPar));
      auto ldpar = [&](int which, int ch) { return lds_f4(par + (which * kCz + ch) * 4); };
      auto zchunk = [&](int c) {
        return st + kStZ + (c >> 3) * kSlabBytes + gt * 128 + (((c & 7) ^ (gt & 7)) << 4);
      };
      if (!named_barrier_and(bar_id, kComputeThreads, mbar_wait(&full[s], ph, abort_flag))) {
        ok = false;
        break;
      }
      // ---- x = LayerNorm(z) in fp32 (mean, then the biased variance about it;
      // packed fp32x2 arithmetic on channel pairs), written to TMEM as bf16
      {
        uint4 zr[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) zr[c] = *reinterpret_cast<const uint4*>(zchunk(c));
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
          const float2 d0 = __fadd2_rn(chan2(zr[c].x), nmu), d1 = __fadd2_rn(chan2(zr[c].y), nmu);
          const float2 d2 = __fadd2_rn(chan2(zr[c].z), nmu), d3 = __fadd2_rn(chan2(zr[c].w), nmu);
          acc[0] = __ffma2_rn(d0, d0, acc[0]);
          acc[1] = __ffma2_rn(d1, d1, acc[1]);
          acc[0] = __ffma2_rn(d2, d2, acc[0]);
          acc[1] = __ffma2_rn(d3, d3, acc[1]);
        }
        const float var = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
        const float rstd = rsqrtf(var * (1.0f / kCz) + a.eps);
        const float2 rstd2 = make_float2(rstd, rstd);
        auto xpair = [&](uint32_t w, float gx, float gy, float bx, float by) {
          const float2 x = __ffma2_rn(__fmul2_rn(__fadd2_rn(chan2(w), nmu), rstd2),
                                      make_float2(gx, gy), make_float2(bx, by));
          return pack_bf16x2(x.x, x.y);
        };
#pragma unroll
        for (int hq = 0; hq < 4; ++hq) {  // 32 channels = 16 TMEM columns at a time
          uint32_t xs[16];
#pragma unroll
          for (int cq = 0; cq < 4; ++cq) {
            const int c = 4 * hq + cq;
            const float4 g0 = ldpar(2, 8 * c), g1 = ldpar(2, 8 * c + 4);
            const float4 b0 = ldpar(3, 8 * c), b1 = ldpar(3, 8 * c + 4);
            xs[4 * cq + 0] = xpair(zr[c].x, g0.x, g0.y, b0.x, b0.y);
            xs[4 * cq + 1] = xpair(zr[c].y, g0.z, g0.w, b0.z, b0.w);
            xs[4 * cq + 2] = xpair(zr[c].z, g1.x, g1.y, b1.x, b1.y);
            xs[4 * cq + 3] = xpair(zr[c].w, g1.z, g1.w, b1.z, b1.w);
          }
          tmem_st16(t_o + lane_base + 16 * hq, xs);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      named_barrier_sync(bar_id, kComputeThreads);
      tc_fence_after();
      // ---- D_g = X Wg^T
      if (gt == 0) issue(t_g, t_o, sWg, &mma_g[s]);
      if (!named_barrier_and(bar_id, kComputeThreads, mbar_wait(&mma_g[s], ph, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // ---- a = bf16(sigmoid(D_g + bg) * o) over D_g: head h (channels 32h ..
      // 32h+31) is read from columns 32h.. and written to 16h.., which this
      // thread has read already
#pragma unroll 1
      for (int h = 0; h < kHeads; ++h) {
        uint32_t v[32];
        tmem_ld32(t_g + lane_base + h * 32, v);
        uint4 ov[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          ov[q] = *reinterpret_cast<const uint4*>(st + kStO + h * kOHeadBytes + gt * 64 +
                                                  ((q ^ ((gt >> 1) & 3)) << 4));
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t ow[4] = {ov[q].x, ov[q].y, ov[q].z, ov[q].w};
          const float4 b0 = ldpar(1, h * kD + 8 * q), b1 = ldpar(1, h * kD + 8 * q + 4);
          const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // sigmoid(t) = 1/2 + tanh(t/2)/2: one special-function op per value
            const float t0 = __uint_as_float(v[8 * q + 2 * e]) + bb[2 * e];
            const float t1 = __uint_as_float(v[8 * q + 2 * e + 1]) + bb[2 * e + 1];
            const float g0 = fmaf(0.5f, tanh_approx(0.5f * t0), 0.5f);
            const float g1 = fmaf(0.5f, tanh_approx(0.5f * t1), 0.5f);
            pk[4 * q + e] = pack_bf16x2(g0 * bf16lo_to_f32(ow[e]), g1 * bf16hi_to_f32(ow[e]));
          }
        }
        tmem_st16(t_g + lane_base + h * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      named_barrier_sync(bar_id, kComputeThreads);
      tc_fence_after();
      // ---- D_out = A Wo^T (over X, which the gate MMA has read)
      if (gt == 0) issue(t_o, t_g, sWo, &mma_o[s]);
      if (!named_barrier_and(bar_id, kComputeThreads, mbar_wait(&mma_o[s], ph, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // ---- out = D_out + bo + z, in place over z
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(t_o + lane_base + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = cc * 4 + q;
          uint8_t* zp = zchunk(c);
          const uint4 zv = *reinterpret_cast<const uint4*>(zp);
          const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
          const float4 o0 = ldpar(0, 8 * c), o1 = ldpar(0, 8 * c + 4);
          const float bo[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float y0 = __uint_as_float(v[q * 8 + 2 * e]) + bo[2 * e] + bf16lo_to_f32(zw[e]);
            const float y1 =
                __uint_as_float(v[q * 8 + 2 * e + 1]) + bo[2 * e + 1] + bf16hi_to_f32(zw[e]);
            pk[e] = pack_bf16x2(y0, y1);
          }
          *reinterpret_cast<uint4*>(zp) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_barrier_sync(bar_id, kComputeThreads);
      if (gt == 0) {
        int c1, c2;
        zcoords(tile, c1, c2);
        for (int slab = 0; slab < 2; ++slab)
          tma_store_3d(&map_out, st + kStZ + slab * kSlabBytes, 64 * slab, c1, c2);
        bulk_commit();
        stored = true;
        bulk_wait_read_all();  // the stage's shared memory may be refilled after this
        mbar_arrive(&empty[s]);
      }
    }
    if (!ok && gt == 0) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
    }
    // the stores must be complete (not only read out of shared memory) at exit
    if (gt == 0 && stored) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace gout
}  // namespace tri
