// gate_out.cuh — sigmoid gate, output projection (tcgen05) and residual add,
// bf16 pair representation.
//
// Persistent CTAs walk tiles of 128 pairs (i, j0..j0+127) of one problem row.
// Two groups of eight warps take the tiles in turn.  Each group owns two tile
// buffers in shared memory and 256 TMEM columns:
//   Z buffer: the residual z ([128][128], 128-byte swizzle, two 64-channel
//     slabs; the ending-node block reads the swapped view, pair (i, j) =
//     Z[j][i], as a box that is one pair wide and 128 pairs deep);
//   O buffer: o (4 head boxes of [128 pairs][32], 64-byte swizzle), and later
//     the out tile on its way to the TMA store;
//   TMEM: X, then A (bf16 pairs) in columns 0..63; z (bf16 pairs) in 64..127;
//     D_g, then D_out in 128..255 (lane = pair).
// The gate is recomputed here rather than read: g = sigmoid(Wg LayerNorm(z) +
// bg) needs only z, which this kernel reads anyway for the residual, so the
// projection kernel never writes a gate tensor and this kernel never reads one.
// Two threads share a pair: warp w of a group owns the pairs 32 (w % 4) ..
// +31 (its TMEM lane quadrant) and the channel half w / 4.  One thread of the
// group (the leader) issues its TMA loads, copies and MMAs; it refills a
// buffer as soon as the group is done with it, so no producer warp is needed.
// Per tile:
//   1. the leader copies z from the Z buffer into TMEM (tcgen05.cp) while each
//      thread sums its 64 channels of z - K and (z - K)^2 (K = channel 0 of the
//      pair, a shift that keeps the one-pass variance free of cancellation);
//      the two threads of a pair exchange these partial sums through shared
//      memory and both form the mean, the biased variance and rsqrt, then store
//      their 64 channels of x = LayerNorm(z) to TMEM as bf16;
//   2. D_g = X (Wg/2)^T (8 tcgen05 MMAs, N = 128), so t = D_g + bg/2 is half
//      the gate's logit and sigmoid(2t) = (1 + tanh t) / 2; the Z buffer is
//      refilled with the group's next tile once this MMA (and the copy) is done;
//   3. a' = bf16((1 + tanh t) o), one special-function op and one fma per
//      value, over X: twice the gated output, which Wo/2 undoes;
//   4. D_out = A' (Wo/2)^T (8 MMAs) over D_g;
//   5. out = D_out + bo + z, written over o in the O buffer (128-byte swizzle)
//      and stored with TMA (through the swapped view again for the ending
//      node); the leader refills the O buffer with the group's next tile once
//      that tile's z has arrived and its copies are issued (by then the store
//      has read the buffer), which keeps the read-out of the store off the
//      group's path.
// Wg/2 and Wo/2 stay resident in shared memory (halving a bf16 weight is
// exact).  Every element of out is read (as z) and written by the same CTA,
// tile by tile, so out may alias Z.
//
// HBM-bound: per pair it reads 512 B (o, z) and writes 256 B.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace gout {

constexpr int kGroupThreads = 256;               // one group: two threads per pair of a tile
constexpr int kGroups = 2;
constexpr int kThreads = kGroups * kGroupThreads;
constexpr int kTileM = 128;
constexpr uint32_t kWBytes = kCz * kHD * 2;          // 32768: one 128 x 128 weight image
constexpr uint32_t kWAtomBytes = kCz * 128;          // 16384: one 64-element K slab of it
constexpr uint32_t kOHeadBytes = kTileM * kD * 2;    // 8192: [128 pairs][32] bf16
constexpr uint32_t kSlabBytes = kTileM * 128;        // 16384: [128 pairs][64] bf16
constexpr uint32_t kBufBytes = 2 * kSlabBytes;       // 32768: one Z or O buffer
constexpr uint32_t kSmemWo = 0;
constexpr uint32_t kSmemWg = kWBytes;
constexpr uint32_t kSmemBufs = 2 * kWBytes;          // group g: Z at 2g, O at 2g + 1
constexpr uint32_t kSmemPar = kSmemBufs + 2 * kGroups * kBufBytes;  // bo, bg / 2, gamma, beta
constexpr uint32_t kSmemXch = kSmemPar + 4 * kCz * 4;  // [group][half][pair] float2
constexpr uint32_t kSmemBar = kSmemXch + kGroups * 2 * kTileM * 8;
constexpr int kBarsPerGroup = 4;  // z_full, o_full, mma_g, mma_o
constexpr uint32_t kNumBars = 1 + kBarsPerGroup * kGroups;
constexpr uint32_t kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;  // per group: X / A (64 columns), z (64), D_g / D_out (128)

// 16 warps: four share a sub-partition's 16K registers, so at most 128 each.
__global__ void __launch_bounds__(kThreads, 1)
    gate_out(const __grid_constant__ CUtensorMap map_o, const __grid_constant__ CUtensorMap map_z,
             const __grid_constant__ CUtensorMap map_out, const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_par = reinterpret_cast<float*>(smem + kSmemPar);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* w_bar = bars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int idx = tid; idx < kCz; idx += kThreads) {
    s_par[idx] = a.b_o[idx];
    s_par[kCz + idx] = 0.5f * a.b_g[idx];  // t = (Wg x + bg) / 2
    s_par[2 * kCz + idx] = a.gamma[idx];
    s_par[3 * kCz + idx] = a.beta[idx];
  }
  if (tid == 0) {
    for (uint32_t b = 0; b < kNumBars; ++b) mbar_init(&bars[b], 1);
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

  const int grp = warp >> 3;               // group
  const int gw = warp & 7;                 // warp within the group
  const int hc = gw >> 2;                  // channel half: 64 hc .. 64 hc + 63
  const int p = (gw & 3) * 32 + lane;      // pair within the tile = TMEM lane
  const bool leader = gw == 0 && lane == 0;
  const uint32_t bar_id = 1 + grp;
  uint64_t* gbar = bars + 1 + kBarsPerGroup * grp;
  uint64_t *z_full = gbar, *o_full = gbar + 1, *mma_g = gbar + 2, *mma_o = gbar + 3;
  uint8_t* zbuf = smem + kSmemBufs + (2 * grp) * kBufBytes;
  uint8_t* obuf = zbuf + kBufBytes;
  float2* xch = reinterpret_cast<float2*>(smem + kSmemXch) + grp * 2 * kTileM;
  const uint32_t lane_base = static_cast<uint32_t>((gw & 3) * 32) << 16;
  const uint32_t t_xa = tmem + grp * 256, t_z = t_xa + 64, t_d = t_xa + 128;
  const uint32_t sWo = smem_u32(smem + kSmemWo), sWg = smem_u32(smem + kSmemWg);
  const uint32_t zbuf_u32 = smem_u32(zbuf);
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);

  const int jtiles = (a.N + kTileM - 1) / kTileM;
  const long long ntiles = static_cast<long long>(a.rows) * jtiles;
  const long long tile0 = blockIdx.x + grp * static_cast<long long>(gridDim.x);
  const long long tstep = kGroups * static_cast<long long>(gridDim.x);
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
  // the leader's loads; z_loaded / o_loaded count those issued, z_done / o_done
  // those the group has waited for, so that none is left in flight at exit
  long long z_loaded = 0, o_loaded = 0, z_done = 0, o_done = 0;
  auto load_z = [&](long long tile) {
    int c1, c2;
    zcoords(tile, c1, c2);
    mbar_arrive_expect_tx(z_full, kBufBytes);
    for (int slab = 0; slab < 2; ++slab)
      tma_load_3d(zbuf + slab * kSlabBytes, &map_z, z_full, 64 * slab, c1, c2);
    ++z_loaded;
  };
  auto load_o = [&](long long tile) {
    const int r = static_cast<int>(tile / jtiles);
    const int j0 = static_cast<int>(tile % jtiles) * kTileM;
    mbar_arrive_expect_tx(o_full, kBufBytes);
    for (int h = 0; h < kHeads; ++h)
      tma_load_3d(obuf + h * kOHeadBytes, &map_o, o_full, 0, j0, r * kHeads + h);
    ++o_loaded;
  };
  bool w_ready = false;
  // D[128 x 128] = A (TMEM, bf16 pairs) W^T (W resident, K-major 128-byte
  // swizzle), issued by the leader
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
  // fault injection: the leader of group 0 of CTA 0 never loads its first z
  // tile, so the group's bounded wait expires and the launch reports
  // TRI_ATTN_ERR_TIMEOUT
  const bool stall = a.debug_stall && blockIdx.x == 0 && grp == 0;
  if (leader) {
    if (grp == 0) {
      tma_prefetch_desc(&map_o);
      tma_prefetch_desc(&map_z);
      mbar_arrive_expect_tx(w_bar, 2 * kWBytes);
      bulk_load(smem + kSmemWo, a.wo_img, kWBytes, w_bar);
      bulk_load(smem + kSmemWg, a.wg_img, kWBytes, w_bar);
    }
    if (tile0 < ntiles) {
      if (!stall) load_z(tile0);
      load_o(tile0);
    }
  }

  bool ok = true, stored = false;
  long long k = 0;
  for (long long tile = tile0; tile < ntiles; tile += tstep, ++k) {
    const uint32_t ph = static_cast<uint32_t>(k) & 1;
    const bool more = tile + tstep < ntiles;
    // bo, bg / 2, gamma, beta and the swizzle phases, re-derived per tile so
    // that they are read where used instead of held in registers across the loop
    const uint32_t par = opaque_u32(smem_u32(s_par));
    auto ldpar = [&](int which, int ch) { return lds_f4(par + (which * kCz + ch) * 4); };
    const uint32_t sw = opaque_u32(p & 7), sw64 = opaque_u32((p >> 1) & 3);
    // 16-byte chunk c (channels 64 hc + 8c ..) of this thread's row of a
    // 128-byte swizzled [128][128] tile
    auto chunk = [&](uint8_t* buf, int c) {
      return buf + hc * kSlabBytes + p * 128 + ((c ^ sw) << 4);
    };
    if (!named_barrier_and(bar_id, kGroupThreads, mbar_wait(z_full, ph, abort_flag))) {
      ok = false;
      break;
    }
    z_done = k + 1;
    tc_fence_after();
    if (leader) {
      // z to TMEM columns 64..127 by the tensor core's copy (32 bytes, 16
      // channels, of every row per copy), while the threads normalise
#pragma unroll
      for (int c = 0; c < 8; ++c)
        tmem_cp_128x256b(t_z + 8 * c, smem_desc(zbuf_u32 + (c >> 2) * kSlabBytes + (c & 3) * 32,
                                                1024, kSwizzle128B));
      if (k > 0) {
        bulk_wait_read_all();  // the previous tile's store has read the O buffer
        load_o(tile);
      }
    }
    // ---- x = LayerNorm(z): one pass over this thread's 64 channels (mixed-
    // precision adds widen z exactly), partial sums exchanged with the other
    // thread of the pair, which adds them in the same order
    {
      uint4 zr[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) zr[c] = *reinterpret_cast<const uint4*>(chunk(zbuf, c));
      const float K = bf16lo_to_f32(*reinterpret_cast<const uint32_t*>(zbuf + p * 128 + (sw << 4)));
      const float2 nK = make_float2(-K, -K);
      float2 s1[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t w[4] = {zr[c].x, zr[c].y, zr[c].z, zr[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 d = add_bf16x2_f32x2(w[e], nK);
          s1[e & 1] = __fadd2_rn(s1[e & 1], d);
          s2[e & 1] = __ffma2_rn(d, d, s2[e & 1]);
        }
      }
      const float2 part = make_float2((s1[0].x + s1[0].y) + (s1[1].x + s1[1].y),
                                      (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y));
      xch[hc * kTileM + p] = part;
      named_barrier_sync(bar_id, kGroupThreads);
      const float2 other = xch[(hc ^ 1) * kTileM + p];
      const float t1 = hc == 0 ? part.x + other.x : other.x + part.x;
      const float t2 = hc == 0 ? part.y + other.y : other.y + part.y;
      const float md = t1 * (1.0f / kCz);  // mean - K
      const float rstd = rsqrtf(fmaxf(t2 * (1.0f / kCz) - md * md, 0.f) + a.eps);
      const float2 nmu = make_float2(-(K + md), -(K + md)), rstd2 = make_float2(rstd, rstd);
      auto xpair = [&](uint32_t w, float gx, float gy, float bx, float by) {
        const float2 x = __ffma2_rn(__fmul2_rn(add_bf16x2_f32x2(w, nmu), rstd2),
                                    make_float2(gx, gy), make_float2(bx, by));
        return pack_bf16x2(x.x, x.y);
      };
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {  // 32 channels = 16 TMEM columns at a time
        uint32_t xs[16];
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {
          const int c = 4 * hq + cq, ch = 64 * hc + 8 * c;
          const float4 g0 = ldpar(2, ch), g1 = ldpar(2, ch + 4);
          const float4 b0 = ldpar(3, ch), b1 = ldpar(3, ch + 4);
          xs[4 * cq + 0] = xpair(zr[c].x, g0.x, g0.y, b0.x, b0.y);
          xs[4 * cq + 1] = xpair(zr[c].y, g0.z, g0.w, b0.z, b0.w);
          xs[4 * cq + 2] = xpair(zr[c].z, g1.x, g1.y, b1.x, b1.y);
          xs[4 * cq + 3] = xpair(zr[c].w, g1.z, g1.w, b1.z, b1.w);
        }
        tmem_st16(t_xa + lane_base + 32 * hc + 16 * hq, xs);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    named_barrier_sync(bar_id, kGroupThreads);  // every z read, every X stored
    tc_fence_after();
    // ---- D_g = X (Wg/2)^T; its commit also covers the copies of z
    if (leader) issue(t_d, t_xa, sWg, mma_g);
    {
      const bool got = mbar_wait(mma_g, ph, abort_flag) && mbar_wait(o_full, ph, abort_flag);
      if (!named_barrier_and(bar_id, kGroupThreads, got)) {
        ok = false;
        break;
      }
    }
    o_done = k + 1;
    tc_fence_after();
    // the Z buffer is free: every thread has read it, the copies have completed
    if (leader && more) load_z(tile + tstep);
    // ---- a' = bf16((1 + tanh t) o) over X, t = D_g + bg/2, half a head (16
    // channels) at a time: this thread's heads are 2 hc and 2 hc + 1
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      const int hh = 4 * hc + q;  // half-head: channels 16 hh .. 16 hh + 15
      uint32_t v[16];
      tmem_ld16(t_d + lane_base + 16 * hh, v);
      const int h = hh >> 1;
      uint4 ov[2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int qc = 2 * (hh & 1) + q2;  // 16-byte chunk of the head's 64-byte row
        ov[q2] = *reinterpret_cast<const uint4*>(obuf + h * kOHeadBytes + p * 64 +
                                                 ((qc ^ sw64) << 4));
      }
      tmem_ld_wait();
      tmem_regs_ready(v);
      uint32_t pk[8];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const uint32_t ow[4] = {ov[q2].x, ov[q2].y, ov[q2].z, ov[q2].w};
        const float4 b0 = ldpar(1, 16 * hh + 8 * q2), b1 = ldpar(1, 16 * hh + 8 * q2 + 4);
        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float th0 = tanh_approx(__uint_as_float(v[8 * q2 + 2 * e]) + bb[2 * e]);
          const float th1 = tanh_approx(__uint_as_float(v[8 * q2 + 2 * e + 1]) + bb[2 * e + 1]);
          const float o0 = bf16lo_to_f32(ow[e]), o1 = bf16hi_to_f32(ow[e]);
          pk[4 * q2 + e] = pack_bf16x2(fmaf(th0, o0, o0), fmaf(th1, o1, o1));
        }
      }
      tmem_st8(t_xa + lane_base + 8 * hh, pk);
    }
    tmem_st_wait();
    tc_fence_before();
    named_barrier_sync(bar_id, kGroupThreads);  // every o and D_g read, every A' stored
    tc_fence_after();
    // ---- D_out = A' (Wo/2)^T over D_g
    if (leader) issue(t_d, t_xa, sWo, mma_o);
    if (!named_barrier_and(bar_id, kGroupThreads, mbar_wait(mma_o, ph, abort_flag))) {
      ok = false;
      break;
    }
    tc_fence_after();
    // ---- out = D_out + bo + z, this thread's 64 channels, written over o
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t v[32], zv[16];
      tmem_ld32(t_d + lane_base + 64 * hc + 32 * cc, v);
      tmem_ld16(t_z + lane_base + 32 * hc + 16 * cc, zv);
      tmem_ld_wait();
      tmem_regs_ready(v);
      tmem_regs_ready(zv);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const int c = 4 * cc + qq, ch = 64 * hc + 8 * c;
        const float4 o0 = ldpar(0, ch), o1 = ldpar(0, ch + 4);
        const float bo[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t zw = zv[4 * qq + e];
          pk[e] = pack_bf16x2(__uint_as_float(v[8 * qq + 2 * e]) + bo[2 * e] + bf16lo_to_f32(zw),
                              __uint_as_float(v[8 * qq + 2 * e + 1]) + bo[2 * e + 1] +
                                  bf16hi_to_f32(zw));
        }
        *reinterpret_cast<uint4*>(chunk(obuf, c)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_barrier_sync(bar_id, kGroupThreads);
    if (leader) {
      int c1, c2;
      zcoords(tile, c1, c2);
      for (int slab = 0; slab < 2; ++slab)
        tma_store_3d(&map_out, obuf + slab * kSlabBytes, 64 * slab, c1, c2);
      bulk_commit();
      stored = true;

    }
  }
  if (leader) {
    if (!ok) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
    }
    // never leave a copy in flight into this CTA's shared memory, nor a store
    // unfinished
    if (grp == 0 && !mbar_wait(w_bar, 0, nullptr)) report_status(a.status, kStatusTimeout);
    if (z_loaded > z_done &&
        !mbar_wait(z_full, static_cast<uint32_t>(z_loaded - 1) & 1, nullptr))
      report_status(a.status, kStatusTimeout);
    if (o_loaded > o_done &&
        !mbar_wait(o_full, static_cast<uint32_t>(o_loaded - 1) & 1, nullptr))
      report_status(a.status, kStatusTimeout);
    if (stored) bulk_wait_all();
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
