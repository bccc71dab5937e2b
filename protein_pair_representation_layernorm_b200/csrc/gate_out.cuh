// gate_out.cuh — sigmoid gate, output projection (tcgen05) and residual add,
// bf16 pair representation.
//
// Persistent CTAs walk tiles of 128 pairs (i, j0..j0+127) of one problem row
// through a two-stage pipeline.  A producer warp moves each tile in with TMA:
// o and g (4 head boxes each of [128 pairs][32], 64-byte swizzle) and the
// residual z ([128][128], 128-byte swizzle; the ending-node block reads the
// swapped view, pair (i, j) = Z[j][i], as a box that is one pair wide and 128
// pairs deep).  Thread t of the four compute warps owns pair j0+t: it forms
// bf16(g * o) and, once every thread has read its g, writes it over the g
// buffer in the layout of the MMA A operand (K-major, 128-byte swizzle); one
// thread issues 8 tcgen05
// MMAs, D[128 x 128] = (G*O) Wo^T with Wo resident in shared memory, into one of
// two 128-column TMEM accumulators; each thread then adds bo and z and writes
// out_ij in place over z, and one thread stores the tile with TMA (through the
// swapped view again for the ending node).  Every element of out is read (as z)
// and written by the same CTA, tile by tile, so out may alias Z.
//
// HBM-bound: per pair it reads 768 B (o, g, z) and writes 256 B.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace gout {

constexpr int kComputeThreads = 128;
constexpr int kThreads = kComputeThreads + 32;   // + producer warp
constexpr int kProducerWarp = 4;
constexpr int kTileM = 128;
constexpr int kStages = 2;
constexpr uint32_t kWoBytes = kCz * kHD * 2;     // 32768
constexpr uint32_t kWoAtomBytes = kCz * 128;     // 16384
constexpr uint32_t kOHeadBytes = kTileM * kD * 2;    // 8192: [128 pairs][32] bf16
constexpr uint32_t kSlabBytes = kTileM * 128;        // 16384: [128 pairs][64] bf16
constexpr uint32_t kStO = 0;
constexpr uint32_t kStG = kHeads * kOHeadBytes;      // 32768
constexpr uint32_t kStZ = kStG + 2 * kSlabBytes;     // 65536
constexpr uint32_t kStageBytes = kStZ + 2 * kSlabBytes;  // 98304
constexpr uint32_t kSmemW = 0;
constexpr uint32_t kSmemStages = kWoBytes;
constexpr uint32_t kSmemBo = kSmemStages + kStages * kStageBytes;
constexpr uint32_t kSmemBar = kSmemBo + kCz * 4;
constexpr uint32_t kNumBars = 1 + 3 * kStages;
constexpr uint32_t kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;
constexpr uint32_t kTmemCols = 256;  // two 128-column accumulators

__global__ void __launch_bounds__(kThreads, 1)
    gate_out(const __grid_constant__ CUtensorMap map_o, const __grid_constant__ CUtensorMap map_g,
             const __grid_constant__ CUtensorMap map_z, const __grid_constant__ CUtensorMap map_out,
             const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_bo = reinterpret_cast<float*>(smem + kSmemBo);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* w_bar = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + kStages;
  uint64_t* mma_bar = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int idx = tid; idx < kCz; idx += kThreads) s_bo[idx] = a.b_o[idx];
  if (tid == 0) {
    mbar_init(w_bar, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&mma_bar[s], 1);
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
      tma_prefetch_desc(&map_g);
      tma_prefetch_desc(&map_z);
      mbar_arrive_expect_tx(w_bar, kWoBytes);
      bulk_load(smem + kSmemW, a.wo_img, kWoBytes, w_bar);
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
        for (int h = 0; h < kHeads; ++h)
          tma_load_3d(st + kStG + h * kOHeadBytes, &map_g, &full[s], 0, j0, r * kHeads + h);
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
    const int gt = tid;                     // pair within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t sW_u32 = smem_u32(smem + kSmemW);
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);
    bool w_ready = false, ok = true, stored = false;
    long long n = 0;
    for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++n) {
      const int s = static_cast<int>(n % kStages);
      const uint32_t ph = static_cast<uint32_t>(n / kStages) & 1;
      uint8_t* st = smem + kSmemStages + s * kStageBytes;
      if (!named_barrier_and(1, kComputeThreads, mbar_wait(&full[s], ph, abort_flag))) {
        ok = false;
        break;
      }
      // ---- A = bf16(g * o): 16-byte chunk c = channels 8c..8c+7 = head c/4, part c%4
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int h = c >> 2, q = c & 3;
        const uint32_t off = h * kOHeadBytes + gt * 64 + ((q ^ ((gt >> 1) & 3)) << 4);
        const uint4 gv = *reinterpret_cast<const uint4*>(st + kStG + off);
        const uint4 ov = *reinterpret_cast<const uint4*>(st + kStO + off);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pk[4 * c + e] = pack_bf16x2(bf16lo_to_f32(ow[e]) * bf16lo_to_f32(gw[e]),
                                      bf16hi_to_f32(ow[e]) * bf16hi_to_f32(gw[e]));
      }
      named_barrier_sync(1, kComputeThreads);  // every g has been read: reuse its buffer for A
      uint8_t* grow = st + kStG + gt * 128;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4*>(grow + (c >> 3) * kSlabBytes + (((c & 7) ^ (gt & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      named_barrier_sync(1, kComputeThreads);
      tc_fence_after();
      const uint32_t acc = tmem + s * 128;
      if (gt == 0) {
        bool ready = true;
        if (!w_ready) ready = w_ready = mbar_wait(w_bar, 0, abort_flag);
        if (ready) {
          const uint32_t sA = smem_u32(st + kStG);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = smem_desc(sA + (kk >> 2) * kSlabBytes + (kk & 3) * 32, 1024,
                                          kSwizzle128B);
            const uint64_t bd = smem_desc(sW_u32 + (kk >> 2) * kWoAtomBytes + (kk & 3) * 32,
                                          1024, kSwizzle128B);
            mma_ss(acc, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&mma_bar[s]);
        } else {
          *abort_flag = 1;
          report_status(a.status, kStatusTimeout);
        }
      }
      if (!named_barrier_and(1, kComputeThreads, mbar_wait(&mma_bar[s], ph, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // ---- out = acc + bo + z, in place over z
      uint8_t* zrow = st + kStZ + gt * 128;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(acc + lane_base + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = cc * 4 + q;  // 16-byte chunk of the 128 channels
          uint8_t* zp = zrow + (c >> 3) * kSlabBytes + (((c & 7) ^ (gt & 7)) << 4);
          const uint4 zv = *reinterpret_cast<const uint4*>(zp);
          const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int ch = c * 8 + 2 * e;
            const float y0 = __uint_as_float(v[q * 8 + 2 * e]) + s_bo[ch] + bf16lo_to_f32(zw[e]);
            const float y1 =
                __uint_as_float(v[q * 8 + 2 * e + 1]) + s_bo[ch + 1] + bf16hi_to_f32(zw[e]);
            pk[e] = pack_bf16x2(y0, y1);
          }
          *reinterpret_cast<uint4*>(zp) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_barrier_sync(1, kComputeThreads);
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
    if (gt == 0 && stored) {
      // the stores must be complete (not only read out of shared memory) at exit
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
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
