// gate_out.cuh — sigmoid gate, output projection (tcgen05) and residual add,
// bf16 pair representation.
//
// One CTA of 128 threads handles 128 pairs (i, j0..j0+127) of one problem row.
// Thread t owns pair j0+t: it forms  g * o  (g = sigmoid gate already applied
// by pair_ln_proj, o = attention output of the 4 heads), rounds it to bf16 and
// writes it into the MMA A tile (K-major, 128-byte swizzle).  Thread 0 issues 8
// tcgen05 MMAs, D[128 x 128] = (G*O) Wo^T, fp32 in 128 TMEM columns; each
// thread then adds bo and its own residual z_ij (loaded at the start, together
// with o and g, so that all of a thread's loads are in flight at once) and writes
// out_ij as bf16 with 16-byte vector stores.  The ending-node block reads the residual from and
// writes the result to the swapped view (pair (i, j) is Z[j][i]).  A thread
// reads z_ij before writing out_ij, so out may alias Z.
//
// HBM-bound: per pair it reads 768 B (o, g, z) and writes 256 B.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace gout {

constexpr int kThreads = 128;
constexpr int kTileM = 128;
constexpr uint32_t kWoBytes = kCz * kHD * 2;     // 32768
constexpr uint32_t kWoAtomBytes = kCz * 128;     // 16384
constexpr uint32_t kATileBytes = kTileM * kHD * 2;
constexpr uint32_t kAAtomBytes = kTileM * 128;
constexpr uint32_t kSmemW = 0;
constexpr uint32_t kSmemA = kWoBytes;
constexpr uint32_t kSmemBo = kSmemA + kATileBytes;
constexpr uint32_t kSmemBar = kSmemBo + kCz * 4;
constexpr uint32_t kSmemBytes = kSmemBar + 64 + 1024;
constexpr uint32_t kTmemCols = 128;

__global__ void __launch_bounds__(kThreads) gate_out(const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem + kSmemW;
  uint8_t* sA = smem + kSmemA;
  float* s_bo = reinterpret_cast<float*>(smem + kSmemBo);
  uint64_t* w_bar = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* mma_bar = w_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(w_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  for (int idx = tid; idx < kCz; idx += kThreads) s_bo[idx] = a.b_o[idx];
  if (tid == 0) {
    mbar_init(w_bar, 1);
    mbar_init(mma_bar, 1);
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
  if (tid == 0) {
    mbar_arrive_expect_tx(w_bar, kWoBytes);
    bulk_load(sW, a.wo_img, kWoBytes, w_bar);
  }

  const int r = blockIdx.y;
  const int i = a.row0 + r;
  const int j = blockIdx.x * kTileM + tid;
  const bool jv = j < a.N;

  // ---- the residual pair vector: loaded now so that it is in flight with o and g
  const long long zoff = jv ? pair_offset(a.orient, a.N, i, j) : 0;
  uint4 zv[16];
  if (jv) {
    const uint4* zp = reinterpret_cast<const uint4*>(a.Z + zoff);
#pragma unroll
    for (int q = 0; q < 16; ++q) zv[q] = zp[q];
  }

  // ---- A = bf16(g * o), K index = h*d + e
#pragma unroll
  for (int h = 0; h < kHeads; ++h) {
    uint4 ov[4], gv[4];
    if (jv) {
      const uint4* op = reinterpret_cast<const uint4*>(
          a.O + ((static_cast<long long>(r) * kHeads + h) * a.N + j) * kD);
      const uint4* gp = reinterpret_cast<const uint4*>(
          a.G + (static_cast<long long>(r) * a.N + j) * kHD + h * kD);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ov[q] = __ldg(op + q);
        gv[q] = __ldg(gp + q);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) ov[q] = gv[q] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t ow[4] = {ov[q].x, ov[q].y, ov[q].z, ov[q].w};
      const uint32_t gw[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        pk[e] = pack_bf16x2(bf16lo_to_f32(ow[e]) * bf16lo_to_f32(gw[e]),
                            bf16hi_to_f32(ow[e]) * bf16hi_to_f32(gw[e]));
      const int c = h * 4 + q;  // 16-byte chunk along K
      uint8_t* dst = sA + (c >> 3) * kAAtomBytes + tid * 128 + (((c & 7) ^ (tid & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0) {
    if (mbar_wait(w_bar, 0, abort_flag)) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);
      const uint32_t sA_u32 = smem_u32(sA), sW_u32 = smem_u32(sW);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad =
            smem_desc(sA_u32 + (kk >> 2) * kAAtomBytes + (kk & 3) * 32, 1024, kSwizzle128B);
        const uint64_t bd =
            smem_desc(sW_u32 + (kk >> 2) * kWoAtomBytes + (kk & 3) * 32, 1024, kSwizzle128B);
        mma_ss(tmem, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(mma_bar);
    } else {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
      mbar_wait(w_bar, 0, nullptr);  // do not exit with the copy in flight
    }
  }
  const bool done = mbar_wait(mma_bar, 0, abort_flag);
  if (__syncthreads_and(done ? 1 : 0)) {
    tc_fence_after();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + cc * 32, v);
      tmem_ld_wait();
      if (!jv) continue;
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 zq = zv[cc * 4 + q];
        const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = cc * 32 + q * 8 + 2 * e;
          const float y0 = __uint_as_float(v[q * 8 + 2 * e]) + s_bo[c0] + bf16lo_to_f32(zw[e]);
          const float y1 =
              __uint_as_float(v[q * 8 + 2 * e + 1]) + s_bo[c0 + 1] + bf16hi_to_f32(zw[e]);
          pk[q * 4 + e] = pack_bf16x2(y0, y1);
        }
      }
      uint4* op = reinterpret_cast<uint4*>(a.out + zoff + cc * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        op[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  } else if (tid == 0) {
    report_status(a.status, kStatusTimeout);
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
