// pair_ln_proj.cuh — LayerNorm + fused Q/K/V projection (tcgen05) + logit
// bias, bf16 pair representation.
//
// Persistent CTAs of two independent groups of 8 warps.  Each group walks its
// own tiles of 128 pairs of one problem row (pairs (i, j0..j0+127)).  The tile of
// Z arrives by TMA straight into the group's MMA A buffer (K-major, 128-byte
// swizzle: two boxes of 64 channels; the ending-node block reads the swapped
// view, pair (i, j) = Z[j][i], as a box one pair wide and 128 pairs deep).
// Two threads share a pair: warp w of the group (w = 0..7) owns the pairs
// 32 (w % 4) .. +31 (its TMEM lane quadrant) and the channel half w / 4, which
// is exactly one 64-channel box of the A buffer.  Per tile each thread
//   1. reads its 64 channels (128 B) from the buffer,
//   2. sums, in one pass, z - K and (z - K)^2 (K = channel 0 of the pair, a
//      shift that keeps the variance free of cancellation) and the four logit-
//      bias dot products Wb gamma (z - K) (Wb pre-scaled by log2 e),
//   3. exchanges these six partial sums with the other thread of its pair
//      through shared memory (both add them in the same order, so the two
//      agree bit for bit), which gives the mean, the biased variance, rsqrt,
//      and the bias  rstd (S_h - (mean - K) sum_c Wb gamma) + Wb beta,
//      kMaskedLogit at masked keys and at the padding columns j >= N,
//   4. writes its normalised channels as bf16 back in place, which makes the
//      buffer the A operand.
// One thread of the group then issues the projection D = X W^T in two halves,
// N = 256 (q|k) and then N = 128 (v), W = [Wq; Wk; Wv] resident in shared
// memory for the whole kernel, each half accumulating in fp32 in the group's
// 256 TMEM columns; the next tile's TMA is issued as soon as the second half
// has consumed the buffer.  In the epilogue of the q|k half the two threads of
// a pair take q (scaled by log2(e)/sqrt(d)) and k, in that of the v half two
// heads of v each: the thread reads its TMEM lane and writes the pair's 64-byte
// row of each head of the head-major output ([rows][H][N][d], bf16) with two
// 32-byte stores straight from registers (a warp's 32 pairs fill a contiguous
// 2 KB block).  The gate is not produced here: gate_out recomputes it from
// LayerNorm(z), which it reads anyway, so it never goes through memory.  While
// one group runs its MMAs the other normalises or stores, so the tensor core,
// the ALUs and HBM overlap.
//
// This is the HBM-bound step: per pair it reads 256 B and writes 768 B + 8 B.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace tri {
namespace plp {

constexpr int kGroupThreads = 256;                   // two threads per pair
constexpr int kGroupsPerCta = 2;
constexpr int kThreads = kGroupThreads * kGroupsPerCta;
constexpr int kTileM = 128;
constexpr int kNOut = 3 * kHD;                       // q | k | v
constexpr uint32_t kWImgBytes = kNOut * kCz * 2;     // 98304
constexpr uint32_t kWAtomBytes = kNOut * 128;        // one 64-element K slab of W
constexpr uint32_t kATileBytes = kTileM * kCz * 2;   // 32768
constexpr uint32_t kAAtomBytes = kTileM * 128;       // 16384: one 64-channel box
constexpr uint32_t kSmemW = 0;
constexpr uint32_t kSmemA = kWImgBytes;                                  // + grp * kATileBytes
constexpr uint32_t kSmemPar = kSmemA + kGroupsPerCta * kATileBytes;     // fp32 params
// w_b * gamma [H][c_z], gamma, beta, then per head sum_c w_b gamma and w_b . beta
constexpr uint32_t kParFloats = kHeads * kCz + 2 * kCz + 2 * kHeads;
constexpr int kPartials = 2 + kHeads;                // sum, sum of squares, 4 bias dots
constexpr uint32_t kSmemXch = kSmemPar + ((kParFloats * 4 + 15) / 16) * 16;
// [group][channel half][partial][pair]
constexpr uint32_t kXchBytes = kGroupsPerCta * 2 * kPartials * kTileM * 4;
constexpr uint32_t kSmemBar = kSmemXch + kXchBytes;
constexpr uint32_t kSmemBytes = kSmemBar + 64 + 1024;                   // + alignment slack
static_assert(kGroupsPerCta * 2 * 8 + 8 + 8 <= 64, "barrier area");
constexpr uint32_t kTmemCols = 512;                                     // 256 per group

__global__ void __launch_bounds__(kThreads, 1)
    pair_ln_proj(const __grid_constant__ CUtensorMap map_z, const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_wbg = reinterpret_cast<float*>(smem + kSmemPar);  // w_b[h][c] * gamma[c]
  float* s_gamma = s_wbg + kHeads * kCz;
  float* s_beta = s_gamma + kCz;
  float* s_wsum = s_beta + kCz;      // [h]: sum_c w_b[h][c] gamma[c]
  float* s_wbeta = s_wsum + kHeads;  // [h]: sum_c w_b[h][c] beta[c]
  float* s_xch = reinterpret_cast<float*>(smem + kSmemXch);
  uint64_t* w_bar = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint64_t* mma_bar = w_bar + 1;                // one per group
  uint64_t* z_full = mma_bar + kGroupsPerCta;   // one per group
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(z_full + kGroupsPerCta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = tid / kGroupThreads;
  const int gt = tid % kGroupThreads;
  const int wq = (warp % 8) & 3;                // TMEM lane quadrant
  const int hc = (warp % 8) >> 2;               // channel half (LN) / output of a half (epilogue)
  const int p = wq * 32 + lane;                 // pair within the tile = TMEM lane
  const uint32_t bar_id = 1 + grp;
  const bool qkv = a.write_qkv != 0;
  uint8_t* sA = smem + kSmemA + grp * kATileBytes;

  for (int idx = tid; idx < kHeads * kCz; idx += kThreads)
    s_wbg[idx] = a.w_b[idx] * a.gamma[idx % kCz];
  for (int idx = tid; idx < kCz; idx += kThreads) {
    s_gamma[idx] = a.gamma[idx];
    s_beta[idx] = a.beta[idx];
  }
  if (warp < kHeads) {  // per-head constants of the bias: one warp per head
    float sw = 0.f, sb = 0.f;
    for (int c = lane; c < kCz; c += 32) {
      const float w = a.w_b[warp * kCz + c];
      sw = fmaf(w, a.gamma[c], sw);
      sb = fmaf(w, a.beta[c], sb);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sw += __shfl_xor_sync(0xffffffffu, sw, o);
      sb += __shfl_xor_sync(0xffffffffu, sb, o);
    }
    if (lane == 0) {
      s_wsum[warp] = sw;
      s_wbeta[warp] = sb;
    }
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
  if (warp == 0 && qkv) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot + static_cast<uint32_t>(grp * 256);
  if (tid == 0 && qkv) {
    mbar_arrive_expect_tx(w_bar, kWImgBytes);
    for (uint32_t off = 0; off < kWImgBytes; off += 32768)
      bulk_load(smem + kSmemW + off, a.w_img + off, 32768, w_bar);
  }

  const int jtiles = (a.N + kTileM - 1) / kTileM;
  const long long ntiles = static_cast<long long>(a.rows) * jtiles;
  const long long stride = static_cast<long long>(gridDim.x) * kGroupsPerCta;
  const uint32_t sA_u32 = smem_u32(sA), sW_u32 = smem_u32(smem + kSmemW);
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, false);   // q | k
  constexpr uint32_t kIdescV = idesc_bf16_f32(128, 128, false);  // v
  uint32_t mma_phase = 0;
  bool w_ready = false;
  const bool mma_thread = gt == 0;
  // the group's exchange area: [channel half][partial][pair]
  float* xch = s_xch + grp * (2 * kPartials * kTileM);
  uint8_t* row = sA + hc * kAAtomBytes + p * 128;  // this thread's 64 channels

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
    const int j = static_cast<int>(tile % jtiles) * kTileM + p;
    const bool jv = j < a.N;

    if (!named_barrier_and(bar_id, kGroupThreads, mbar_wait(&z_full[grp], z_phase, abort_flag))) {
      if (gt == 0) report_status(a.status, kStatusTimeout);
      break;
    }
    z_phase ^= 1;
    z_pending = false;
    // this thread's 64 channels: 16-byte chunk c of the row sits at c ^ (p % 8)
    uint4 zr[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      zr[c] = *reinterpret_cast<const uint4*>(row + ((c ^ (p & 7)) << 4));
    // the shift K: channel 0 of the pair (first bf16 of chunk 0 of the first box)
    const float K =
        bf16lo_to_f32(*reinterpret_cast<const uint32_t*>(sA + p * 128 + ((p & 7) << 4)));

    // ---- one pass: sum of (z - K), of (z - K)^2 and the four bias dot products
    auto chan2 = [](uint32_t w) { return make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w)); };
    const float2 nK = make_float2(-K, -K);
    float2 s1[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 sb[kHeads] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
    const float4* w4 = reinterpret_cast<const float4*>(s_wbg);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t w[4] = {zr[c].x, zr[c].y, zr[c].z, zr[c].w};
      float2 d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        d[e] = __fadd2_rn(chan2(w[e]), nK);
        s1[e & 1] = __fadd2_rn(s1[e & 1], d[e]);
        s2[e & 1] = __ffma2_rn(d[e], d[e], s2[e & 1]);
      }
      const int cb = hc * 64 + c * 8;  // first channel of this chunk
#pragma unroll
      for (int h = 0; h < kHeads; ++h) {
        const float4 wa = w4[(h * kCz + cb) / 4], wb = w4[(h * kCz + cb) / 4 + 1];
        float2 acc2 = sb[h];
        acc2 = __ffma2_rn(make_float2(wa.x, wa.y), d[0], acc2);
        acc2 = __ffma2_rn(make_float2(wa.z, wa.w), d[1], acc2);
        acc2 = __ffma2_rn(make_float2(wb.x, wb.y), d[2], acc2);
        acc2 = __ffma2_rn(make_float2(wb.z, wb.w), d[3], acc2);
        sb[h] = acc2;
      }
    }
    float part[kPartials];
    part[0] = (s1[0].x + s1[0].y) + (s1[1].x + s1[1].y);
    part[1] = (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y);
#pragma unroll
    for (int h = 0; h < kHeads; ++h) part[2 + h] = sb[h].x + sb[h].y;
    // ---- exchange with the other thread of the pair; both sum half 0 + half 1
#pragma unroll
    for (int k = 0; k < kPartials; ++k) xch[(hc * kPartials + k) * kTileM + p] = part[k];
    named_barrier_sync(bar_id, kGroupThreads);
    float tot[kPartials];
#pragma unroll
    for (int k = 0; k < kPartials; ++k) {
      const float other = xch[((hc ^ 1) * kPartials + k) * kTileM + p];
      tot[k] = hc == 0 ? part[k] + other : other + part[k];
    }
    const float md = tot[0] * (1.0f / kCz);            // mean - K
    const float var = fmaxf(tot[1] * (1.0f / kCz) - md * md, 0.f);
    const float rstd = rsqrtf(var + a.eps);
    if (a.write_bias && j < a.ld_bias) {
      // heads 2 hc and 2 hc + 1: rstd (S_h - (mean - K) sum_c Wb gamma) + Wb . beta
      const bool key_valid = jv && (a.mask == nullptr || a.mask[j] != 0);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * hc + hh;
        const float b = fmaf(fmaf(-md, s_wsum[h], tot[2 + h]), rstd, s_wbeta[h]);
        a.bias[(static_cast<long long>(h) * a.bias_rows + (i - a.bias_row0)) * a.ld_bias + j] =
            __float2bfloat16_rn(key_valid ? b : kMaskedLogit);
      }
    }
    if (!qkv) {
      // bias only: the buffer (and the exchange area) is free once every
      // thread of the group has read them
      named_barrier_sync(bar_id, kGroupThreads);
      if (mma_thread && tile + stride < ntiles) {
        issue_z(tile + stride);
        z_pending = true;
      }
      continue;
    }

    // ---- normalise this thread's 64 channels into the A operand, in place
    {
      const float mu = K + md;
      const float2 nmu = make_float2(-mu, -mu), rstd2 = make_float2(rstd, rstd);
      const float4* g4 = reinterpret_cast<const float4*>(s_gamma + hc * 64);
      const float4* b4 = reinterpret_cast<const float4*>(s_beta + hc * 64);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        // read again rather than held across the exchange (register pressure)
        const uint4 zc = *reinterpret_cast<const uint4*>(row + ((c ^ (p & 7)) << 4));
        const uint32_t w[4] = {zc.x, zc.y, zc.z, zc.w};
        uint32_t o[4];
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const float4 gm = g4[2 * c + hq], bt = b4[2 * c + hq];
          const float2 d0 = __fadd2_rn(chan2(w[2 * hq]), nmu);
          const float2 d1 = __fadd2_rn(chan2(w[2 * hq + 1]), nmu);
          const float2 x0 = __ffma2_rn(__fmul2_rn(d0, rstd2), make_float2(gm.x, gm.y),
                                       make_float2(bt.x, bt.y));
          const float2 x1 = __ffma2_rn(__fmul2_rn(d1, rstd2), make_float2(gm.z, gm.w),
                                       make_float2(bt.z, bt.w));
          o[2 * hq] = pack_bf16x2(x0.x, x0.y);
          o[2 * hq + 1] = pack_bf16x2(x1.x, x1.y);
        }
        *reinterpret_cast<uint4*>(row + ((c ^ (p & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }

    fence_proxy_async_smem();
    tc_fence_before();
    named_barrier_sync(bar_id, kGroupThreads);
    tc_fence_after();

    bool ok = true;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      // ---- MMA: D = X W_half^T, W_half = rows 0..255 of W (q|k) or 256..383 (v)
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
            mma_ss(tmem, ad, bd, half == 0 ? kIdesc : kIdescV, kk > 0 ? 1u : 0u);
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

      // ---- epilogue, one 32-column chunk (one head) at a time: after the q|k
      // half the two threads of a pair take q and k (4 heads each), after the v
      // half two heads of v each; a chunk is the pair's 64-byte row of that head,
      // written with two 32-byte stores
      const uint32_t col0 = tmem + lane_base + (half == 0 ? hc * 128 : hc * 64);
      __nv_bfloat16* out = half == 0 ? (hc == 0 ? a.Q : a.K) : a.V;
      const float sc = half == 0 && hc == 0 ? a.q_scale : 1.0f;
      // every chunk packs into registers of its own, all kept live until the
      // last store has been issued, so no store waits for the previous one to
      // release its registers
      auto chunks = [&](auto nch) {
        constexpr int kN = decltype(nch)::value;
        uint32_t pk[kN][16];
#pragma unroll
        for (int cc = 0; cc < kN; ++cc) {
          uint32_t v[32];
          tmem_ld32(col0 + cc * 32, v);
          tmem_ld_wait();
          tmem_regs_ready(v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[cc][e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
          const int h = half == 0 ? cc : 2 * hc + cc;
          if (jv) {
            uint32_t* dst = reinterpret_cast<uint32_t*>(
                out + ((static_cast<long long>(r) * kHeads + h) * a.N + j) * kD);
            st_global_v8(dst, pk[cc][0], pk[cc][1], pk[cc][2], pk[cc][3], pk[cc][4], pk[cc][5],
                         pk[cc][6], pk[cc][7]);
            st_global_v8(dst + 8, pk[cc][8], pk[cc][9], pk[cc][10], pk[cc][11], pk[cc][12],
                         pk[cc][13], pk[cc][14], pk[cc][15]);
          }
        }
#pragma unroll
        for (int cc = 0; cc < kN; ++cc)
#pragma unroll
          for (int e = 0; e < 16; ++e) asm volatile("" ::"r"(pk[cc][e]));
      };
      if (half == 0)
        chunks(std::integral_constant<int, kHeads>{});
      else
        chunks(std::integral_constant<int, 2>{});
      tc_fence_before();
      named_barrier_sync(bar_id, kGroupThreads);  // TMEM (and, after the second half, A) reused
      tc_fence_after();
    }
    if (!ok) {
      if (gt == 0) report_status(a.status, kStatusTimeout);
      break;
    }
  }

  // ---- teardown: no copy may still be writing this CTA's smem
  if (tid == 0 && qkv && !w_ready) {
    if (!mbar_wait(w_bar, 0, nullptr)) report_status(a.status, kStatusTimeout);
  }
  if (mma_thread && z_pending) {
    if (!mbar_wait(&z_full[grp], z_phase, nullptr)) report_status(a.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && qkv) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, kTmemCols);
  }
}

}  // namespace plp
}  // namespace tri
