// Split-KV attention pass on warp-level tensor-core tiles (m16n8k16).
//
// This is the decode / short-query path: the g*L query rows that share one KV
// head are packed into 16-row warp tiles, so one pass over that head's keys
// serves all of them, and the keys are split across CTAs so the work stays
// parallel over S even when B*Hkv is small (mlx issue #3826: the verify
// window lost its split over S and paid a padded 64-row tile per head; the
// fix there was a split over S with a log-sum-exp merge).  It is also a
// complete, general path: any L, causal and window masks, any head dims up
// to 256.
//
// CTA = (row tile, split, batch*KV head).  Warps: WR x WK consumer warps (WR
// row groups of 16 rows, WK slices of each key block) and one producer warp
// that streams Q once and K/V key blocks through an NST-stage ring with TMA
// (128-byte swizzled boxes of 64 columns, zero fill past S and past D).
// Each consumer keeps an fp32 online softmax (running max m, running sum l,
// rescaled O) in registers; P is rounded to the 16-bit input type for the
// P*V tile.  The WK slices are merged in shared memory at the end; the
// result goes to `out` (one split) or to fp32 partials + LSE (several).
#pragma once

#include "params.cuh"

namespace sdpa {

template <int DQK, int DV, int BN, int WR, int WK, int NST>
struct SplitKvCfg {
  static constexpr int kRT = 16 * WR;             // rows per CTA
  static constexpr int kKW = BN / WK;             // keys per warp per block
  static constexpr int kQBoxes = (DQK + 63) / 64; // 64-column TMA boxes
  static constexpr int kVBoxes = (DV + 63) / 64;
  static constexpr int kConsumers = WR * WK;
  static constexpr int kThreads = (kConsumers + 1) * 32;
  static constexpr uint32_t kQBytes = kQBoxes * kRT * 128;
  static constexpr uint32_t kKBytes = kQBoxes * BN * 128;
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;
  static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
  static constexpr uint32_t kRingBytes = NST * kStageBytes;
  // output staging (reuses the ring): per key slice, the CTA's rows in fp32,
  // each padded by 8 floats so the fragment stores spread over the banks
  static constexpr int kOutStride = DV + 8;
  static constexpr uint32_t kOutBytes = WK * kRT * kOutStride * 4;
  static constexpr uint32_t kBarOffset =
      kQBytes + (kRingBytes > kOutBytes ? kRingBytes : kOutBytes);
  static constexpr uint32_t kSmemBytes = kBarOffset + (2 * NST + 1) * 8 + 1024;  // + align slack
  static_assert(DQK % 16 == 0 && DV % 16 == 0, "head dims padded to 16");
  static_assert(kKW % 16 == 0, "each warp takes whole 16-key chunks");
  static_assert(BN % 8 == 0 && BN <= 256, "TMA box height");
  static_assert((kRT * 128) % 1024 == 0 && (BN * 128) % 1024 == 0, "swizzle atoms");
};

template <bool kBF16, int DQK, int DV, int BN, int WR, int WK, int NST, int MINB>
__global__ void __launch_bounds__(SplitKvCfg<DQK, DV, BN, WR, WK, NST>::kThreads, MINB)
    splitkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using Cfg = SplitKvCfg<DQK, DV, BN, WR, WK, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sRing = smem + Cfg::kQBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOffset);
  uint64_t *empty = full + NST;
  uint64_t *qbar = empty + NST;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // --- work item -----------------------------------------------------------
  int bid = blockIdx.x;
  const int row_tile = bid % p.row_tiles;
  bid /= p.row_tiles;
  const int split = bid % p.splits;
  const int bh = bid / p.splits;  // b * Hkv + kv head
  const TileRows tr = tile_rows(p, row_tile, Cfg::kRT);
  int k_lo, k_hi;
  tile_key_range(p, tr, BN, split, k_lo, k_hi);
  const int nblocks = (k_hi - k_lo) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::kConsumers);
    }
    mbar_init(qbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Launched as a programmatic dependent of whatever precedes it on the
  // stream: the setup here may overlap that grid's tail.  Before waiting for
  // it, the producer asks for this CTA's Q tile and first NST key blocks to
  // be brought into L2.  A prefetch only warms L2, which is where every
  // write of that grid lands too, so it cannot hand a stale value to the
  // loads, and those (and every other global access) come after the wait.
  if (warp == Cfg::kConsumers && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
#pragma unroll
    for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
      tma_prefetch_l2_2d(&tm_q, bx * 64, bh * p.R + tr.row0);
    const int npf = nblocks < NST ? nblocks : NST;
    for (int t = 0; t < npf; ++t) {
#pragma unroll
      for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
        tma_prefetch_l2_3d(&tm_k, bx * 64, k_lo + t * BN, bh);
#pragma unroll
      for (int bx = 0; bx < Cfg::kVBoxes; ++bx)
        tma_prefetch_l2_3d(&tm_v, bx * 64, k_lo + t * BN, bh);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Let the dependent combine launch now: its CTAs wait in griddepcontrol.wait
  // until this grid has finished, so its launch latency overlaps this pass.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == Cfg::kConsumers) {
    // ===================== producer warp =====================
    if (lane == 0) {
      const int grow0 = bh * p.R + tr.row0;
      mbar_arrive_expect_tx(qbar, Cfg::kQBytes);
#pragma unroll
      for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
        tma_load_2d(sQ + bx * Cfg::kRT * 128, &tm_q, qbar, bx * 64, grow0);
      int issued = 0;
      for (int t = 0; t < nblocks; ++t) {
        const int s = t % NST;
        const uint32_t ph = (uint32_t)(t / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, p.wd, kWdTmaEmpty)) break;
        uint8_t *sK = sRing + s * Cfg::kStageBytes;
        uint8_t *sV = sK + Cfg::kKBytes;
        mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
        const int k0 = k_lo + t * BN;
#pragma unroll
        for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
          tma_load_3d(sK + bx * BN * 128, &tm_k, &full[s], bx * 64, k0, bh);
#pragma unroll
        for (int bx = 0; bx < Cfg::kVBoxes; ++bx)
          tma_load_3d(sV + bx * BN * 128, &tm_v, &full[s], bx * 64, k0, bh);
        issued = t + 1;
      }
      // Drain: no copy may still be landing in shared memory when the CTA
      // exits (matters only when a wait gave up).
      mbar_wait_drain(qbar, 0, p.wd);
      for (int t = issued - NST > 0 ? issued - NST : 0; t < issued; ++t)
        mbar_wait_drain(&full[t % NST], (uint32_t)(t / NST) & 1u, p.wd);
    }
    return;
  }

  // ===================== consumer warps =====================
  const int rw = warp % WR;   // row group
  const int kw = warp / WR;   // key slice
  const int kw0 = kw * Cfg::kKW;
  constexpr int kNT = Cfg::kKW / 8;   // n8 tiles of scores per warp
  constexpr int kOT = DV / 8;         // n8 tiles of output
  constexpr int kKS = DQK / 16;       // k16 steps of Q K^T

  // the two rows this thread holds (local to the CTA tile) and their positions
  const int lr_a = rw * 16 + (lane >> 2);
  const int lr_b = lr_a + 8;
  const int pos_a = ((tr.row0 + lr_a) % p.L) + p.off;
  const int pos_b = ((tr.row0 + lr_b) % p.L) + p.off;

  float o[kOT][4];
#pragma unroll
  for (int i = 0; i < kOT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  bool ok = mbar_wait(qbar, 0, p.wd, kWdTmaFull);
  const uint32_t sQa = smem_u32(sQ);

  for (int t = 0; ok && t < nblocks; ++t) {
    const int s = t % NST;
    const uint32_t ph = (uint32_t)(t / NST) & 1u;
    if (!mbar_wait(&full[s], ph, p.wd, kWdTmaFull)) {
      ok = false;
      break;
    }
    const uint32_t sK = smem_u32(sRing + s * Cfg::kStageBytes);
    const uint32_t sV = sK + Cfg::kKBytes;
    const int k0 = k_lo + t * BN;

    // ---- S = Q K^T for this warp's 16 rows x kKW keys ----
    float sc[kNT][4];
#pragma unroll
    for (int i = 0; i < kNT; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      uint32_t a0, a1, a2, a3;
      {
        const int m = lane >> 3;
        const uint32_t row = rw * 16 + (m & 1) * 8 + (lane & 7);
        const uint32_t chunk = ks * 2 + (m >> 1);
        ldsm_x4(sQa + (chunk >> 3) * (Cfg::kRT * 128) + sw128_offset(row, chunk & 7), a0, a1, a2,
                a3);
      }
#pragma unroll
      for (int n2 = 0; n2 < kNT / 2; ++n2) {
        const int m = lane >> 3;
        const uint32_t key = kw0 + n2 * 16 + (m >> 1) * 8 + (lane & 7);
        const uint32_t chunk = ks * 2 + (m & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + (chunk >> 3) * (BN * 128) + sw128_offset(key, chunk & 7), b0, b1, b2, b3);
        mma_16816<kBF16>(sc[2 * n2], a0, a1, a2, a3, b0, b1);
        mma_16816<kBF16>(sc[2 * n2 + 1], a0, a1, a2, a3, b2, b3);
      }
    }

    // ---- scale into the log2 domain, mask, online softmax ----
#pragma unroll
    for (int i = 0; i < kNT; ++i) {
      sc[i][0] *= p.scale_log2;
      sc[i][1] *= p.scale_log2;
      sc[i][2] *= p.scale_log2;
      sc[i][3] *= p.scale_log2;
    }
    if (block_needs_mask(p, tr, k0, BN)) {
#pragma unroll
      for (int i = 0; i < kNT; ++i) {
        const int col = k0 + kw0 + i * 8 + (lane & 3) * 2;
        if (!key_visible(p, pos_a, col)) sc[i][0] = -INFINITY;
        if (!key_visible(p, pos_a, col + 1)) sc[i][1] = -INFINITY;
        if (!key_visible(p, pos_b, col)) sc[i][2] = -INFINITY;
        if (!key_visible(p, pos_b, col + 1)) sc[i][3] = -INFINITY;
      }
    }
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int i = 0; i < kNT; ++i) {
      mx_a = fmaxf(mx_a, fmaxf(sc[i][0], sc[i][1]));
      mx_b = fmaxf(mx_b, fmaxf(sc[i][2], sc[i][3]));
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a);
    const float mn_b = fmaxf(m_b, mx_b);
    // a row with nothing visible yet keeps m = -inf; use 0 as its reference
    const float ref_a = mn_a == -INFINITY ? 0.f : mn_a;
    const float ref_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = fast_exp2(m_a - ref_a);
    const float al_b = fast_exp2(m_b - ref_b);
    m_a = mn_a;
    m_b = mn_b;
    float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
    for (int i = 0; i < kNT; ++i) {
      sc[i][0] = fast_exp2(sc[i][0] - ref_a);
      sc[i][1] = fast_exp2(sc[i][1] - ref_a);
      sc[i][2] = fast_exp2(sc[i][2] - ref_b);
      sc[i][3] = fast_exp2(sc[i][3] - ref_b);
      rs_a += sc[i][0] + sc[i][1];
      rs_b += sc[i][2] + sc[i][3];
    }
    l_a = l_a * al_a + rs_a;
    l_b = l_b * al_b + rs_b;
#pragma unroll
    for (int i = 0; i < kOT; ++i) {
      o[i][0] *= al_a;
      o[i][1] *= al_a;
      o[i][2] *= al_b;
      o[i][3] *= al_b;
    }

    // ---- O += P V ----
#pragma unroll
    for (int kc = 0; kc < kNT / 2; ++kc) {
      const uint32_t a0 = pack2<kBF16>(sc[2 * kc][0], sc[2 * kc][1]);
      const uint32_t a1 = pack2<kBF16>(sc[2 * kc][2], sc[2 * kc][3]);
      const uint32_t a2 = pack2<kBF16>(sc[2 * kc + 1][0], sc[2 * kc + 1][1]);
      const uint32_t a3 = pack2<kBF16>(sc[2 * kc + 1][2], sc[2 * kc + 1][3]);
#pragma unroll
      for (int n2 = 0; n2 < kOT / 2; ++n2) {
        const int m = lane >> 3;
        const uint32_t key = kw0 + kc * 16 + (m & 1) * 8 + (lane & 7);
        const uint32_t chunk = n2 * 2 + (m >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + (chunk >> 3) * (BN * 128) + sw128_offset(key, chunk & 7), b0, b1, b2, b3);
        mma_16816<kBF16>(o[2 * n2], a0, a1, a2, a3, b0, b1);
        mma_16816<kBF16>(o[2 * n2 + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // row sums: reduce the per-thread partials over the quad
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

  // ---- epilogue ----
  // Once every consumer has left the loop the ring is free.  Each warp
  // weights its key slice of its rows (the WK slices of a row meet through
  // their (m, l) in shared memory), folds in the row's 1/l, and stages the
  // result there in fp32; then all consumer threads sum the slices and write
  // the tile out row by row, four columns per thread and step.
  __shared__ float2 s_ml[Cfg::kConsumers * 16];  // [key slice][row]: (m, l)
  float *s_o = reinterpret_cast<float *>(sRing);  // [key slice][row][kOutStride]
  constexpr int kOutStride = Cfg::kOutStride;
  const bool va = lr_a < tr.nvalid, vb = lr_b < tr.nvalid;
  const long grow_a = (long)bh * p.R + tr.row0 + lr_a;
  const long grow_b = grow_a + 8;
  const long total_rows = (long)p.B * p.Hq * p.L;
  asm volatile("bar.sync 1, %0;" ::"n"(Cfg::kConsumers * 32) : "memory");
  float f_a = 1.f, f_b = 1.f;  // weight of this slice within its row
  if constexpr (WK > 1) {
    if ((lane & 3) == 0) {
      s_ml[kw * Cfg::kRT + lr_a] = make_float2(m_a, l_a);
      s_ml[kw * Cfg::kRT + lr_b] = make_float2(m_b, l_b);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(Cfg::kConsumers * 32) : "memory");
    float mm_a = -INFINITY, mm_b = -INFINITY;
#pragma unroll
    for (int k = 0; k < WK; ++k) {
      mm_a = fmaxf(mm_a, s_ml[k * Cfg::kRT + lr_a].x);
      mm_b = fmaxf(mm_b, s_ml[k * Cfg::kRT + lr_b].x);
    }
    // a row with no visible key in any slice keeps m = -inf and l = 0
    const float rf_a = mm_a == -INFINITY ? 0.f : mm_a;
    const float rf_b = mm_b == -INFINITY ? 0.f : mm_b;
    float ls_a = 0.f, ls_b = 0.f;
#pragma unroll
    for (int k = 0; k < WK; ++k) {
      const float2 xa = s_ml[k * Cfg::kRT + lr_a];
      const float2 xb = s_ml[k * Cfg::kRT + lr_b];
      ls_a += fast_exp2(xa.x - rf_a) * xa.y;
      ls_b += fast_exp2(xb.x - rf_b) * xb.y;
    }
    f_a = fast_exp2(m_a - rf_a);
    f_b = fast_exp2(m_b - rf_b);
    m_a = mm_a;
    m_b = mm_b;
    l_a = ls_a;
    l_b = ls_b;
  }
  float inv_a, inv_b;
  if (p.splits == 1) {
    inv_a = finish_row(p, grow_a, m_a, l_a);  // folds in the head's sink, if any
    inv_b = finish_row(p, grow_b, m_b, l_b);
  } else {
    inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
    inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  }
  if (kw == 0 && (lane & 3) == 0) {
    float *lse = p.splits == 1 ? p.lse_out : p.part_lse + (long)split * total_rows;
    if (lse != nullptr) {
      if (va) lse[grow_a] = row_lse(m_a, l_a);
      if (vb) lse[grow_b] = row_lse(m_b, l_b);
    }
  }
  {
    const float sa = f_a * inv_a, sb = f_b * inv_b;
    float *row_a = s_o + (kw * Cfg::kRT + lr_a) * kOutStride + (lane & 3) * 2;
    float *row_b = row_a + 8 * kOutStride;
#pragma unroll
    for (int i = 0; i < kOT; ++i) {
      *reinterpret_cast<float2 *>(row_a + i * 8) = make_float2(o[i][0] * sa, o[i][1] * sa);
      *reinterpret_cast<float2 *>(row_b + i * 8) = make_float2(o[i][2] * sb, o[i][3] * sb);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(Cfg::kConsumers * 32) : "memory");
  const int q4 = p.Dv / 4;  // Dv is a multiple of 8
  const int items = tr.nvalid * q4;
  const long grow0 = (long)bh * p.R + tr.row0;
  for (int it = threadIdx.x; it < items; it += Cfg::kConsumers * 32) {
    const int r = it / q4;
    const int c = (it - r * q4) * 4;
    float4 acc = *reinterpret_cast<const float4 *>(s_o + r * kOutStride + c);
#pragma unroll
    for (int k = 1; k < WK; ++k) {
      const float4 x = *reinterpret_cast<const float4 *>(s_o + (k * Cfg::kRT + r) * kOutStride + c);
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    const long at = (grow0 + r) * p.Dv + c;
    if (p.splits == 1) {
      uint2 w;
      w.x = pack2<kBF16>(acc.x, acc.y);
      w.y = pack2<kBF16>(acc.z, acc.w);
      *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(p.out) + at) = w;
    } else {
      *reinterpret_cast<float4 *>(p.part_o + (long)split * total_rows * p.Dv + at) = acc;
    }
  }
  (void)ok;
}

}  // namespace sdpa
