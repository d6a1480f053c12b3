// Attention for head dims above 256 (up to 512), split over the output
// columns instead of over the keys.
//
// With Dv = 512 one warp cannot hold the fp32 output of its 16 rows in
// registers (256 per thread), and one 128-row tensor-memory tile would need
// all 512 TMEM columns for O alone.  So the four consumer warps of a 16-row
// group share each key block: for S = Q K^T warp w takes keys
// [w BN/4, (w+1) BN/4) of the block over the whole Dqk, and for O += P V warp
// w owns output columns [w Dv/4, (w+1) Dv/4) over all BN keys.  The block's
// row maximum and P cross between the four warps through shared memory, with
// two named barriers per block.  The online softmax itself is the one of the
// split-KV kernel (fp32 running max and sum per row, O rescaled when the max
// moves, P rounded to the 16-bit input type for the P V product).
//
// CTA = (row tile of 16 WR packed rows, key split, batch*KV head), WR row
// groups of four warps plus one TMA producer warp that streams Q once and
// K/V blocks through an NST-stage ring (128-byte swizzled 64-column boxes,
// zero fill past S and past the head dims).  Several key splits are merged by
// the log-sum-exp combine as on the split-KV path.
//
// The pages' vector and full kernels stop at head dim 256 and raise for 512
// (mlx PR #4185, "Kernel support"); this kernel is the 512 case.
#pragma once

#include "params.cuh"

namespace sdpa {

template <int DQK, int DV, int BN, int WR, int NST>
struct WideCfg {
  static constexpr int kWD = 4;                   // warps sharing one 16-row group
  static constexpr int kRT = 16 * WR;             // rows per CTA
  static constexpr int kKW = BN / kWD;            // keys per warp for S
  static constexpr int kCols = DV / kWD;          // output columns per warp
  static constexpr int kQBoxes = DQK / 64;
  static constexpr int kVBoxes = DV / 64;
  static constexpr int kConsumers = WR * kWD;
  static constexpr int kThreads = (kConsumers + 1) * 32;
  static constexpr uint32_t kQBytes = kQBoxes * kRT * 128;
  static constexpr uint32_t kKBytes = kQBoxes * BN * 128;
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;
  static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
  static constexpr uint32_t kRingOff = kQBytes;
  static constexpr uint32_t kPStride = BN * 2;    // bytes per P row (16-byte chunks XOR-swizzled)
  static constexpr uint32_t kPOff = kRingOff + NST * kStageBytes;
  static constexpr uint32_t kXOff = kPOff + kRT * kPStride;
  static constexpr uint32_t kXBytes = WR * kWD * 16 * 4;
  static constexpr uint32_t kBarOff = kXOff + kXBytes;
  static constexpr uint32_t kSmemBytes = kBarOff + (2 * NST + 1) * 8;
  static_assert(DQK % 64 == 0 && DV % 64 == 0, "64-column TMA boxes");
  static_assert(BN == 32, "one n8 score tile per warp; four 16-byte P chunks per row");
  static_assert(kCols % 16 == 0, "pairs of n8 output tiles per warp");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// Byte offset of 16-byte chunk `chunk` (0..3) of P row `row`: the chunk
// index is XORed with (row / 2) % 4 so that the eight rows one ldmatrix
// reads fall on distinct banks.
__device__ __forceinline__ uint32_t wide_p_offset(uint32_t row, uint32_t chunk) {
  return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

template <bool kBF16, int DQK, int DV, int BN, int WR, int NST>
__global__ void __launch_bounds__(WideCfg<DQK, DV, BN, WR, NST>::kThreads, 1)
    wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using Cfg = WideCfg<DQK, DV, BN, WR, NST>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) wd_record(p.wd, kWdSmemAlign);
    return;
  }
  uint8_t *smem = smem_raw;
  uint8_t *sQ = smem;
  uint8_t *sRing = smem + Cfg::kRingOff;
  uint8_t *sP = smem + Cfg::kPOff;
  float *xbuf = reinterpret_cast<float *>(smem + Cfg::kXOff);  // [WR][kWD][16]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
  uint64_t *empty = full + NST;
  uint64_t *qbar = empty + NST;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // --- work item: row tile fastest, then split, then batch*KV head ---
  int bid = blockIdx.x;
  const int row_tile = bid % p.row_tiles;
  bid /= p.row_tiles;
  const int split = bid % p.splits;
  const int bh = bid / p.splits;
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
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == Cfg::kConsumers) {
    // ===================== producer warp =====================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(qbar, Cfg::kQBytes);
#pragma unroll
      for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
        tma_load_2d(sQ + bx * Cfg::kRT * 128, &tm_q, qbar, bx * 64, bh * p.R + tr.row0);
      int issued = 0;
      for (int t = 0; t < nblocks; ++t) {
        const int s = t % NST;
        if (!mbar_wait(&empty[s], ((uint32_t)(t / NST) & 1u) ^ 1u, p.wd, kWdTmaEmpty)) break;
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
      mbar_wait_drain(qbar, 0, p.wd);
      for (int t = issued - NST > 0 ? issued - NST : 0; t < issued; ++t)
        mbar_wait_drain(&full[t % NST], (uint32_t)(t / NST) & 1u, p.wd);
    }
    return;
  }

  // ===================== consumer warps =====================
  const int rw = warp / Cfg::kWD;   // row group
  const int wd = warp % Cfg::kWD;   // key slice for S, column slice for O
  const int kw0 = wd * Cfg::kKW;
  const int col0 = wd * Cfg::kCols;
  constexpr int kOT = Cfg::kCols / 8;  // n8 output tiles per warp
  constexpr int kKS = DQK / 16;        // k16 steps of Q K^T
  const uint32_t bar_id = 1 + rw;      // named barrier of this row group
  float *xg = xbuf + rw * Cfg::kWD * 16;

  const int lr_a = lane >> 2;          // rows of this thread inside the 16-row group
  const int lr_b = lr_a + 8;
  const int tr_a = rw * 16 + lr_a;     // ... inside the CTA tile
  const int tr_b = rw * 16 + lr_b;
  const int pos_a = ((tr.row0 + tr_a) % p.L) + p.off;
  const int pos_b = ((tr.row0 + tr_b) % p.L) + p.off;

  float o[kOT][4];
#pragma unroll
  for (int i = 0; i < kOT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  bool ok = __all_sync(0xffffffffu, mbar_wait(qbar, 0, p.wd, kWdTmaFull));
  const uint32_t sQa = smem_u32(sQ);
  const uint32_t sPa = smem_u32(sP) + rw * 16 * Cfg::kPStride;

  for (int t = 0; t < nblocks; ++t) {
    // every warp of the row group runs every block (the named barriers need
    // all four); after a failed wait a warp keeps going without touching the
    // ring and stops releasing stages, so the producer gives up too
    const int s = t % NST;
    if (ok) ok = mbar_wait(&full[s], (uint32_t)(t / NST) & 1u, p.wd, kWdTmaFull);
    ok = __all_sync(0xffffffffu, ok);
    const uint32_t sK = smem_u32(sRing + s * Cfg::kStageBytes);
    const uint32_t sV = sK + Cfg::kKBytes;
    const int k0 = k_lo + t * BN;

    // ---- S = Q K^T: 16 rows x this warp's 8 keys, over all of Dqk ----
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
#pragma unroll 4
      for (int ks = 0; ks < kKS; ks += 2) {
        const int m = lane >> 3;
        uint32_t b0, b1, b2, b3;
        {
          const uint32_t key = kw0 + (lane & 7);
          const uint32_t chunk = ks * 2 + m;
          ldsm_x4(sK + (chunk >> 3) * (BN * 128) + sw128_offset(key, chunk & 7), b0, b1, b2, b3);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t row = rw * 16 + (m & 1) * 8 + (lane & 7);
          const uint32_t chunk = (ks + h) * 2 + (m >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(sQa + (chunk >> 3) * (Cfg::kRT * 128) + sw128_offset(row, chunk & 7), a0, a1,
                  a2, a3);
          if (h == 0) mma_16816<kBF16>(sc, a0, a1, a2, a3, b0, b1);
          else mma_16816<kBF16>(sc, a0, a1, a2, a3, b2, b3);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] *= p.scale_log2;
    if (block_needs_mask(p, tr, k0, BN)) {
      const int col = k0 + kw0 + (lane & 3) * 2;
      if (!key_visible(p, pos_a, col)) sc[0] = -INFINITY;
      if (!key_visible(p, pos_a, col + 1)) sc[1] = -INFINITY;
      if (!key_visible(p, pos_b, col)) sc[2] = -INFINITY;
      if (!key_visible(p, pos_b, col + 1)) sc[3] = -INFINITY;
    }
    float mx_a = fmaxf(sc[0], sc[1]), mx_b = fmaxf(sc[2], sc[3]);
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    if ((lane & 3) == 0) {
      xg[wd * 16 + lr_a] = mx_a;
      xg[wd * 16 + lr_b] = mx_b;
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(Cfg::kWD * 32) : "memory");
#pragma unroll
    for (int w = 0; w < Cfg::kWD; ++w) {
      mx_a = fmaxf(mx_a, xg[w * 16 + lr_a]);
      mx_b = fmaxf(mx_b, xg[w * 16 + lr_b]);
    }
    const float mn_a = fmaxf(m_a, mx_a);
    const float mn_b = fmaxf(m_b, mx_b);
    const float ref_a = mn_a == -INFINITY ? 0.f : mn_a;
    const float ref_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = fast_exp2(m_a - ref_a);
    const float al_b = fast_exp2(m_b - ref_b);
    m_a = mn_a;
    m_b = mn_b;
    const float p0 = fast_exp2(sc[0] - ref_a), p1 = fast_exp2(sc[1] - ref_a);
    const float p2 = fast_exp2(sc[2] - ref_b), p3 = fast_exp2(sc[3] - ref_b);
    l_a = l_a * al_a + (p0 + p1);
    l_b = l_b * al_b + (p2 + p3);
#pragma unroll
    for (int i = 0; i < kOT; ++i) {
      o[i][0] *= al_a;
      o[i][1] *= al_a;
      o[i][2] *= al_b;
      o[i][3] *= al_b;
    }
    {  // P of this warp's 8 keys into the row group's P tile
      const uint32_t kcol = kw0 + (lane & 3) * 2;   // key within the block
      const uint32_t chunk = kcol >> 3, within = (kcol & 7) * 2;
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(sPa + wide_p_offset(lr_a, chunk) + within),
                   "r"(pack2<kBF16>(p0, p1))
                   : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(sPa + wide_p_offset(lr_b, chunk) + within),
                   "r"(pack2<kBF16>(p2, p3))
                   : "memory");
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(Cfg::kWD * 32) : "memory");

    // ---- O[:, this warp's columns] += P V ----
    if (ok) {
#pragma unroll
      for (int kc = 0; kc < BN / 16; ++kc) {
        const int m = lane >> 3;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sPa + wide_p_offset((m & 1) * 8 + (lane & 7), kc * 2 + (m >> 1)), a0, a1, a2, a3);
#pragma unroll
        for (int n2 = 0; n2 < kOT / 2; ++n2) {
          const uint32_t key = kc * 16 + (m & 1) * 8 + (lane & 7);
          const uint32_t chunk = col0 / 8 + n2 * 2 + (m >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sV + (chunk >> 3) * (BN * 128) + sw128_offset(key, chunk & 7), b0, b1, b2, b3);
          mma_16816<kBF16>(o[2 * n2], a0, a1, a2, a3, b0, b1);
          mma_16816<kBF16>(o[2 * n2 + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&empty[s]);
  }

  // ---- row sums: quad, then across the four warps of the row group ----
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  // the last block's maxima were read before its second barrier, so the
  // exchange buffer is free again
  if ((lane & 3) == 0) {
    xg[wd * 16 + lr_a] = l_a;
    xg[wd * 16 + lr_b] = l_b;
  }
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(Cfg::kWD * 32) : "memory");
  l_a = 0.f;
  l_b = 0.f;
#pragma unroll
  for (int w = 0; w < Cfg::kWD; ++w) {
    l_a += xg[w * 16 + lr_a];
    l_b += xg[w * 16 + lr_b];
  }

  // ---- epilogue: this warp's output columns ----
  float inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
  float inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  const bool va = tr_a < tr.nvalid, vb = tr_b < tr.nvalid;
  const long grow_a = (long)bh * p.R + tr.row0 + tr_a;
  const long grow_b = (long)bh * p.R + tr.row0 + tr_b;
  const int c0 = col0 + (lane & 3) * 2;
  if (p.splits == 1) {
    inv_a = finish_row(p, grow_a, m_a, l_a);
    inv_b = finish_row(p, grow_b, m_b, l_b);
    if (p.lse_out != nullptr && wd == 0 && (lane & 3) == 0) {
      if (va) p.lse_out[grow_a] = row_lse(m_a, l_a);
      if (vb) p.lse_out[grow_b] = row_lse(m_b, l_b);
    }
    uint32_t *out32 = reinterpret_cast<uint32_t *>(p.out);
#pragma unroll
    for (int i = 0; i < kOT; ++i) {
      const int col = c0 + i * 8;
      if (col < p.Dv) {
        if (va) out32[(grow_a * p.Dv + col) >> 1] = pack2<kBF16>(o[i][0] * inv_a, o[i][1] * inv_a);
        if (vb) out32[(grow_b * p.Dv + col) >> 1] = pack2<kBF16>(o[i][2] * inv_b, o[i][3] * inv_b);
      }
    }
  } else {
    const long total_rows = (long)p.B * p.Hq * p.L;
    float *po = p.part_o + (long)split * total_rows * p.Dv;
#pragma unroll
    for (int i = 0; i < kOT; ++i) {
      const int col = c0 + i * 8;
      if (col < p.Dv) {
        if (va)
          *reinterpret_cast<float2 *>(po + grow_a * p.Dv + col) =
              make_float2(o[i][0] * inv_a, o[i][1] * inv_a);
        if (vb)
          *reinterpret_cast<float2 *>(po + grow_b * p.Dv + col) =
              make_float2(o[i][2] * inv_b, o[i][3] * inv_b);
      }
    }
    if (wd == 0 && (lane & 3) == 0) {
      float *pl = p.part_lse + (long)split * total_rows;
      if (va) pl[grow_a] = row_lse(m_a, l_a);
      if (vb) pl[grow_b] = row_lse(m_b, l_b);
    }
  }
}

}  // namespace sdpa
