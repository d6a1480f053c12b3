// Attention on tcgen05 with two 128-row query tiles per CTA, their softmax
// phases interleaved ("ping-pong"), for head dims up to 128.
//
// At head dims <= 128 one 128x128 block of scores costs the tensor core
// 512-1024 cycles but its softmax (128 exponentials per row, the row max, P
// rounded and written back) several times that, and one tile's softmax
// alternates between latency-bound phases (waiting for scores, loading them
// from tensor memory, storing P) and an exponential phase bound by the MUFU
// unit.  Two tiles in one CTA share every K/V block loaded into shared memory
// and keep the tensor core and the MUFU busy with one tile while the other
// waits: while tile A's softmax works on S_A(j), the tensor core runs
// P_B(j-1) V and S_B(j), and the other way round.
//
// Tiles A and B are rows [0, 128) and [128, 256) of a 256-row tile of packed
// (head-in-group, query) rows of one (batch, KV head).  Both walk the union
// of their key ranges (kb_start / kb_lim of the 256 rows, mlx PR #3552,
// "Implementation"); blocks outside one tile's own range are masked for it
// element by element like any edge block.
//
// Warp roles (320 threads):
//   warps 0-3  softmax of tile A: warp w owns TMEM lanes / rows 32 w .. +31,
//              one row per thread and all BN columns of a block, so a row's
//              max needs no exchange between warps.  fp32 online softmax with
//              a lazily moved running max (see tc.cuh); P is rounded to the
//              16-bit input type and written over the row's own scores.
//   warps 4-7  softmax of tile B, the same on lanes 32 (w-4) .. +31.
//   warp 8     TMA producer: Q of both tiles once, then K_0, V_0, K_1, V_1,
//              ... through a ring of NSLOT slots.
//   warp 9     allocates TMEM and issues every MMA from one thread, in the
//              order S_A(0), S_B(0), then per block j: P_A(j) V_j, S_A(j+1),
//              P_B(j) V_j, S_B(j+1).  Each K/V slot is released after its
//              second use.
//
// Key-split mode (KSPLIT): one 128-row tile whose two softmax groups take
// alternate key blocks instead of separate rows.  Group 0 takes blocks 0, 2,
// 4, ... of the CTA's key range and group 1 blocks 1, 3, 5, ...; both use the
// same Q tile, each K/V block is loaded once and used once (load order K_0,
// K_1, V_0, K_2, V_1, K_3, ...; MMA order S_0(0), S_1(0), then per block b:
// P(b) V_b, S(b + 2)).  Each group keeps its own running max, sum and O, and
// the epilogue merges the two like two key splits (m = max(m_0, m_1),
// O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) + l_1 2^(m_1 - m))),
// each group writing half of the output columns.  This gives 128 rows the
// same overlap of two softmax phases with each other's MMAs that the
// row-pair mode gives 256 rows: for verify windows and short prefill whose
// rows per KV head fill one 128-row tile, with keys to spare.
//
// TMEM: tile t uses columns [256 t, 256 t + BN) for S (P over the first BN/2
// of them) and [256 t + BN, 256 t + BN + DV) for O.  With one score buffer
// per tile, S_t(j+1) overwrites P_t(j) right after P_t(j) V is issued: one
// thread's MMAs run in issue order.  For the same reason, once S_t(j) is
// complete, P_t(j-1) V is complete too, so the softmax may rescale O_t in
// tensor memory without waiting for anything else.
//
// Separate P (row pairs, BN + BN/2 + DV <= 256, i.e. head dims <= 64): P has
// its own columns [256 t + BN, 256 t + 3 BN/2) and O follows it.  The tile's
// softmax signals s_free once it has loaded S_t(j), and the next scores
// S_t(j+1) are issued then, ahead of P_t(j) V, so they compute during the
// softmax instead of after it: MMA order S_A(j+1), P_A(j) V, S_B(j+1),
// P_B(j) V.  P_t(j) V now completes after S_t(j+1), so the softmax of block
// j+1 waits for it (pv_done) before it rescales O_t or writes P_t(j+1).
#pragma once

#include "params.cuh"

namespace sdpa {

template <int DQK, int DV, int BN, int NSLOT, bool KSPLIT = false>
struct PpCfg {
  static constexpr int kBM = 128;  // rows per tile
  static constexpr int kQBoxes = (DQK + 63) / 64;
  static constexpr int kVBoxes = (DV + 63) / 64;
  static constexpr int kKS = DQK / 16;
  static constexpr int kPVK = BN / 16;
  static constexpr uint32_t kQTileBytes = kQBoxes * kBM * 128;
  static constexpr uint32_t kQBytes = (KSPLIT ? 1 : 2) * kQTileBytes;
  static constexpr uint32_t kKBytes = kQBoxes * BN * 128;
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;
  static constexpr uint32_t kSlotBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr uint32_t kSlotOff = kQBytes;
  // key-split merge: (m, l) of every row from each group
  static constexpr uint32_t kXOff = kSlotOff + NSLOT * kSlotBytes;
  static constexpr uint32_t kXBytes = KSPLIT ? 2 * kBM * 8 : 0;
  static constexpr uint32_t kBarOff = kXOff + kXBytes;
  static constexpr int kNumBars = 2 * NSLOT + 14;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kTileCols = 256;  // TMEM columns per tile
  static_assert(DQK % 16 == 0 && DV % 16 == 0 && DV >= 16, "head dims");
  static_assert(BN == 128 || (BN == 96 && !KSPLIT), "key block");
  static_assert(BN + DV <= kTileCols, "TMEM columns per tile");
  // P in its own columns (see above) where the tile's TMEM has room for it
  static constexpr bool kSepP = !KSPLIT && BN + BN / 2 + DV <= kTileCols;
  static constexpr int kPCol = kSepP ? BN : 0;           // P within the tile's columns
  static constexpr int kOCol = kSepP ? BN + BN / 2 : BN;  // O within the tile's columns
  static_assert(kSmemBytes <= 232448, "shared memory");
  // the epilogue stages each tile's output rows in the K/V slots: 64 columns
  // of a 16-bit type, or 32 fp32 split partials, per 16 KB box
  static constexpr int kF32Boxes = (DV + 31) / 32;
  static constexpr uint32_t kStage16 = kVBoxes * kBM * 128;
  static constexpr uint32_t kStageF32 = kF32Boxes * kBM * 128;
  static_assert((KSPLIT ? 1 : 2) * kStageF32 <= NSLOT * kSlotBytes, "output staging");
};

template <bool kBF16, int DQK, int DV, int BN, int NSLOT, bool KSPLIT>
__global__ void __launch_bounds__(320, 1)
    tc_pp_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_p, const AttnParams p) {
  using Cfg = PpCfg<DQK, DV, BN, NSLOT, KSPLIT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) wd_record(p.wd, kWdSmemAlign);
    return;
  }
  uint8_t *smem = smem_raw;
  uint8_t *sQ = smem;  // [tile][box][128 rows][128 B]
  uint8_t *sSlots = smem + Cfg::kSlotOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
  uint64_t *slot_full = bars;                 // [NSLOT]
  uint64_t *slot_empty = bars + NSLOT;        // [NSLOT]
  uint64_t *q_full = bars + 2 * NSLOT;        // Q of both tiles landed
  uint64_t *s_full = q_full + 1;              // [2] S_t(j) complete
  uint64_t *p_full = s_full + 2;              // [2] P_t(j) in TMEM (4 warps each)
  uint64_t *o_final = p_full + 2;             // [2] every P_t V complete
  uint64_t *fin_bar = o_final + 2;            // all MMAs complete (teardown)
  uint64_t *s_free = fin_bar + 1;             // [2] separate P: S_t(j) loaded (4 warps each)
  uint64_t *pv_done = s_free + 2;             // [2] separate P: P_t(j) V complete
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pv_done + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // --- work item: (batch*KV head) fastest, then split, then the row tile
  // (256 rows, or 128 in key-split mode), heaviest first ---
  int bid = blockIdx.x;
  const int BH = p.B * p.Hkv;
  const int bh = bid % BH;
  bid /= BH;
  const int split = bid % p.splits;
  const int pair_tile = p.row_tiles - 1 - bid / p.splits;
  const TileRows tpair = tile_rows(p, pair_tile, (KSPLIT ? 1 : 2) * Cfg::kBM);
  int k_lo, k_hi;
  tile_key_range(p, tpair, BN, split, k_lo, k_hi);
  const int nblk = (k_hi - k_lo) / BN;  // key blocks of the CTA (both groups together)

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    mbar_init(q_full, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);
      mbar_init(&o_final[t], 1);
      mbar_init(&s_free[t], 4);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(fin_bar, 1);
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Launched as a programmatic dependent of the previous grid on the stream:
  // the set-up above ran under that grid's tail; nothing below touches
  // global memory before that grid has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 8) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int grow0 = bh * p.R + tpair.row0;
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
#pragma unroll
      for (int t = 0; t < (KSPLIT ? 1 : 2); ++t)
#pragma unroll
        for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
          tma_load_2d(sQ + t * Cfg::kQTileBytes + bx * (Cfg::kBM * 128), &tm_q, q_full, bx * 64,
                      grow0 + t * Cfg::kBM);
      int u = 0;
      bool ok = true;
      if constexpr (KSPLIT) {
        // K_0, K_1, then V_b, K_{b+2} for b = 0, 1, ...: the order the MMA
        // thread consumes them, each block used once
        auto emit = [&](bool is_k, int blk) {
          const int slot = u % NSLOT;
          if (!mbar_wait(&slot_empty[slot], ((uint32_t)(u / NSLOT) & 1u) ^ 1u, p.wd,
                         kWdTmaEmpty)) {
            ok = false;
            return;
          }
          uint8_t *dst = sSlots + slot * Cfg::kSlotBytes;
          const int k0 = k_lo + blk * BN;
          if (is_k) {
            mbar_arrive_expect_tx(&slot_full[slot], Cfg::kKBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
              tma_load_3d(dst + bx * (BN * 128), &tm_k, &slot_full[slot], bx * 64, k0, bh);
          } else {
            mbar_arrive_expect_tx(&slot_full[slot], Cfg::kVBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kVBoxes; ++bx)
              tma_load_3d(dst + bx * (BN * 128), &tm_v, &slot_full[slot], bx * 64, k0, bh);
          }
          ++u;
        };
        if (nblk > 0) emit(true, 0);
        if (ok && nblk > 1) emit(true, 1);
        for (int b = 0; ok && b < nblk; ++b) {
          emit(false, b);
          if (ok && b + 2 < nblk) emit(true, b + 2);
        }
      }
      for (int j = 0; !KSPLIT && ok && j < nblk; ++j) {
        const int k0 = k_lo + j * BN;
        for (int kv = 0; ok && kv < 2; ++kv, ++u) {
          const int slot = u % NSLOT;
          if (!mbar_wait(&slot_empty[slot], ((uint32_t)(u / NSLOT) & 1u) ^ 1u, p.wd,
                         kWdTmaEmpty)) {
            ok = false;
            break;
          }
          uint8_t *dst = sSlots + slot * Cfg::kSlotBytes;
          if (kv == 0) {
            mbar_arrive_expect_tx(&slot_full[slot], Cfg::kKBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
              tma_load_3d(dst + bx * (BN * 128), &tm_k, &slot_full[slot], bx * 64, k0, bh);
          } else {
            mbar_arrive_expect_tx(&slot_full[slot], Cfg::kVBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kVBoxes; ++bx)
              tma_load_3d(dst + bx * (BN * 128), &tm_v, &slot_full[slot], bx * 64, k0, bh);
          }
        }
      }
      // drain copies still landing (only ever waits after an abort)
      mbar_wait_drain(q_full, 0, p.wd);
      for (int v = u - NSLOT > 0 ? u - NSLOT : 0; v < u; ++v)
        mbar_wait_drain(&slot_full[v % NSLOT], (uint32_t)(v / NSLOT) & 1u, p.wd);
    }
  } else if (warp == 9) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_f16(kBF16, 128, BN, false, false);
      constexpr uint32_t kIdescPV = umma_idesc_f16(kBF16, 128, DV, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t slot_addr = smem_u32(sSlots);
      bool ok = mbar_wait(q_full, 0, p.wd, kWdTmaFull);
      // K_j is load 2 j of the ring and V_j load 2 j + 1
      auto slot_of = [&](int load) { return load % NSLOT; };
      auto wait_load = [&](int load) -> bool {
        return mbar_wait(&slot_full[slot_of(load)], (uint32_t)(load / NSLOT) & 1u, p.wd,
                         kWdTmaFull);
      };
      auto issue_s = [&](int t, int j) {
        const uint32_t kb = slot_addr + slot_of(2 * j) * Cfg::kSlotBytes;
        const uint64_t a0 = umma_desc_sw128(q_addr + t * Cfg::kQTileBytes, 16, 1024);
        const uint64_t b0 = umma_desc_sw128(kb, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < Cfg::kKS; ++ks) {
          const uint64_t a = umma_desc_advance(a0, (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32);
          const uint64_t bd = umma_desc_advance(b0, (ks >> 2) * (BN * 128) + (ks & 3) * 32);
          tc_mma_ss(tmem + t * Cfg::kTileCols, a, bd, kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t vb = slot_addr + slot_of(2 * j + 1) * Cfg::kSlotBytes;
        const uint64_t v0 = umma_desc_sw128_mn(vb, BN * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < Cfg::kPVK; ++ks) {
          const uint64_t bd = umma_desc_advance(v0, ks * 2048);
          tc_mma_ts(tmem + t * Cfg::kTileCols + Cfg::kOCol,
                    tmem + t * Cfg::kTileCols + Cfg::kPCol + ks * 8, bd, kIdescPV,
                    (j > 0 || ks > 0) ? 1u : 0u);
        }
        if constexpr (Cfg::kSepP) tc_commit(&pv_done[t]);
      };
      auto wait_p = [&](int t, int j) -> bool {
        if (!mbar_wait(&p_full[t], (uint32_t)j & 1u, p.wd, kWdSoftmax)) return false;
        tc_fence_after();
        return true;
      };
      if constexpr (KSPLIT) {
        // key-split order: S_0(0) from K_0, S_1(0) from K_1, then per block b
        // of the CTA (group b % 2): P(b) V_b, then S of the group's next block
        // (K_{b+2}) into the buffer P(b) V_b has just been issued to read
        int u = 0;
        auto take = [&](int &slot) -> bool {  // the next load of the ring, in order
          slot = u % NSLOT;
          const bool w =
              mbar_wait(&slot_full[slot], (uint32_t)(u / NSLOT) & 1u, p.wd, kWdTmaFull);
          ++u;
          return w;
        };
        auto s_into = [&](int t, int slot) {
          const uint64_t a0 = umma_desc_sw128(q_addr, 16, 1024);
          const uint64_t b0 = umma_desc_sw128(slot_addr + slot * Cfg::kSlotBytes, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < Cfg::kKS; ++ks) {
            const uint64_t a = umma_desc_advance(a0, (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32);
            const uint64_t bd = umma_desc_advance(b0, (ks >> 2) * (BN * 128) + (ks & 3) * 32);
            tc_mma_ss(tmem + t * Cfg::kTileCols, a, bd, kIdescS, ks > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[t]);
          tc_commit(&slot_empty[slot]);
        };
        auto pv_from = [&](int t, int slot, bool first) {
          const uint64_t v0 = umma_desc_sw128_mn(slot_addr + slot * Cfg::kSlotBytes, BN * 128, 1024);
#pragma unroll
          for (int ks = 0; ks < Cfg::kPVK; ++ks) {
            const uint64_t bd = umma_desc_advance(v0, ks * 2048);
            tc_mma_ts(tmem + t * Cfg::kTileCols + BN, tmem + t * Cfg::kTileCols + ks * 8, bd,
                      kIdescPV, (!first || ks > 0) ? 1u : 0u);
          }
          tc_commit(&slot_empty[slot]);
        };
        int slot = 0;
        for (int b = 0; ok && b < 2 && b < nblk; ++b) {
          ok = take(slot);
          if (!ok) break;
          tc_fence_after();
          s_into(b, slot);
        }
        for (int b = 0; ok && b < nblk; ++b) {
          const int t = b & 1;
          ok = take(slot) && wait_p(t, b >> 1);
          if (!ok) break;
          pv_from(t, slot, b < 2);
          if (b + 2 < nblk) {
            ok = take(slot);
            if (!ok) break;
            tc_fence_after();
            s_into(t, slot);
          }
        }
      } else if constexpr (Cfg::kSepP) {
        if (ok && nblk > 0) {
          ok = wait_load(0);
          if (ok) {
            tc_fence_after();
            issue_s(0, 0);
            issue_s(1, 0);
            tc_commit(&slot_empty[slot_of(0)]);
          }
        }
        auto wait_s_free = [&](int t, int j) -> bool {
          if (!mbar_wait(&s_free[t], (uint32_t)j & 1u, p.wd, kWdSoftmax)) return false;
          tc_fence_after();
          return true;
        };
        for (int j = 0; ok && j < nblk; ++j) {
          const bool more = j + 1 < nblk;
          // tile A: S_A(j+1) once its softmax has loaded S_A(j), then P_A(j) V
          if (more) {
            ok = wait_load(2 * j + 2) && wait_s_free(0, j);
            if (!ok) break;
            issue_s(0, j + 1);
          }
          ok = wait_load(2 * j + 1) && wait_p(0, j);
          if (!ok) break;
          issue_pv(0, j);
          // tile B the same; each slot's second use frees it
          if (more) {
            ok = wait_s_free(1, j);
            if (!ok) break;
            issue_s(1, j + 1);
            tc_commit(&slot_empty[slot_of(2 * j + 2)]);
          }
          ok = wait_p(1, j);
          if (!ok) break;
          issue_pv(1, j);
          tc_commit(&slot_empty[slot_of(2 * j + 1)]);
        }
      } else {
        if (ok && nblk > 0) {
          ok = wait_load(0);
          if (ok) {
            tc_fence_after();
            issue_s(0, 0);
            issue_s(1, 0);
            tc_commit(&slot_empty[slot_of(0)]);
          }
        }
        for (int j = 0; ok && j < nblk; ++j) {
          const bool more = j + 1 < nblk;
          // tile A: P_A(j) V_j, then S_A(j+1)
          ok = wait_load(2 * j + 1) && wait_p(0, j);
          if (!ok) break;
          issue_pv(0, j);
          if (more) {
            ok = wait_load(2 * j + 2);
            if (!ok) break;
            tc_fence_after();
            issue_s(0, j + 1);
          }
          // tile B: P_B(j) V_j, then S_B(j+1); each slot's second use frees it
          ok = wait_p(1, j);
          if (!ok) break;
          issue_pv(1, j);
          tc_commit(&slot_empty[slot_of(2 * j + 1)]);
          if (more) {
            issue_s(1, j + 1);
            tc_commit(&slot_empty[slot_of(2 * j + 2)]);
          }
        }
      }
      if (ok && nblk > 0) {
        tc_commit(&o_final[0]);
        tc_commit(&o_final[1]);
      }
      tc_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0, p.wd);
    }
  } else {
    // ============ softmax: tile t = warp / 4, rows 32 (warp % 4) + lane ============
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_col = (uint32_t)(t * Cfg::kTileCols);
    const uint32_t p_col = s_col + Cfg::kPCol;
    const uint32_t o_col = s_col + Cfg::kOCol;
    TileRows tr = KSPLIT ? tpair : tile_rows(p, pair_tile * 2 + t, Cfg::kBM);
    if (tr.nvalid <= 0) {  // past the slab: compute on zeros, store nothing
      tr.nvalid = 0;
      tr.pos_min = tpair.pos_min;
      tr.pos_max = tpair.pos_max;
    }
    const int pos = ((tr.row0 + r) % p.L) + p.off;
    const float c = p.scale_log2;
    // scale 0 weighs every visible key the same: the scores are zeroed and 1
    // is used as the factor, so a masked key (set to the neutral value below)
    // still gives exp2(-inf) = 0 and never exp2(-inf * 0) = NaN
    const bool c_zero = p.scale_log2 == 0.f;
    const float c_eff = c_zero ? 1.f : c;
    const bool c_pos = c >= 0.f;
    const float neutral = c_pos ? -INFINITY : INFINITY;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // blocks of this group: all of the CTA's (row pairs), or every other one
    // starting at block t (key split)
    const int nb = KSPLIT ? (nblk - t + 1) / 2 : nblk;
    for (int j = 0; j < nb; ++j) {
      bool w = true;
      if (lane == 0) w = mbar_wait(&s_full[t], (uint32_t)j & 1u, p.wd, kWdMma);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c32 = 0; c32 < BN / 32; ++c32)
        tmem_ld32(tmem + lane_base + s_col + c32 * 32, s + c32 * 32);
      tmem_wait_ld();
      if constexpr (Cfg::kSepP) {
        // S_t(j) is in registers: the next scores may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[t]);
      }

      const int kbase = k_lo + (KSPLIT ? 2 * j + t : j) * BN;
      const bool masked = block_needs_mask(p, tr, kbase, BN);
      // The common block (positive scale, no masked key) takes the plain
      // reduction; the rare ones (scale 0, masked keys, negative scale) their
      // own copy, so that their per-element work is not folded into it.
      float mr[1];
      if (!masked && c_pos && !c_zero) {
        mr[0] = row_reduce_max(s);
      } else {
        if (c_zero) {
#pragma unroll
          for (int i = 0; i < BN; ++i) s[i] = 0.f;
        }
        if (masked) {
          const VisibleRange vis = visible_range(p, pos, kbase);
#pragma unroll
          for (int i = 0; i < BN; ++i)
            if (!vis(i)) s[i] = neutral;
        }
        mr[0] = c_pos ? row_reduce_max(s) : row_reduce_min(s);
      }
      const float mblk = isinf(mr[0]) ? -INFINITY : mr[0] * c_eff;
      const float m_new = fmaxf(m_used, mblk);
      const bool need = m_new > m_used + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m_used - m_new);
        m_used = m_new;
        l *= alpha;
      }
      // The TMEM loads and stores are warp-wide (.sync.aligned): the rescale
      // runs for the whole warp when any of its rows moved its max.  O_t holds
      // P_t(0..j-1) V and is stable: S_t(j) was issued after P_t(j-1) V by the
      // same thread and has completed; with separate P, P_t(j-1) V is waited
      // for here (it also frees the P columns for P_t(j)).
      if constexpr (Cfg::kSepP) {
        if (j > 0) {
          bool w = true;
          if (lane == 0) w = mbar_wait(&pv_done[t], (uint32_t)(j - 1) & 1u, p.wd, kWdMma);
          if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c16 = 0; c16 < DV / 16; ++c16) {
          float o[16];
          tmem_ld16(tmem + lane_base + o_col + c16 * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= alpha;
          tmem_st16(tmem + lane_base + o_col + c16 * 16, o);
        }
      }
      // ---- P = exp2(s c - m), row sum, packed P over this row's scores ----
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      const float2 c2 = make_float2(c_eff, c_eff), nm2 = make_float2(-mref, -mref);
      float2 acc[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) acc[q4] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c32 = 0; c32 < BN / 32; ++c32) {
        uint32_t pk[16];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
          const int i = c32 * 32 + 2 * i2;
          float2 e2 = fma2(make_float2(s[i], s[i + 1]), c2, nm2);
          e2.x = fast_exp2(e2.x);
          e2.y = fast_exp2(e2.y);
          acc[i2 & 3] = add2(acc[i2 & 3], e2);
          pk[i2] = pack2<kBF16>(e2.x, e2.y);
        }
        tmem_st_u16x(tmem + lane_base + p_col + c32 * 16, pk);
      }
      const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
      const float2 at = add2(a01, a23);
      l += at.x + at.y;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }

    // ------------------------------ epilogue ------------------------------
    // Output rows go to shared memory in the TMA store's swizzled box layout
    // (the K/V slots are free once o_final has fired: every MMA of the CTA
    // has completed by then), then one thread stores the boxes; rows past
    // the slab and columns past Dv are clipped by the tensor map.  In
    // key-split mode the two groups' (m, l, O) are merged first and each
    // group stages half of the columns.
    if (ok && nblk > 0) {
      bool w = true;
      if (lane == 0) {
        if constexpr (KSPLIT)
          w = mbar_wait(&o_final[0], 0, p.wd, kWdMma) && mbar_wait(&o_final[1], 0, p.wd, kWdMma);
        else
          w = mbar_wait(&o_final[t], 0, p.wd, kWdMma);
      }
      ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
      tc_fence_after();
    }
    constexpr int kOChunks = DV / 16;
    float m_row = m_used, l_row = l, f0 = 1.f, f1 = 0.f;
    bool have0, have1;  // group (tile) 0 / 1 holds O that this thread reads
    int oc_begin = 0, oc_end = kOChunks;
    if constexpr (KSPLIT) {
      float2 *xml = reinterpret_cast<float2 *>(smem + Cfg::kXOff);  // [group][row]
      xml[t * Cfg::kBM + r] = make_float2(m_used, l);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const float2 other = xml[(1 - t) * Cfg::kBM + r];
      m_row = fmaxf(m_used, other.x);
      const float mref = m_row == -INFINITY ? 0.f : m_row;
      const float f_self = m_used == -INFINITY ? 0.f : exp2f(m_used - mref);
      const float f_other = other.x == -INFINITY ? 0.f : exp2f(other.x - mref);
      l_row = l * f_self + other.y * f_other;
      f0 = t == 0 ? f_self : f_other;
      f1 = t == 0 ? f_other : f_self;
      have0 = ok && nblk > 0;
      have1 = ok && nblk > 1;  // group 1 has a block
      constexpr int kHalf = (kOChunks + 1) / 2;
      oc_begin = t == 0 ? 0 : kHalf;
      oc_end = t == 0 ? kHalf : kOChunks;
    } else {
      have0 = ok && nblk > 0;  // this tile's own O
      have1 = false;
    }
    // 16 output columns of this row from TMEM (both groups' O, weighted, in
    // key-split mode; the tile's own O otherwise)
    auto load_o = [&](int c16, float (&o)[16]) {
      float a[16], b[16];
      const uint32_t own = KSPLIT ? (uint32_t)BN : o_col;
      if (have0) tmem_ld16(tmem + lane_base + own + c16 * 16, a);
      if (KSPLIT && have1) tmem_ld16(tmem + lane_base + Cfg::kTileCols + BN + c16 * 16, b);
      if (have0 || have1) tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e)
        o[e] = (have0 ? a[e] * f0 : 0.f) + (KSPLIT && have1 ? b[e] * f1 : 0.f);
    };
    const bool valid = r < tr.nvalid;
    const long grow = (long)bh * p.R + tr.row0 + r;
    const long total_rows = (long)p.B * p.Hq * p.L;
    const bool split_out = p.splits > 1;
    uint8_t *stage =
        sSlots + (KSPLIT ? 0 : t * (split_out ? Cfg::kStageF32 : Cfg::kStage16));
    if (!split_out) {
      const float inv = finish_row(p, grow, m_row, l_row);  // folds in the sink, if any
      if (p.lse_out != nullptr && valid && (!KSPLIT || t == 0))
        p.lse_out[grow] = row_lse(m_row, l_row);
#pragma unroll 1
      for (int c16 = oc_begin; c16 < oc_end; ++c16) {
        float o[16];
        load_o(c16, o);
        uint32_t w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = pack2<kBF16>(o[2 * e] * inv, o[2 * e + 1] * inv);
        stage_16bit_x16(stage, r, c16, w8);
      }
    } else {
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      if (valid && (!KSPLIT || t == 0))
        p.part_lse[(long)split * total_rows + grow] = have0 ? row_lse(m_row, l_row) : -INFINITY;
#pragma unroll 1
      for (int c16 = oc_begin; c16 < oc_end; ++c16) {
        float o[16];
        load_o(c16, o);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          stage_f32_x4(stage, r, c16 * 4 + q4, o[q4 * 4] * inv, o[q4 * 4 + 1] * inv,
                       o[q4 * 4 + 2] * inv, o[q4 * 4 + 3] * inv);
      }
    }
    fence_proxy_async_smem();
    if constexpr (KSPLIT)
      asm volatile("bar.sync 1, 256;" ::: "memory");  // both groups
    else if (t == 0)  // this tile's four warps
      asm volatile("bar.sync 2, 128;" ::: "memory");
    else
      asm volatile("bar.sync 3, 128;" ::: "memory");
    if ((KSPLIT ? warp == 0 : quarter == 0) && lane == 0 && tr.nvalid > 0) {
      if (!split_out) {
        for (int bx = 0; bx < Cfg::kVBoxes && bx * 64 < p.Dv; ++bx)
          tma_store_3d(&tm_o, stage + bx * (Cfg::kBM * 128), bx * 64, tr.row0, bh);
      } else {
        for (int bx = 0; bx < Cfg::kF32Boxes && bx * 32 < p.Dv; ++bx)
          tma_store_3d(&tm_p, stage + bx * (Cfg::kBM * 128), bx * 32, tr.row0,
                       split * BH + bh);
      }
      bulk_commit_group();
      bulk_wait_group0();
    }
  }

  // ------------------------------ teardown ------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace sdpa
