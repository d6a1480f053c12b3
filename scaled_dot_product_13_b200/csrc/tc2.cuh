// Attention on a pair of SMs: tcgen05 cta_group::2 MMAs over 256-row tiles.
//
// The same method as tc.cuh (key-block range from kb_start / kb_lim, edge
// masks, fp32 online softmax with a lazily moved running max, P in tensor
// memory), but two CTAs of a cluster own one 256-row tile together: CTA r
// holds rows [128 r, 128 r + 128) of Q, of S and of O, while each K block is
// split by keys (CTA r loads keys [r BN/2, (r+1) BN/2) of it) and each V block
// by columns (CTA r loads columns [r DV/2, (r+1) DV/2)).  The even CTA issues
// M=256 MMAs that read both CTAs' shared and tensor memory.  Every K/V byte a
// CTA loads therefore feeds 256 query rows instead of 128, which halves the
// load traffic per FLOP: with 128-row tiles and head dim 256 the kernel is
// limited by how fast K/V reach shared memory, not by the tensor cores.
//
// Loads stay plain TMA into the loading CTA's own shared memory (no
// multicast).  A forwarder warp of the odd CTA relays the completion of each
// of its loads to the even CTA's barriers; the even CTA's MMA thread commits
// to a barrier in both CTAs with one multicast commit (each tcgen05
// instruction costs the issuing thread about 57 cycles).
//
// Warp roles per CTA (224 threads):
//   warps 0-3  softmax on this CTA's 128 rows, one row per thread with all
//              BN columns of a block, so a row's max needs no exchange
//              between warps; lazily moved running max as in tc.cuh.  P_j is
//              written over the row's own scores in this CTA's TMEM and
//              signalled with a CTA-scope arrive: on the even CTA's p_full,
//              or on the odd CTA's p_local.
//   warp 4     TMA producer for this CTA's halves.
//   warp 5     TMEM allocation (pair); the MMA issuer in the even CTA; in
//              the odd CTA it relays each completed p_local phase to the
//              even CTA's p_full.  A cluster-scope release costs the issuing
//              warp several hundred cycles, so it is taken once per block
//              here instead of once per softmax warp on the softmax's path.
//   warp 6     odd CTA: forwards its load completions to the even CTA.
//
// TMEM per CTA: two score buffers of BN columns (P_j over the first BN/2
// columns of buffer j % 2), O at [2 BN, 2 BN + DV).  A score buffer is reused
// two blocks later: the MMA for S_{j+2} is issued after P_j V by the same
// thread, and one thread's tcgen05 MMAs execute in order.
//
// Head dims above 256 run in column halves (grid.y): a launch column loads
// and writes DV of the output columns, and both compute the full scores.
//
// Looping form (PERSIST): a grid of at most one pair per two SMs walks the
// pair tiles in rounds (tc2_item).  Q has two buffers,
// so the next tile's Q load and its first two score MMAs run under the
// current tile's last blocks and epilogue, and a pair pays the launch,
// barrier and TMEM set-up once instead of once per tile.  Block and tile
// counters run on across tiles, so every barrier's phase follows from them.
// A tile's output is staged in its own Q buffer (free once the tile's MMAs
// have completed) and stored from there; the producer refills that buffer
// for the tile after next only once the store has read it (q_empty).  The
// next tile's first P V, which overwrites O, waits for P of that tile's
// first block, which the softmax warps write after they have read O out.
#pragma once

#include "params.cuh"

// How many of every four exponential pairs of the softmax go to the FMA-pipe
// polynomial instead of the MUFU ex2 unit (0-4).  Build-time knob.
#ifndef SDPA_TC2_POLY_OF4
#define SDPA_TC2_POLY_OF4 1
#endif

namespace sdpa {

template <int DQK, int DV, int BN, int NSLOT, bool PERSIST = false>
struct Tc2Cfg {
  static constexpr int kBM = 128;              // rows per CTA (256 per pair)
  static constexpr int kQBufs = PERSIST ? 2 : 1;
  static constexpr int kQBoxes = DQK / 64;
  static constexpr int kVHalf = DV / 2;         // V columns per CTA
  static constexpr int kVBoxes = kVHalf / 64;
  static constexpr int kKS = DQK / 16;
  static constexpr int kPVK = BN / 16;
  static constexpr uint32_t kQBytes = kQBoxes * kBM * 128;
  static constexpr uint32_t kKBytes = kQBoxes * (BN / 2) * 128;  // this CTA's K half
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;        // this CTA's V half
  static constexpr uint32_t kSlotBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr uint32_t kSlotOff = kQBufs * kQBytes;
  static constexpr uint32_t kBarOff = kSlotOff + NSLOT * kSlotBytes;
  static constexpr int kNumBars = 3 * NSLOT + 20;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kThreads = 224;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kOCol = 2 * BN;
  static_assert(DQK % 64 == 0 && (DV == 128 || DV == 256), "pair split needs 64-column halves");
  static_assert(BN == 64 || BN == 128, "key block");
  static_assert(2 * BN + DV <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory");
  // the epilogue stages the CTA's 128 output rows, 64 columns of a 16-bit
  // type or 32 fp32 split partials per 16 KB box: in the K/V slots (one
  // tile per pair), or in the tile's Q buffer (looping form, 16-bit only)
  static constexpr int kOutBoxes = (DV + 63) / 64;
  static constexpr int kF32Boxes = (DV + 31) / 32;
  static_assert(PERSIST ? kOutBoxes * kBM * 128 <= kQBytes
                        : kOutBoxes * kBM * 128 <= NSLOT * kSlotBytes,
                "output staging");
  // whether split partials fit the slots (head dim 512 per column half: not)
  static constexpr bool kSplitStage = !PERSIST && kF32Boxes * kBM * 128 <= NSLOT * kSlotBytes;
};

// One work item of a pair: (batch*KV head) fastest, then split, then the
// 256-row tile, heaviest first.  Rows are packed head-major (row = head in
// the group * L + query), so when whole tiles fit a head's L rows, tiles at
// the same query positions of the group's heads are equally heavy (causal
// and windowed rows see more keys further down): the order then takes the
// last positions of every head first.  Both CTAs derive the same key range.
struct Tc2Tile {
  int bh, split, k_lo, k_hi, nblk;
  TileRows tpair;  // the pair's 256 rows
  TileRows tr;     // this CTA's 128 of them
};

template <int BN, int kBM>
__device__ __forceinline__ Tc2Tile tc2_tile(const AttnParams &p, int item, uint32_t rank) {
  Tc2Tile w;
  const int BH = p.B * p.Hkv;
  w.bh = item % BH;
  item /= BH;
  w.split = item % p.splits;
  const int r = item / p.splits;  // rank of the tile, heaviest first
  const int g = p.R / p.L;
  int pair_tile;
  if (g > 1 && p.L % (2 * kBM) == 0) {
    const int per_head = p.L / (2 * kBM);
    pair_tile = (r % g) * per_head + (per_head - 1 - r / g);
  } else {
    pair_tile = p.row_tiles - 1 - r;
  }
  w.tpair = tile_rows(p, pair_tile, 2 * kBM);
  tile_key_range(p, w.tpair, BN, w.split, w.k_lo, w.k_hi);
  w.nblk = (w.k_hi - w.k_lo) / BN;
  w.tr = tile_rows(p, pair_tile * 2 + (int)rank, kBM);
  if (w.tr.nvalid <= 0) {
    w.tr.nvalid = 0;
    w.tr.pos_min = w.tpair.pos_min;
    w.tr.pos_max = w.tpair.pos_max;
  }
  return w;
}

// The it-th work item of pair `pid` of `npairs`, or -1 when it has no more:
// round it hands items [it*npairs, (it+1)*npairs) out, every other round in
// reverse pair order, so that pairs given the heavier items of one round
// get the lighter ones of the next.
__device__ __forceinline__ int tc2_item(int it, int pid, int npairs, int n_items) {
  const long long idx = (long long)it * npairs + ((it & 1) ? npairs - 1 - pid : pid);
  return idx < n_items ? (int)idx : -1;
}

template <bool kBF16, int DQK, int DV, int BN, int NSLOT, bool PERSIST>
__global__ void __launch_bounds__(224, 1)
    tc2_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_p, const AttnParams p) {
  using Cfg = Tc2Cfg<DQK, DV, BN, NSLOT, PERSIST>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // same layout in both CTAs, so both take this exit together
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) wd_record(p.wd, kWdSmemAlign);
    return;
  }
  // the looping form, and instances whose slots cannot hold fp32 partials,
  // write finished 16-bit rows only (no key splits)
  if (!Cfg::kSplitStage && p.splits != 1) {
    if (threadIdx.x == 0) wd_record(p.wd, kWdConfig);
    return;
  }
  uint8_t *smem = smem_raw;
  uint8_t *sQ = smem;  // [kQBufs][kQBytes]
  uint8_t *sSlots = smem + Cfg::kSlotOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
  uint64_t *slot_full = bars;                // [NSLOT] this CTA's loads landed
  uint64_t *slot_empty = slot_full + NSLOT;  // [NSLOT] the pair's MMA is done with the slot
  uint64_t *peer_full = slot_empty + NSLOT;  // [NSLOT] even CTA: the odd CTA's loads landed
  uint64_t *q_full = peer_full + NSLOT;      // [2] per Q buffer
  uint64_t *peer_q = q_full + 2;             // [2] even CTA: the odd CTA's Q landed
  uint64_t *q_empty = peer_q + 2;            // [2] looping form: the store has read the buffer
  uint64_t *s_full = q_empty + 2;            // [2]
  uint64_t *p_full = s_full + 2;             // [2] even CTA: P_j of both CTAs written
  uint64_t *p_local = p_full + 2;            // [2] odd CTA: P_j of its four warps written
  uint64_t *o_bar = p_local + 2;
  uint64_t *o_final = o_bar + 1;
  uint64_t *fin_bar = o_final + 1;           // all MMAs of the pair complete
  uint64_t *bye_bar = fin_bar + 1;           // teardown: the other CTA is done with us
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bye_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  // --- the pair's work items (tc2_item): one per pair unless looping ---
  const int BH = p.B * p.Hkv;
  const int n_items = BH * p.splits * p.row_tiles;
  const int pid = (int)(blockIdx.x >> 1);
  const int npairs = (int)(gridDim.x >> 1);
  // the DV output columns of this launch column (head dims above 256 run in
  // column halves, grid.y = 2: both halves compute the same scores)
  const int dv0 = (int)blockIdx.y * DV;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
      mbar_init(&peer_full[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&peer_q[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 5);  // the even CTA's four warps, the odd CTA's relay
      mbar_init(&p_local[b], 4);
    }
    mbar_init(o_bar, 1);
    mbar_init(o_final, 1);
    mbar_init(fin_bar, 1);
    mbar_init(bye_bar, 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // barriers of both CTAs are initialised before any remote arrive
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Launched as a programmatic dependent of the previous grid on the stream:
  // the set-up above ran under that grid's tail; nothing below touches
  // global memory before that grid has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 4) {
    // ====================== TMA producer (this CTA's halves) ======================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int u = 0, it = 0;
      bool ok = true;
      for (; ok; ++it) {
        const int item = tc2_item(it, pid, npairs, n_items);
        if (item < 0) break;
        const Tc2Tile w = tc2_tile<BN, Cfg::kBM>(p, item, rank);
        const int qb = it % Cfg::kQBufs, use = it / Cfg::kQBufs;
        // a Q buffer is refilled once the store of the output staged in it
        // (two tiles back) has read it
        if (PERSIST && use > 0 &&
            !mbar_wait(&q_empty[qb], (uint32_t)(use - 1) & 1u, p.wd, kWdTmaEmpty)) {
          ok = false;
          break;
        }
        const int grow0 = w.bh * p.R + w.tpair.row0 + (int)rank * Cfg::kBM;
        uint8_t *q_dst = sQ + qb * Cfg::kQBytes;
        mbar_arrive_expect_tx(&q_full[qb], Cfg::kQBytes);
#pragma unroll
        for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
          tma_load_2d(q_dst + bx * (Cfg::kBM * 128), &tm_q, &q_full[qb], bx * 64, grow0);
        auto emit = [&](bool is_k, int blk) {
          const int slot = u % NSLOT;
          if (!mbar_wait_cluster(&slot_empty[slot], ((uint32_t)(u / NSLOT) & 1u) ^ 1u, p.wd,
                                 kWdTmaEmpty)) {
            ok = false;
            return;
          }
          uint8_t *dst = sSlots + slot * Cfg::kSlotBytes;
          const int k0 = w.k_lo + blk * BN;
          if (is_k) {
            mbar_arrive_expect_tx(&slot_full[slot], Cfg::kKBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
              tma_load_3d(dst + bx * ((BN / 2) * 128), &tm_k, &slot_full[slot], bx * 64,
                          k0 + (int)rank * (BN / 2), w.bh);
          } else {
            mbar_arrive_expect_tx(&slot_full[slot], Cfg::kVBytes);
#pragma unroll
            for (int bx = 0; bx < Cfg::kVBoxes; ++bx)
              tma_load_3d(dst + bx * (BN * 128), &tm_v, &slot_full[slot],
                          dv0 + (int)rank * Cfg::kVHalf + bx * 64, k0, w.bh);
          }
          ++u;
        };
        const int nblk = w.nblk;
        if (nblk > 0) emit(true, 0);
        if (ok && nblk > 1) emit(true, 1);
        for (int j = 0; ok && j < nblk; ++j) {
          emit(false, j);
          if (ok && j + 2 < nblk) emit(true, j + 2);
        }
      }
      // nothing may still land at exit: the last load into each Q buffer
      // and into each slot
      for (int qb = 0; qb < Cfg::kQBufs; ++qb) {
        const int uses = (it - qb + Cfg::kQBufs - 1) / Cfg::kQBufs;
        if (uses > 0) mbar_wait_drain(&q_full[qb], (uint32_t)(uses - 1) & 1u, p.wd);
      }
      for (int v = u - NSLOT > 0 ? u - NSLOT : 0; v < u; ++v)
        mbar_wait_drain(&slot_full[v % NSLOT], (uint32_t)(v / NSLOT) & 1u, p.wd);
    }
  } else if (warp == 6) {
    // ============ odd CTA: relay its load completions to the even CTA ============
    if (!leader && lane == 0) {
      int u = 0, it = 0;
      bool ok = true;
      for (; ok; ++it) {
        const int item = tc2_item(it, pid, npairs, n_items);
        if (item < 0) break;
        const int nblk = tc2_tile<BN, Cfg::kBM>(p, item, rank).nblk;
        const int qb = it % Cfg::kQBufs, use = it / Cfg::kQBufs;
        if (!mbar_wait(&q_full[qb], (uint32_t)use & 1u, p.wd, kWdTmaFull)) break;
        mbar_arrive_cluster(mapa_shared(smem_u32(&peer_q[qb]), 0));
        const int nloads = nblk > 0 ? 2 * nblk : 0;
        for (int v = 0; v < nloads; ++v, ++u) {
          const int slot = u % NSLOT;
          if (!mbar_wait(&slot_full[slot], (uint32_t)(u / NSLOT) & 1u, p.wd, kWdTmaFull)) {
            ok = false;
            break;
          }
          mbar_arrive_cluster(mapa_shared(smem_u32(&peer_full[slot]), 0));
        }
      }
    }
  } else if (warp == 5) {
    // ====================== MMA issuer (even CTA only) ======================
    if (leader && lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_f16(kBF16, 256, BN, false, false);
      constexpr uint32_t kIdescPV = umma_idesc_f16(kBF16, 256, DV, false, true);
      uint32_t q_addr = smem_u32(sQ);
      const uint32_t slot_addr = smem_u32(sSlots);
      // one commit to the barrier at this offset in both CTAs
      auto both = [&](uint64_t *bar) { tc_commit_pair_both(bar); };
      bool ok = true;
      int u = 0;
      auto take_slot = [&](int &slot) -> bool {
        slot = u % NSLOT;
        const uint32_t ph = (uint32_t)(u / NSLOT) & 1u;
        if (!mbar_wait(&slot_full[slot], ph, p.wd, kWdTmaFull)) return false;
        if (!mbar_wait_cluster(&peer_full[slot], ph, p.wd, kWdTmaFull)) return false;
        ++u;
        return true;
      };
      // x: the key block's index counted over all of the pair's tiles
      auto issue_s = [&](int x) -> bool {
        int slot;
        if (!take_slot(slot)) return false;
        const int b = x & 1;
        tc_fence_after();
        const uint64_t a0 = umma_desc_sw128(q_addr, 16, 1024);
        const uint64_t b0 = umma_desc_sw128(slot_addr + slot * Cfg::kSlotBytes, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < Cfg::kKS; ++ks) {
          const uint64_t a = umma_desc_advance(a0, (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32);
          const uint64_t bd = umma_desc_advance(b0, (ks >> 2) * ((BN / 2) * 128) + (ks & 3) * 32);
          tc_mma_ss_pair(tmem + b * BN, a, bd, kIdescS, ks > 0 ? 1u : 0u);
        }
        both(&s_full[b]);
        both(&slot_empty[slot]);
        return true;
      };
      // j: the block within the tile (the first one overwrites O)
      auto issue_pv = [&](int j, int x) -> bool {
        int slot;
        if (!take_slot(slot)) return false;
        const int b = x & 1;
        if (!mbar_wait_cluster(&p_full[b], (uint32_t)(x >> 1) & 1u, p.wd, kWdSoftmax)) return false;
        tc_fence_after();
        const uint64_t v0 = umma_desc_sw128_mn(slot_addr + slot * Cfg::kSlotBytes, BN * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < Cfg::kPVK; ++ks) {
          const uint64_t bd = umma_desc_advance(v0, ks * 2048);
          tc_mma_ts_pair(tmem + Cfg::kOCol, tmem + b * BN + ks * 8, bd, kIdescPV,
                         (j > 0 || ks > 0) ? 1u : 0u);
        }
        both(o_bar);
        both(&slot_empty[slot]);
        return true;
      };
      int it = 0, x0 = 0;
      for (; ok; ++it) {
        const int item = tc2_item(it, pid, npairs, n_items);
        if (item < 0) break;
        const int nblk = tc2_tile<BN, Cfg::kBM>(p, item, rank).nblk;
        const int qb = it % Cfg::kQBufs, use = it / Cfg::kQBufs;
        ok = mbar_wait(&q_full[qb], (uint32_t)use & 1u, p.wd, kWdTmaFull) &&
             mbar_wait_cluster(&peer_q[qb], (uint32_t)use & 1u, p.wd, kWdTmaFull);
        q_addr = smem_u32(sQ + qb * Cfg::kQBytes);
        if (ok && nblk > 0) ok = issue_s(x0);
        if (ok && nblk > 1) ok = issue_s(x0 + 1);
        for (int j = 0; ok && j < nblk; ++j) {
          ok = issue_pv(j, x0 + j);
          if (ok && j + 2 < nblk) ok = issue_s(x0 + j + 2);
        }
        if (ok && nblk > 0) both(o_final);
        x0 += nblk;
      }
      both(fin_bar);
    } else if (!leader && lane == 0) {
      // ============ odd CTA: relay P_x of its softmax warps ============
      const uint32_t leader_p_full = mapa_shared(smem_u32(p_full), 0);
      int it = 0, x = 0;
      bool ok = true;
      for (; ok; ++it) {
        const int item = tc2_item(it, pid, npairs, n_items);
        if (item < 0) break;
        const int nblk = tc2_tile<BN, Cfg::kBM>(p, item, rank).nblk;
        for (int j = 0; j < nblk; ++j, ++x) {
          const int b = x & 1;
          if (!mbar_wait(&p_local[b], (uint32_t)(x >> 1) & 1u, p.wd, kWdSoftmax)) {
            ok = false;
            break;
          }
          mbar_arrive_cluster(leader_p_full + (uint32_t)b * 8u);
        }
      }
    }
  } else {
    // ====== softmax warps 0-3: one row of this CTA's 128 per thread ======
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float c = p.scale_log2;
    // scale 0 weighs every visible key the same: the scores are zeroed and 1
    // is used as the factor, so a masked key (set to the neutral value below)
    // still gives exp2(-inf) = 0 and never exp2(-inf * 0) = NaN
    const bool c_zero = p.scale_log2 == 0.f;
    const float c_eff = c_zero ? 1.f : c;
    const bool c_pos = c >= 0.f;
    const float neutral = c_pos ? -INFINITY : INFINITY;
    const long total_rows = (long)p.B * p.Hq * p.L;
    const bool split_out = p.splits > 1;
    bool ok = true;
    // looping form: the Q buffer whose staged output a TMA store may still be
    // reading (warp 0 lane 0 issued the store); handed back to the producer
    // once the store has read it
    int pend_q = -1;
    auto release_q = [&]() {
      if (PERSIST && warp == 0 && lane == 0 && pend_q >= 0) {
        bulk_wait_group_read0();
        mbar_arrive(&q_empty[pend_q]);
        pend_q = -1;
      }
    };
    int it = 0, x0 = 0, nfin = 0;
    for (; ok; ++it) {
      const int item = tc2_item(it, pid, npairs, n_items);
      if (item < 0) break;
      const Tc2Tile w = tc2_tile<BN, Cfg::kBM>(p, item, rank);
      const TileRows &tr = w.tr;
      const int nblk = w.nblk;
      const int qb = it % Cfg::kQBufs;
      const int pos = ((tr.row0 + r) % p.L) + p.off;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < nblk; ++j) {
        const int x = x0 + j;  // block index over the pair's tiles
        const int b = x & 1;
        bool wt = true;
        if (lane == 0) wt = mbar_wait_cluster(&s_full[b], (uint32_t)(x >> 1) & 1u, p.wd, kWdMma);
        if (!__shfl_sync(0xffffffffu, (int)wt, 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[BN];
        auto load_s = [&]() {
#pragma unroll
          for (int c32 = 0; c32 < BN / 32; ++c32)
            tmem_ld32(tmem + lane_base + b * BN + c32 * 32, s + c32 * 32);
          tmem_wait_ld();
        };
        load_s();

        // ---- P = exp2(s c - m) against the reference in use, packed to the
        // 16-bit type, 32 columns at a time; returns the row sum.  The looping
        // form stores each chunk over the row's own scores as soon as it is
        // made; the one-tile form holds P until the block's check below ----
        uint32_t pk[BN / 2];
        auto exp_block = [&]() -> float {
          const float mref = m_used == -INFINITY ? 0.f : m_used;
          const float2 c2 = make_float2(c_eff, c_eff), nm2 = make_float2(-mref, -mref);
          float2 acc[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) acc[q4] = make_float2(0.f, 0.f);
#pragma unroll
          for (int c32 = 0; c32 < BN / 32; ++c32) {
#pragma unroll
            for (int i2 = 0; i2 < 16; ++i2) {
              const int i = c32 * 32 + 2 * i2;
              float2 t = fma2(make_float2(s[i], s[i + 1]), c2, nm2);
              if ((i2 & 3) < SDPA_TC2_POLY_OF4) {
                t = exp2_poly2(t);  // FMA / ALU pipes
              } else {
                t.x = fast_exp2(t.x);  // MUFU
                t.y = fast_exp2(t.y);
              }
              acc[i2 & 3] = add2(acc[i2 & 3], t);
              pk[c32 * 16 + i2] = pack2<kBF16>(t.x, t.y);
            }
            if constexpr (PERSIST) tmem_st_u16x(tmem + lane_base + b * BN + c32 * 16, pk + c32 * 16);
          }
          const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
          const float2 at = add2(a01, a23);
          return at.x + at.y;
        };

        const int kbase = w.k_lo + j * BN;
        const bool masked = block_needs_mask(p, tr, kbase, BN);
        // One tile per pair: plain blocks (positive scale, no masked key, a
        // reference already set) first take P against the current reference.
        // The reference only moves when a score exceeds it by more than 8
        // (log2 units): then some P is above 2^7.875 (the rounding of s c - m
        // stays below 1/8 while |m| < 2^20), so a row sum below 224 rules it
        // out and the row max is taken only for the rare block whose sum
        // reaches 224 (or is NaN); P, the reference and the sum are those of
        // the max-first order, bit for bit.  The looping form keeps the
        // max-first order: its chunked P stores overwrite the scores a
        // fallback would reload, and holding P instead measured slower there.
        const bool optimistic = !PERSIST && !masked && c_pos && !c_zero &&
                                !__any_sync(0xffffffffu, m_used == -INFINITY);
        float lsum = 0.f;
        bool by_max = true;
        if (optimistic) {
          lsum = exp_block();
          by_max = __any_sync(0xffffffffu, !(lsum < 224.f));
          if (by_max) load_s();  // the scores are still in TMEM (P not stored)
        }
        if (by_max) {
          // The common block (positive scale, no masked key) takes the plain
          // reduction; the rare ones (scale 0, masked keys, negative scale)
          // their own copy, so that their per-element work is not folded in.
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
          const bool any_need = __any_sync(0xffffffffu, need);
          if (j > 0 && any_need) {
            // S_x was issued after P_{x-2} V by the same thread, and P_x V
            // waits for p_full: o_bar is in phase x-1 or x here.  The TMEM
            // loads and stores are warp-wide, so the whole warp rescales its
            // rows.
            if (lane == 0) wt = mbar_wait_cluster(o_bar, (uint32_t)(x - 1) & 1u, p.wd, kWdMma);
            if (!__shfl_sync(0xffffffffu, (int)wt, 0)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int c16 = 0; c16 < DV / 16; ++c16) {
              float o[16];
              tmem_ld16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] *= alpha;
              tmem_st16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
            }
          }
          // P (again, where the reference moved: every lane recomputes, and
          // an unchanged reference gives the same P and sum)
          if (!optimistic || any_need) lsum = exp_block();
        }
        // one tile per pair: P over the first BN/2 columns of the row's own
        // scores, once the block's check has passed
        if constexpr (!PERSIST) {
#pragma unroll
          for (int c32 = 0; c32 < BN / 32; ++c32)
            tmem_st_u16x(tmem + lane_base + b * BN + c32 * 16, pk + c32 * 16);
        }
        l += lsum;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(leader ? &p_full[b] : &p_local[b]);
        // the previous tile's store has long read its buffer by now
        if (j == 0) release_q();
      }

      // ------------------------------ epilogue ------------------------------
      if (ok && nblk > 0) {
        bool wt = true;
        if (lane == 0) wt = mbar_wait_cluster(o_final, (uint32_t)nfin & 1u, p.wd, kWdMma);
        ok = __shfl_sync(0xffffffffu, (int)wt, 0) != 0;
        tc_fence_after();
      }
      if (nblk > 0) ++nfin;
      release_q();  // a tile without blocks released nothing above
      const bool valid = r < tr.nvalid;
      const long grow = (long)w.bh * p.R + tr.row0 + r;
      const bool have_o = ok && nblk > 0;
      // O leaves TMEM kOGroup chunks of 16 columns per wait
      constexpr int kOChunks = DV / 16;
      constexpr int kOGroup = kOChunks <= 5 ? kOChunks : 4;
      static_assert(kOChunks % kOGroup == 0, "whole groups of O chunks");
      auto load_o = [&](int g, float (&o)[kOGroup][16]) {
        if (have_o) {
    #pragma unroll
          for (int k = 0; k < kOGroup; ++k)
            tmem_ld16(tmem + lane_base + Cfg::kOCol + (g * kOGroup + k) * 16, o[k]);
          tmem_wait_ld();
        } else {
    #pragma unroll
          for (int k = 0; k < kOGroup; ++k)
    #pragma unroll
            for (int e = 0; e < 16; ++e) o[k][e] = 0.f;
        }
      };
      // Output rows are staged in the TMA store's swizzled box layout, in this
      // CTA's K/V slots (free: o_final fired once every MMA of the pair had
      // completed) or, looping, in this tile's Q buffer (free for the same
      // reason), then one thread stores them in boxes of 128 rows; rows past
      // the slab and columns past Dv are clipped by the tensor map.
      uint8_t *stage = PERSIST ? sQ + qb * Cfg::kQBytes : sSlots;
      if (!split_out) {
        const float inv = finish_row(p, grow, m_used, l);  // folds in the sink, if any
        if (p.lse_out != nullptr && valid && dv0 == 0) p.lse_out[grow] = row_lse(m_used, l);
#pragma unroll 1
        for (int g = 0; g < kOChunks / kOGroup; ++g) {
          float o[kOGroup][16];
          load_o(g, o);
#pragma unroll
          for (int k = 0; k < kOGroup; ++k) {
            uint32_t w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w8[e] = pack2<kBF16>(o[k][2 * e] * inv, o[k][2 * e + 1] * inv);
            stage_16bit_x16(stage, r, g * kOGroup + k, w8);
          }
        }
      } else if constexpr (Cfg::kSplitStage) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if (valid && dv0 == 0)
          p.part_lse[(long)w.split * total_rows + grow] = have_o ? row_lse(m_used, l) : -INFINITY;
#pragma unroll 1
        for (int g = 0; g < kOChunks / kOGroup; ++g) {
          float o[kOGroup][16];
          load_o(g, o);
#pragma unroll
          for (int k = 0; k < kOGroup; ++k)
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              stage_f32_x4(stage, r, (g * kOGroup + k) * 4 + q4, o[k][q4 * 4] * inv,
                           o[k][q4 * 4 + 1] * inv, o[k][q4 * 4 + 2] * inv, o[k][q4 * 4 + 3] * inv);
        }
      }
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the four softmax warps
      if (warp == 0 && lane == 0) {
        if (tr.nvalid > 0) {
          if (!split_out) {
            for (int bx = 0; bx < Cfg::kOutBoxes && dv0 + bx * 64 < p.Dv; ++bx)
              tma_store_3d(&tm_o, stage + bx * (Cfg::kBM * 128), dv0 + bx * 64, tr.row0, w.bh);
          } else if constexpr (Cfg::kSplitStage) {
            for (int bx = 0; bx < Cfg::kF32Boxes && dv0 + bx * 32 < p.Dv; ++bx)
              tma_store_3d(&tm_p, stage + bx * (Cfg::kBM * 128), dv0 + bx * 32, tr.row0,
                           w.split * BH + w.bh);
          }
          bulk_commit_group();
        }
        if (PERSIST)
          pend_q = qb;  // handed back once read, under the next tile's first block
        else
          bulk_wait_group0();
      }
      x0 += nblk;
    }
    // every store has completed before the CTA leaves
    if (warp == 0 && lane == 0) bulk_wait_group0();
  }

  // ------------------------------ teardown ------------------------------
  // Neither CTA may exit while the other can still reach its shared memory:
  // the even CTA's MMAs read the odd CTA's tiles (done once fin_bar fires in
  // both), and the odd CTA arrives on the even CTA's barriers.  Each CTA
  // signals the other's bye_bar after that and waits for its own, bounded.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_wait_cluster_drain(fin_bar, 0, p.wd);
    mbar_arrive_cluster(mapa_shared(smem_u32(bye_bar), rank ^ 1u));
    mbar_wait_cluster_drain(bye_bar, 0, p.wd);
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::kTmemCols);
  }
}

}  // namespace sdpa
