// Attention on tcgen05 tensor cores with TMEM accumulators (sm_100a).
//
// The prefill path, and the split-KV path for packed row counts that fill a
// 128-row MMA tile.  One CTA owns a tile of 128 packed query rows of one
// (batch, KV head) and one range of keys, visited in key blocks of BN:
//   kb_lim (causal) and kb_start (window) bound the block range, and
//   per-element masks run only on the diagonal, window-edge and tail blocks
//   (mlx PR #3552, "Implementation").
//
// Warp roles (192 threads with the default one softmax warp per row group):
//   softmax    4 kParts warps: warps w, w+4, ... share query rows
//              32(w%4) .. +31 (TMEM lanes), each taking 1/kParts of every
//              key block's columns; with kParts > 1 they exchange their row
//              maxima through shared memory behind a bounded mbarrier (with
//              one part a thread owns its whole row).  fp32 online softmax
//              with a lazily updated running max.  P is rounded to the 16-bit
//              input type and written back into tensor memory over the scores
//              it came from.  At the end the epilogue (O / l, rounded,
//              stored), each warp of a row group writing its share of O's
//              columns.
//   producer   (the next warp) TMA producer: Q once, then K and V blocks
//              in the order the MMA consumes them (K0, K1, K2, then V_j,
//              K_{j+3} for j = 0, 1, ...) through a FIFO ring of NSLOT
//              shared-memory slots (128-byte swizzle, zero fill past S and
//              past the head dim).  No L2 prefetch ahead of the loads: it
//              measured slower (the TMA unit serves prefetches before loads).
//   MMA        (the last warp) allocates TMEM and issues tcgen05.mma from
//              one thread: S_j = Q K_j^T (A = Q from shared memory) into
//              score buffer j % 3, and O += P_j V_j with A = P_j read from
//              tensor memory, then S_{j+3}: the scores run up to three
//              blocks ahead of the softmax warps.
//
// TMEM (512 columns x 128 lanes x 32 bit): three score buffers of BN
// columns (P_j overwrites the first BN/2 columns of its buffer as packed
// 16-bit pairs), O at [3 BN, 3 BN + DV).
//
// Running max: the row max m used as the exponent reference is only moved
// when a block's max exceeds it by more than 8 (log2 units), so O in TMEM is
// rescaled rarely.  exp2(s - m) then stays below 2^8, which bf16/fp16 P and
// the fp32 sums hold without loss; l and O share the same reference, so the
// final O / l is the same softmax.  An unmasked block first takes P against
// the reference in use: a row sum below 224 shows that no score passed it by
// 8, and the block's row max (about a fifth of the softmax's time per block)
// is only taken when some row's sum reaches 224.
#pragma once

#include "params.cuh"

// Softmax warps sharing one row of the tile (1, 2 or 4), and how many of every
// four exponential pairs go to the FMA-pipe polynomial instead of the
// MUFU ex2 unit (0-4).  Build-time knobs for measurement.
#ifndef SDPA_TC_PARTS
#define SDPA_TC_PARTS 1
#endif
#ifndef SDPA_TC_POLY_OF4
#define SDPA_TC_POLY_OF4 0
#endif

namespace sdpa {

template <int DQK, int DV, int BN, int NSLOT>
struct TcCfg {
  static constexpr int kBM = 128;
  static constexpr int kBufs = 3;        // score / P buffers in TMEM
  static constexpr int kQBoxes = (DQK + 63) / 64;
  static constexpr int kVBoxes = (DV + 63) / 64;
  static constexpr int kKS = DQK / 16;   // k16 steps of S = Q K^T
  static constexpr int kPVK = BN / 16;   // k16 steps of O += P V
  static constexpr uint32_t kQBytes = kQBoxes * kBM * 128;
  static constexpr uint32_t kKBytes = kQBoxes * BN * 128;
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;
  static constexpr uint32_t kSlotBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr uint32_t kSlotOff = kQBytes;
  static constexpr uint32_t kXOff = kSlotOff + NSLOT * kSlotBytes;  // row-max exchange
  static constexpr int kParts = SDPA_TC_PARTS;      // softmax warps sharing one row
  static constexpr int kSoftmaxWarps = 4 * kParts;
  static constexpr int kProducerWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  static constexpr uint32_t kXBytes = 2 * kParts * kBM * 4;  // [2 bufs][parts][128] row maxima
  static constexpr uint32_t kBarOff = kXOff + kXBytes;
  static constexpr int kNumBars = 2 * NSLOT + 15;
  // exact: the dynamic shared-memory base is 1024-byte aligned (checked at run time)
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
  static constexpr int kCols = BN / kParts;  // key columns per softmax thread
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kOCol = kBufs * BN;
  static_assert(DQK % 16 == 0 && DV % 16 == 0 && DV >= 16 && DV <= 256, "head dims");
  static_assert(BN == 32 || BN == 64 || BN == 128, "key block");
  static_assert(kCols == 16 || kCols % 32 == 0, "TMEM load / store widths");
  static_assert(kBufs * BN + DV <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory");
  // the epilogue stages the tile's output rows in the K/V slots: 64 columns of
  // a 16-bit type, or 32 fp32 split partials, per 16 KB box
  static constexpr int kF32Boxes = (DV + 31) / 32;
  // ... in the K/V slots, or in the Q tile's memory where the slots are too
  // small (head dims 512: Q is done with once the last S has completed)
  static constexpr bool kStageInQ = kF32Boxes * kBM * 128 > NSLOT * kSlotBytes;
  static_assert(!kStageInQ || kF32Boxes * kBM * 128 <= kQBytes, "output staging");
};

template <bool kBF16, int DQK, int DV, int BN, int NSLOT>
__global__ void __launch_bounds__(TcCfg<DQK, DV, BN, NSLOT>::kThreads, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_p, const AttnParams p) {
  using Cfg = TcCfg<DQK, DV, BN, NSLOT>;
  constexpr int NB = Cfg::kBufs;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzle atoms need 1024-byte aligned tiles.  The layout has no
  // slack for realignment, so a misaligned base is reported and the CTA exits
  // before touching barriers or tensor memory.
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) wd_record(p.wd, kWdSmemAlign);
    return;
  }
  uint8_t *smem = smem_raw;
  uint8_t *sQ = smem;
  uint8_t *sSlots = smem + Cfg::kSlotOff;
  float *xmax = reinterpret_cast<float *>(smem + Cfg::kXOff);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
  uint64_t *slot_full = bars;
  uint64_t *slot_empty = bars + NSLOT;
  uint64_t *q_full = bars + 2 * NSLOT;
  uint64_t *s_full = q_full + 1;      // [3] S_j complete (MMA -> softmax)
  uint64_t *p_full = s_full + NB;     // [3] P_j in TMEM, O rescaled (softmax -> MMA)
  uint64_t *o_bar = p_full + NB;      // [2] P_j V complete, on o_bar[j % 2]
  uint64_t *o_final = o_bar + 2;      // one phase: every P V of the tile has completed
  uint64_t *fin_bar = o_final + 1;    // teardown drain of the MMA warp
  uint64_t *part_bar = fin_bar + 1;   // [4] softmax warps of one row group (row-max exchange)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(part_bar + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Output columns of this CTA: all of them, or (head dims above 256, one CTA
  // per 256-column half of V and O, blockIdx.y) the half starting at dv0;
  // each half computes the full scores.
  const int dv0 = (int)blockIdx.y * DV;

  // --- work item: (batch*KV head) fastest, then split, then row tile with
  // the tiles that see the most keys first ---
  int bid = blockIdx.x;
  const int BH = p.B * p.Hkv;
  const int bh = bid % BH;
  bid /= BH;
  const int split = bid % p.splits;
  const int row_tile = p.row_tiles - 1 - bid / p.splits;
  const TileRows tr = tile_rows(p, row_tile, Cfg::kBM);
  int k_lo, k_hi;
  tile_key_range(p, tr, BN, split, k_lo, k_hi);
  const int nblk = (k_hi - k_lo) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    mbar_init(q_full, 1);
    for (int b = 0; b < NB; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], Cfg::kSoftmaxWarps);
    }
    mbar_init(&o_bar[0], 1);
    mbar_init(&o_bar[1], 1);
    mbar_init(o_final, 1);
    mbar_init(fin_bar, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&part_bar[q], Cfg::kParts * 32);
    fence_barrier_init();
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Let a dependent combine launch now (it waits for this grid to finish).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Launched as a programmatic dependent of the previous grid on the stream:
  // the set-up above ran under that grid's tail; nothing below touches
  // global memory before that grid has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == Cfg::kProducerWarp) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int grow0 = bh * p.R + tr.row0;
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
#pragma unroll
      for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
        tma_load_2d(sQ + bx * (Cfg::kBM * 128), &tm_q, q_full, bx * 64, grow0);
      int u = 0;
      bool ok = true;
      // one load into the next ring slot
      auto emit = [&](bool is_k, int blk) {
        const int slot = u % NSLOT;
        const uint32_t ph = (uint32_t)(u / NSLOT) & 1u;
        if (!mbar_wait(&slot_empty[slot], ph ^ 1u, p.wd, kWdTmaEmpty)) {
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
            tma_load_3d(dst + bx * (BN * 128), &tm_v, &slot_full[slot], dv0 + bx * 64, k0, bh);
        }
        ++u;
      };
      if (nblk > 0) emit(true, 0);
      if (ok && nblk > 1) emit(true, 1);
      if (ok && nblk > 2) emit(true, 2);
      for (int j = 0; ok && j < nblk; ++j) {
        emit(false, j);
        if (ok && j + 3 < nblk) emit(true, j + 3);
      }
      // drain copies still landing (only ever waits after an abort)
      mbar_wait_drain(q_full, 0, p.wd);
      for (int v = u - NSLOT > 0 ? u - NSLOT : 0; v < u; ++v)
        mbar_wait_drain(&slot_full[v % NSLOT], (uint32_t)(v / NSLOT) & 1u, p.wd);
    }
  } else if (warp == Cfg::kMmaWarp) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_f16(kBF16, 128, BN, false, false);
      constexpr uint32_t kIdescPV = umma_idesc_f16(kBF16, 128, DV, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t slot_addr = smem_u32(sSlots);
      bool ok = mbar_wait(q_full, 0, p.wd, kWdTmaFull);
      int u = 0;
      // S_n = Q K_n^T into buffer n % 3.  That buffer last held P_{n-3},
      // whose P V this thread issued earlier; one thread's tcgen05 MMAs run
      // in issue order, so no wait is needed before overwriting it.
      auto issue_s = [&](int n) -> bool {
        const int slot = u % NSLOT;
        if (!mbar_wait(&slot_full[slot], (uint32_t)(u / NSLOT) & 1u, p.wd, kWdTmaFull)) return false;
        ++u;
        const int b = n % NB;
        tc_fence_after();
        const uint64_t a0 = umma_desc_sw128(q_addr, 16, 1024);
        const uint64_t b0 = umma_desc_sw128(slot_addr + slot * Cfg::kSlotBytes, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < Cfg::kKS; ++ks) {
          const uint64_t a = umma_desc_advance(a0, (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32);
          const uint64_t bd = umma_desc_advance(b0, (ks >> 2) * (BN * 128) + (ks & 3) * 32);
          tc_mma_ss(tmem + b * BN, a, bd, kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[b]);
        tc_commit(&slot_empty[slot]);
        return true;
      };
      // O += P_j V_j with P_j in TMEM (first BN/2 columns of buffer j % 3)
      auto issue_pv = [&](int j) -> bool {
        const int slot = u % NSLOT;
        if (!mbar_wait(&slot_full[slot], (uint32_t)(u / NSLOT) & 1u, p.wd, kWdTmaFull)) return false;
        ++u;
        const int b = j % NB;
        if (!mbar_wait(&p_full[b], (uint32_t)(j / NB) & 1u, p.wd, kWdSoftmax)) return false;
        tc_fence_after();
        const uint64_t v0 = umma_desc_sw128_mn(slot_addr + slot * Cfg::kSlotBytes, BN * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < Cfg::kPVK; ++ks) {
          const uint64_t bd = umma_desc_advance(v0, ks * 2048);
          tc_mma_ts(tmem + Cfg::kOCol, tmem + b * BN + ks * 8, bd, kIdescPV,
                    (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(&o_bar[j & 1]);
        tc_commit(&slot_empty[slot]);
        return true;
      };
      if (ok && nblk > 0) ok = issue_s(0);
      if (ok && nblk > 1) ok = issue_s(1);
      if (ok && nblk > 2) ok = issue_s(2);
      for (int j = 0; ok && j < nblk; ++j) {
        ok = issue_pv(j);
        if (ok && j + 3 < nblk) ok = issue_s(j + 3);
      }
      // o_bar tells one P V from the next only while at most one is pending;
      // the epilogue needs "all of them", so it gets its own one-shot barrier
      if (ok && nblk > 0) tc_commit(o_final);
      // all MMAs of this CTA complete before TMEM is released
      tc_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0, p.wd);
    }
  } else {
    // ====== softmax warps: rows 32*(w%4) .. +31, column part w/4 of kParts ======
    constexpr int kParts = Cfg::kParts;
    const int quarter = warp & 3;
    const int part = warp >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int pos = ((tr.row0 + r) % p.L) + p.off;
    const float c = p.scale_log2;
    // scale 0 weighs every visible key the same: the scores are zeroed and 1
    // is used as the factor, so a masked key (set to the neutral value below)
    // still gives exp2(-inf) = 0 and never exp2(-inf * 0) = NaN
    const bool c_zero = p.scale_log2 == 0.f;
    const float c_eff = c_zero ? 1.f : c;
    const bool c_pos = c >= 0.f;
    const float neutral = c_pos ? -INFINITY : INFINITY;  // never wins the row reduction
    constexpr int kH = Cfg::kCols;
    constexpr int kOChunks = DV / 16;
    const int oc_begin = part * kOChunks / kParts;
    const int oc_end = (part + 1) * kOChunks / kParts;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t part_phase = 0;
    for (int j = 0; j < nblk; ++j) {
      const int b = j % NB;
      bool w = true;
      if (lane == 0) w = mbar_wait(&s_full[b], (uint32_t)(j / NB) & 1u, p.wd, kWdMma);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kH];
      auto load_s = [&]() {
        if constexpr (kH == 16) {
          float s16[16];
          tmem_ld16(tmem + lane_base + b * BN + part * kH, s16);
#pragma unroll
          for (int i = 0; i < 16; ++i) s[i] = s16[i];
        } else {
#pragma unroll
          for (int c32 = 0; c32 < kH / 32; ++c32)
            tmem_ld32(tmem + lane_base + b * BN + part * kH + c32 * 32, s + c32 * 32);
        }
        tmem_wait_ld();
      };
      load_s();

      // ---- P = exp2(s * c - m) (two lanes per FMA) against the reference m
      // in use, packed to the 16-bit type; returns the row sum ----
      uint32_t pk[kH / 2];
      auto exp_pack = [&]() -> float {
        const float mref = m_used == -INFINITY ? 0.f : m_used;
        const float2 c2 = make_float2(c_eff, c_eff), nm2 = make_float2(-mref, -mref);
        float2 acc[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[t] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kH; i += 2) {
          float2 t = fma2(make_float2(s[i], s[i + 1]), c2, nm2);
          if (((i >> 1) & 3) < SDPA_TC_POLY_OF4) {
            t = exp2_poly2(t);  // FMA / ALU pipes
          } else {
            t.x = fast_exp2(t.x);  // MUFU
            t.y = fast_exp2(t.y);
          }
          acc[(i >> 1) & 3] = add2(acc[(i >> 1) & 3], t);
          pk[i >> 1] = pack2<kBF16>(t.x, t.y);
        }
        const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
        const float2 at = add2(a01, a23);
        return at.x + at.y;
      };

      const int kbase = k_lo + j * BN;
      const bool masked = block_needs_mask(p, tr, kbase, BN);
      // Plain blocks (positive scale, no masked key, a reference already
      // set) first take P against the current reference.  The reference only
      // moves when a score exceeds it by more than 8 (log2 units): then some
      // P is above 2^7.875 (the rounding of s * c - m stays below 1/8 while
      // |m| < 2^20), so a row sum below 224 rules it out and the row max is
      // needed only for the rare block whose sum reaches 224 (or is NaN).
      // (A row of equal scores at the reference, such as the zero-filled
      // padding rows of a partly used tile, sums to BN and stays on the fast
      // side.)
      // Either way P, the reference and the sum are those of the max-first
      // order below, bit for bit.
      const bool optimistic = kParts == 1 && !masked && c_pos && !c_zero &&
                              !__any_sync(0xffffffffu, m_used == -INFINITY);
      float lsum = 0.f;
      bool by_max = true;
      if (optimistic) {
        lsum = exp_pack();
        by_max = __any_sync(0xffffffffu, !(lsum < 224.f));
        if (by_max) load_s();  // the scores are still in TMEM (P not stored)
      }
      if (by_max) {
        // ---- this part's raw row max (masked keys excluded) ----
        // The common block (positive scale, no masked key) takes the plain
        // reduction; the rare ones (scale 0, masked keys, negative scale)
        // their own copy, so that their per-element work is not folded in.
        float mr[1];
        if (!masked && c_pos && !c_zero) {
          mr[0] = row_reduce_max(s);
        } else {
          if (c_zero) {
#pragma unroll
            for (int i = 0; i < kH; ++i) s[i] = 0.f;
          }
          if (masked) {
            const VisibleRange vis = visible_range(p, pos, kbase + part * kH);
#pragma unroll
            for (int i = 0; i < kH; ++i)
              if (!vis(i)) s[i] = neutral;
          }
          mr[0] = c_pos ? row_reduce_max(s) : row_reduce_min(s);
        }
        // ---- combine with the other parts of the row (bounded barrier).
        // The barrier also orders every part's score reads before any part
        // overwrites them with P. ----
        float mraw = mr[0];
        if constexpr (kParts > 1) {
          xmax[((j & 1) * kParts + part) * Cfg::kBM + r] = mr[0];
          tc_fence_before();
          mbar_arrive(&part_bar[quarter]);
          if (!mbar_wait(&part_bar[quarter], part_phase & 1u, p.wd, kWdSoftmax)) {
            ok = false;
            break;
          }
          ++part_phase;
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < kParts; ++q) {
            const float other = xmax[((j & 1) * kParts + q) * Cfg::kBM + r];
            mraw = c_pos ? fmaxf(mraw, other) : fminf(mraw, other);
          }
        }
        const float mblk = isinf(mraw) ? -INFINITY : mraw * c_eff;
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
          // O holds P_0..P_{j-1} V: wait for the last P V, then rescale this
          // warp's columns in TMEM.  P_{j-1} V commits to o_bar[(j-1) % 2] as
          // that barrier's phase (j-1) / 2.  The parity is unambiguous: S_j was
          // issued after P_{j-3} V by the same thread, so S_j's completion
          // implies the barrier's previous phase (P_{j-3} V) completed, and its
          // next one (P_{j+1} V) waits for p_full of a block not yet done.
          if (lane == 0)
            w = mbar_wait(&o_bar[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, p.wd, kWdMma);
          if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c16 = oc_begin; c16 < oc_end; ++c16) {
            float o[16];
            tmem_ld16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= alpha;
            tmem_st16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
          }
          tmem_wait_st();
        }
        // P again where the reference moved (every lane recomputes: an
        // unchanged reference gives the same P and sum)
        if (!optimistic || any_need) lsum = exp_pack();
      }
      l += lsum;
      // P_j into this warp's packed columns of buffer b (over the first
      // BN/2 score columns)
      if constexpr (kH == 16) {
        tmem_st_u8x(tmem + lane_base + b * BN + part * (kH / 2), pk);
      } else {
#pragma unroll
        for (int c16 = 0; c16 < kH / 32; ++c16)
          tmem_st_u16x(tmem + lane_base + b * BN + part * (kH / 2) + c16 * 16, pk + c16 * 16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }

    // ------------------------------ epilogue ------------------------------
    // row sum = the parts' partial sums, exchanged through the max buffer the
    // last block did not use (its last reader passed the last barrier)
    if constexpr (kParts > 1) {
      float *xl = xmax + (nblk & 1) * kParts * Cfg::kBM;
      xl[part * Cfg::kBM + r] = l;
      mbar_arrive(&part_bar[quarter]);
      if (!mbar_wait(&part_bar[quarter], part_phase & 1u, p.wd, kWdSoftmax)) ok = false;
      l = 0.f;
#pragma unroll
      for (int q = 0; q < kParts; ++q) l += xl[q * Cfg::kBM + r];
    }
    if (ok && nblk > 0) {
      bool w = true;
      if (lane == 0) w = mbar_wait(o_final, 0, p.wd, kWdMma);
      ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
      tc_fence_after();
    }
    const bool valid = r < tr.nvalid;
    const long grow = (long)bh * p.R + tr.row0 + r;
    const bool have_o = ok && nblk > 0;
    // Output rows are staged in the K/V slots (free: o_final fired once every
    // MMA of the CTA had completed) in the TMA store's swizzled box layout,
    // then one thread stores them in boxes of 128 rows; rows past the slab
    // and columns past Dv are clipped by the tensor map.
    const long total_rows = (long)p.B * p.Hq * p.L;
    const bool split_out = p.splits > 1;
    uint8_t *stage = Cfg::kStageInQ ? sQ : sSlots;
    auto load_o = [&](int c16, float (&o)[16]) {
      if (have_o) {
        tmem_ld16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] = 0.f;
      }
    };
    if (!split_out) {
      const float inv = finish_row(p, grow, m_used, l);  // folds in the sink, if any
      if (p.lse_out != nullptr && valid && part == 0 && dv0 == 0)
        p.lse_out[grow] = row_lse(m_used, l);
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
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (valid && part == 0 && dv0 == 0)
        p.part_lse[(long)split * total_rows + grow] = have_o ? row_lse(m_used, l) : -INFINITY;
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
    asm volatile("bar.sync 1, %0;" ::"n"(Cfg::kSoftmaxWarps * 32) : "memory");  // softmax warps
    if (warp == 0 && lane == 0 && tr.nvalid > 0) {
      if (!split_out) {
        for (int bx = 0; bx < Cfg::kVBoxes && dv0 + bx * 64 < p.Dv; ++bx)
          tma_store_3d(&tm_o, stage + bx * (Cfg::kBM * 128), dv0 + bx * 64, tr.row0, bh);
      } else {
        for (int bx = 0; bx < Cfg::kF32Boxes && dv0 + bx * 32 < p.Dv; ++bx)
          tma_store_3d(&tm_p, stage + bx * (Cfg::kBM * 128), dv0 + bx * 32, tr.row0,
                       split * BH + bh);
      }
      bulk_commit_group();
      bulk_wait_group0();
    }
  }

  // ------------------------------ teardown ------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace sdpa
