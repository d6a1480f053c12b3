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
//              ... through a ring of NSLOT slots, plus L2 prefetches ahead.
//   warp 9     allocates TMEM and issues every MMA from one thread, in the
//              order S_A(0), S_B(0), then per block j: P_A(j) V_j, S_A(j+1),
//              P_B(j) V_j, S_B(j+1).  Each K/V slot is released after its
//              second use.
//
// TMEM: tile t uses columns [256 t, 256 t + BN) for S (P over the first BN/2
// of them) and [256 t + BN, 256 t + BN + DV) for O.  With one score buffer
// per tile, S_t(j+1) overwrites P_t(j) right after P_t(j) V is issued: one
// thread's MMAs run in issue order.  For the same reason, once S_t(j) is
// complete, P_t(j-1) V is complete too, so the softmax may rescale O_t in
// tensor memory without waiting for anything else.
#pragma once

#include "params.cuh"

namespace sdpa {

template <int DQK, int DV, int BN, int NSLOT>
struct PpCfg {
  static constexpr int kBM = 128;  // rows per tile
  static constexpr int kQBoxes = (DQK + 63) / 64;
  static constexpr int kVBoxes = (DV + 63) / 64;
  static constexpr int kKS = DQK / 16;
  static constexpr int kPVK = BN / 16;
  static constexpr uint32_t kQTileBytes = kQBoxes * kBM * 128;
  static constexpr uint32_t kQBytes = 2 * kQTileBytes;
  static constexpr uint32_t kKBytes = kQBoxes * BN * 128;
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;
  static constexpr uint32_t kSlotBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr uint32_t kSlotOff = kQBytes;
  static constexpr uint32_t kBarOff = kSlotOff + NSLOT * kSlotBytes;
  static constexpr int kNumBars = 2 * NSLOT + 10;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kTileCols = 256;  // TMEM columns per tile
  static constexpr int kPrefetch = 4;    // K/V blocks prefetched into L2 ahead of the loads
  static_assert(DQK % 16 == 0 && DV % 16 == 0 && DV >= 16, "head dims");
  static_assert(BN == 128, "key block");
  static_assert(BN + DV <= kTileCols, "TMEM columns per tile");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

template <bool kBF16, int DQK, int DV, int BN, int NSLOT>
__global__ void __launch_bounds__(320, 1)
    tc_pp_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using Cfg = PpCfg<DQK, DV, BN, NSLOT>;
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
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // --- work item: (batch*KV head) fastest, then split, then the 256-row
  // tile, heaviest first ---
  int bid = blockIdx.x;
  const int BH = p.B * p.Hkv;
  const int bh = bid % BH;
  bid /= BH;
  const int split = bid % p.splits;
  const int pair_tile = p.row_tiles - 1 - bid / p.splits;
  const TileRows tpair = tile_rows(p, pair_tile, 2 * Cfg::kBM);
  int k_lo, k_hi;
  tile_key_range(p, tpair, BN, split, k_lo, k_hi);
  const int nblk = (k_hi - k_lo) / BN;

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

  if (warp == 8) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int grow0 = bh * p.R + tpair.row0;
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
          tma_load_2d(sQ + t * Cfg::kQTileBytes + bx * (Cfg::kBM * 128), &tm_q, q_full, bx * 64,
                      grow0 + t * Cfg::kBM);
      int u = 0;
      bool ok = true;
      for (int j = 0; ok && j < nblk; ++j) {
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
            const int pf = j + Cfg::kPrefetch;
            if (pf < nblk) {
#pragma unroll
              for (int bx = 0; bx < Cfg::kQBoxes; ++bx)
                tma_prefetch_l2_3d(&tm_k, bx * 64, k_lo + pf * BN, bh);
#pragma unroll
              for (int bx = 0; bx < Cfg::kVBoxes; ++bx)
                tma_prefetch_l2_3d(&tm_v, bx * 64, k_lo + pf * BN, bh);
            }
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
        const uint32_t qa = q_addr + t * Cfg::kQTileBytes;
#pragma unroll
        for (int ks = 0; ks < Cfg::kKS; ++ks) {
          const uint64_t a =
              umma_desc_sw128(qa + (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = umma_desc_sw128(kb + (ks >> 2) * (BN * 128) + (ks & 3) * 32, 16, 1024);
          tc_mma_ss(tmem + t * Cfg::kTileCols, a, bd, kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t vb = slot_addr + slot_of(2 * j + 1) * Cfg::kSlotBytes;
#pragma unroll
        for (int ks = 0; ks < Cfg::kPVK; ++ks) {
          const uint64_t bd = umma_desc_sw128_mn(vb + ks * 2048, BN * 128, 1024);
          tc_mma_ts(tmem + t * Cfg::kTileCols + BN, tmem + t * Cfg::kTileCols + ks * 8, bd,
                    kIdescPV, (j > 0 || ks > 0) ? 1u : 0u);
        }
      };
      auto wait_p = [&](int t, int j) -> bool {
        if (!mbar_wait(&p_full[t], (uint32_t)j & 1u, p.wd, kWdSoftmax)) return false;
        tc_fence_after();
        return true;
      };
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
    const uint32_t o_col = s_col + BN;
    TileRows tr = tile_rows(p, pair_tile * 2 + t, Cfg::kBM);
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
    for (int j = 0; j < nblk; ++j) {
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

      if (c_zero) {
#pragma unroll
        for (int i = 0; i < BN; ++i) s[i] = 0.f;
      }
      const int kbase = k_lo + j * BN;
      const bool masked = block_needs_mask(p, tr, kbase, BN);
      if (masked) {
        const VisibleRange vis = visible_range(p, pos, kbase);
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (!vis(i)) s[i] = neutral;
      }
      float mr[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) mr[q4] = s[q4];
      if (c_pos) {
#pragma unroll
        for (int i = 4; i < BN; i += 8) {
          mr[0] = fmax3f(mr[0], s[i], s[i + 1]);
          mr[1] = fmax3f(mr[1], s[i + 2], s[i + 3]);
          if (i + 4 < BN) {
            mr[2] = fmax3f(mr[2], s[i + 4], s[i + 5]);
            mr[3] = fmax3f(mr[3], s[i + 6], s[i + 7]);
          }
        }
        mr[0] = fmax3f(mr[0], mr[1], fmaxf(mr[2], mr[3]));
      } else {
#pragma unroll
        for (int i = 4; i < BN; i += 8) {
          mr[0] = fmin3f(mr[0], s[i], s[i + 1]);
          mr[1] = fmin3f(mr[1], s[i + 2], s[i + 3]);
          if (i + 4 < BN) {
            mr[2] = fmin3f(mr[2], s[i + 4], s[i + 5]);
            mr[3] = fmin3f(mr[3], s[i + 6], s[i + 7]);
          }
        }
        mr[0] = fmin3f(mr[0], mr[1], fminf(mr[2], mr[3]));
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
      // same thread and has completed.
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
        tmem_st_u16x(tmem + lane_base + s_col + c32 * 16, pk);
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
    if (ok && nblk > 0) {
      bool w = true;
      if (lane == 0) w = mbar_wait(&o_final[t], 0, p.wd, kWdMma);
      ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
      tc_fence_after();
    }
    const bool valid = r < tr.nvalid;
    const long grow = (long)bh * p.R + tr.row0 + r;
    const bool have_o = ok && nblk > 0;
    // O leaves TMEM kOGroup chunks of 16 columns per wait
    constexpr int kOChunks = DV / 16;
    constexpr int kOGroup = kOChunks <= 5 ? kOChunks : 4;
    static_assert(kOChunks % kOGroup == 0, "whole groups of O chunks");
    auto load_o = [&](int g, float (&o)[kOGroup][16]) {
      if (have_o) {
    #pragma unroll
        for (int k = 0; k < kOGroup; ++k)
          tmem_ld16(tmem + lane_base + o_col + (g * kOGroup + k) * 16, o[k]);
        tmem_wait_ld();
      } else {
    #pragma unroll
        for (int k = 0; k < kOGroup; ++k)
    #pragma unroll
          for (int e = 0; e < 16; ++e) o[k][e] = 0.f;
      }
    };
    float inv = l > 0.f ? 1.f / l : 0.f;
    if (p.splits == 1) {
      inv = finish_row(p, grow, m_used, l);
      if (p.lse_out != nullptr && valid) p.lse_out[grow] = row_lse(m_used, l);
      uint8_t *orow = reinterpret_cast<uint8_t *>(p.out) + grow * p.Dv * 2;
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
          const int col = (g * kOGroup + k) * 16;
          if (valid && col + 8 <= p.Dv)
            *reinterpret_cast<uint4 *>(orow + col * 2) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
          if (valid && col + 16 <= p.Dv)
            *reinterpret_cast<uint4 *>(orow + col * 2 + 16) =
                make_uint4(w8[4], w8[5], w8[6], w8[7]);
        }
      }
    } else {
      const long total_rows = (long)p.B * p.Hq * p.L;
      float *po = p.part_o + ((long)split * total_rows + grow) * p.Dv;
#pragma unroll 1
      for (int g = 0; g < kOChunks / kOGroup; ++g) {
        float o[kOGroup][16];
        load_o(g, o);
#pragma unroll
        for (int k = 0; k < kOGroup; ++k)
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int col = (g * kOGroup + k) * 16 + q4 * 4;
            if (valid && col + 4 <= p.Dv)
              *reinterpret_cast<float4 *>(po + col) =
                  make_float4(o[k][q4 * 4] * inv, o[k][q4 * 4 + 1] * inv, o[k][q4 * 4 + 2] * inv,
                              o[k][q4 * 4 + 3] * inv);
          }
      }
      if (valid)
        p.part_lse[(long)split * total_rows + grow] = have_o ? row_lse(m_used, l) : -INFINITY;
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
