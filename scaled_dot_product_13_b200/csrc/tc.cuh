// Attention on tcgen05 tensor cores with TMEM accumulators (sm_100a).
//
// The prefill path, and the split-KV path for packed row counts that fill a
// 128-row MMA tile.  One CTA owns a tile of 128 packed query rows of one
// (batch, KV head) and one range of keys, visited in key blocks of BN:
//   kb_lim (causal) and kb_start (window) bound the block range, and
//   per-element masks run only on the diagonal, window-edge and tail blocks
//   (mlx PR #3552, "Implementation").
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile (TMEM lane t);
//              fp32 online softmax with a lazily updated running max, P
//              written to shared memory as the 16-bit input type; at the end
//              the epilogue (O / l, rounded, stored).
//   warp 4     TMA producer: Q once, then K and V blocks, in the order the
//              MMA consumes them (K0, K1, V0, K2, V1, ...), through a FIFO
//              ring of NSLOT shared-memory slots (128-byte swizzle, zero fill
//              past S and past the head dim).
//   warp 5     allocates TMEM and issues tcgen05.mma from one thread:
//              S_j = Q K_j^T into one of two TMEM score buffers, then
//              O += P_{j-1} V_{j-1} into the TMEM output accumulator, so the
//              tensor core computes the next scores while the softmax warps
//              work on the current ones.
//
// TMEM (512 columns x 128 lanes x 32 bit): S buffers at columns [0, BN) and
// [BN, 2BN), O at [2BN, 2BN + DV).
//
// Running max: the row max m used as the exponent reference is only moved
// when a block's max exceeds it by more than 8 (log2 units), so O in TMEM is
// rescaled rarely.  exp2(s - m) then stays below 2^8, which bf16/fp16 P and
// the fp32 sums hold without loss; l and O share the same reference, so the
// final O / l is the same softmax.
#pragma once

#include "params.cuh"

namespace sdpa {

template <int DQK, int DV, int BN, int NSLOT>
struct TcCfg {
  static constexpr int kBM = 128;
  static constexpr int kQBoxes = (DQK + 63) / 64;
  static constexpr int kVBoxes = (DV + 63) / 64;
  static constexpr int kKS = DQK / 16;   // k16 steps of S = Q K^T
  static constexpr int kPVK = BN / 16;   // k16 steps of O += P V
  static constexpr uint32_t kQBytes = kQBoxes * kBM * 128;
  static constexpr uint32_t kKBytes = kQBoxes * BN * 128;
  static constexpr uint32_t kVBytes = kVBoxes * BN * 128;
  static constexpr uint32_t kSlotBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr uint32_t kPBytes = kBM * BN * 2;
  static constexpr uint32_t kPOff = kQBytes;
  static constexpr uint32_t kSlotOff = kPOff + 2 * kPBytes;
  static constexpr uint32_t kBarOff = kSlotOff + NSLOT * kSlotBytes;
  static constexpr int kNumBars = 2 * NSLOT + 13;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kOCol = 2 * BN;
  static_assert(DQK % 16 == 0 && DV % 16 == 0 && DV >= 16 && DV <= 256, "head dims");
  static_assert(BN == 64 || BN == 128, "key block");
  static_assert(2 * BN + DV <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

template <bool kBF16, int DQK, int DV, int BN, int NSLOT>
__global__ void __launch_bounds__(192, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using Cfg = TcCfg<DQK, DV, BN, NSLOT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sP = smem + Cfg::kPOff;
  uint8_t *sSlots = smem + Cfg::kSlotOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kBarOff);
  uint64_t *slot_full = bars;
  uint64_t *slot_empty = bars + NSLOT;
  uint64_t *q_full = bars + 2 * NSLOT;
  uint64_t *s_full = q_full + 1;   // [2]
  uint64_t *s_free = s_full + 2;   // [2]
  uint64_t *p_full = s_free + 2;   // [2]
  uint64_t *p_free = p_full + 2;   // [2]
  uint64_t *o_bar = p_free + 2;
  uint64_t *fin_bar = o_bar + 1;
  uint64_t *o_final = fin_bar + 1;  // one phase: every P V of the tile has completed
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_final + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(o_bar, 1);
    mbar_init(fin_bar, 1);
    mbar_init(o_final, 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
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
      // load order = MMA consumption order: K0, (K_j, V_{j-1}) for j >= 1, V_last
      const int nloads = nblk > 0 ? 2 * nblk : 0;
      for (int t = 0; t < nloads && ok; ++t) {
        bool is_k;
        int blk;
        if (t == 0) {
          is_k = true; blk = 0;
        } else if (t == nloads - 1) {
          is_k = false; blk = nblk - 1;
        } else {
          is_k = (t & 1) != 0;
          blk = is_k ? (t + 1) / 2 : t / 2 - 1;
        }
        const int slot = u % NSLOT;
        const uint32_t ph = (uint32_t)(u / NSLOT) & 1u;
        if (!mbar_wait(&slot_empty[slot], ph ^ 1u, p.wd, kWdTmaEmpty)) {
          ok = false;
          break;
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
      }
      // drain copies still landing (only ever waits after an abort)
      mbar_wait_drain(q_full, 0, p.wd);
      for (int v = u - NSLOT > 0 ? u - NSLOT : 0; v < u; ++v)
        mbar_wait_drain(&slot_full[v % NSLOT], (uint32_t)(v / NSLOT) & 1u, p.wd);
    }
  } else if (warp == 5) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_f16(kBF16, 128, BN, false, false);
      constexpr uint32_t kIdescPV = umma_idesc_f16(kBF16, 128, DV, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      const uint32_t slot_addr = smem_u32(sSlots);
      bool ok = mbar_wait(q_full, 0, p.wd, kWdTmaFull);
      int u = 0;
      auto pv = [&](int i) -> bool {
        const int slot = u % NSLOT;
        if (!mbar_wait(&slot_full[slot], (uint32_t)(u / NSLOT) & 1u, p.wd, kWdTmaFull)) return false;
        ++u;
        const int pb = i & 1;
        if (!mbar_wait(&p_full[pb], (uint32_t)(i >> 1) & 1u, p.wd, kWdSoftmax)) return false;
        tc_fence_after();
        const uint32_t vb = slot_addr + slot * Cfg::kSlotBytes;
        const uint32_t pbase = p_addr + pb * Cfg::kPBytes;
#pragma unroll
        for (int ks = 0; ks < Cfg::kPVK; ++ks) {
          const uint64_t a = umma_desc_sw128(pbase + (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32,
                                             16, 1024);
          const uint64_t b = umma_desc_sw128_mn(vb + ks * 2048, BN * 128, 1024);
          tc_mma_ss(tmem + Cfg::kOCol, a, b, kIdescPV, (i > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(o_bar);
        tc_commit(&p_free[pb]);
        tc_commit(&slot_empty[slot]);
        return true;
      };
      for (int j = 0; ok && j < nblk; ++j) {
        const int slot = u % NSLOT;
        if (!mbar_wait(&slot_full[slot], (uint32_t)(u / NSLOT) & 1u, p.wd, kWdTmaFull)) {
          ok = false;
          break;
        }
        ++u;
        const int sb = j & 1;
        if (!mbar_wait(&s_free[sb], ((uint32_t)(j >> 1) & 1u) ^ 1u, p.wd, kWdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = slot_addr + slot * Cfg::kSlotBytes;
#pragma unroll
        for (int ks = 0; ks < Cfg::kKS; ++ks) {
          const uint64_t a =
              umma_desc_sw128(q_addr + (ks >> 2) * (Cfg::kBM * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(kb + (ks >> 2) * (BN * 128) + (ks & 3) * 32, 16, 1024);
          tc_mma_ss(tmem + sb * BN, a, b, kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        tc_commit(&slot_empty[slot]);
        if (j >= 1 && !pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && nblk > 0) ok = pv(nblk - 1);
      // o_bar tells one P V from the next only while at most one is pending;
      // the epilogue needs "all of them", so it gets its own one-shot barrier
      if (ok && nblk > 0) tc_commit(o_final);
      // all MMAs of this CTA complete before TMEM is released
      tc_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0, p.wd);
    }
  } else {
    // ====================== softmax warps (rows 0..127) ======================
    const int r = warp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int pos = ((tr.row0 + r) % p.L) + p.off;
    const float c = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const uint32_t p_row = smem_u32(sP) + r * 128;
    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      bool w = true;
      if (lane == 0) w = mbar_wait(&s_full[sb], (uint32_t)(j >> 1) & 1u, p.wd, kWdMma);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c32 = 0; c32 < BN / 32; ++c32)
        tmem_ld32(tmem + lane_base + sb * BN + c32 * 32, s + c32 * 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      const int k0 = k_lo + j * BN;
#pragma unroll
      for (int i = 0; i < BN; ++i) s[i] *= c;
      if (block_needs_mask(p, tr, k0, BN)) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (!key_visible(p, pos, k0 + i)) s[i] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < BN; ++i) mx = fmaxf(mx, s[i]);
      const float m_new = fmaxf(m_used, mx);
      const bool need = m_new > m_used + 8.0f;
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m_used - m_new);
        m_used = m_new;
        l *= alpha;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds P_0..P_{j-1} V: wait for the last P V, then rescale in TMEM.
        // Parity is unambiguous here: S_j's completion implies P_{j-2} V
        // completed (one thread issues both, in order), and P_j V is not
        // issued before this warp signals p_full, so o_bar is in phase j-1
        // or j.
        if (lane == 0) w = mbar_wait(o_bar, (uint32_t)(j - 1) & 1u, p.wd, kWdMma);
        if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
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
        tmem_wait_st();
      }
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < BN; ++i) {
        s[i] = fast_exp2(s[i] - mref);
        rs += s[i];
      }
      l += rs;
      // P buffer sb is free once the P V that last read it has completed
      if (lane == 0) w = mbar_wait(&p_free[sb], ((uint32_t)(j >> 1) & 1u) ^ 1u, p.wd, kWdMma);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
        ok = false;
        break;
      }
      const uint32_t pb = p_row + sb * Cfg::kPBytes;
#pragma unroll
      for (int ch = 0; ch < BN / 8; ++ch) {
        const uint32_t addr = pb + (ch >> 3) * (Cfg::kBM * 128) + ((((uint32_t)ch & 7u) ^ ((uint32_t)r & 7u)) << 4);
        st_shared_v4(addr, pack2<kBF16>(s[ch * 8 + 0], s[ch * 8 + 1]),
                     pack2<kBF16>(s[ch * 8 + 2], s[ch * 8 + 3]),
                     pack2<kBF16>(s[ch * 8 + 4], s[ch * 8 + 5]),
                     pack2<kBF16>(s[ch * 8 + 6], s[ch * 8 + 7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }

    // ------------------------------ epilogue ------------------------------
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (ok && nblk > 0) {
      bool w = true;
      if (lane == 0) w = mbar_wait(o_final, 0, p.wd, kWdMma);
      ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
      tc_fence_after();
    }
    const bool valid = r < tr.nvalid;
    const long grow = (long)bh * p.R + tr.row0 + r;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const bool have_o = ok && nblk > 0;
    if (p.splits == 1) {
      uint8_t *orow = reinterpret_cast<uint8_t *>(p.out) + grow * p.Dv * 2;
#pragma unroll 1
      for (int c16 = 0; c16 < DV / 16; ++c16) {
        float o[16];
        if (have_o) {
          tmem_ld16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0.f;
        }
        uint32_t w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = pack2<kBF16>(o[2 * e] * inv, o[2 * e + 1] * inv);
        const int col = c16 * 16;
        if (valid && col + 8 <= p.Dv)
          *reinterpret_cast<uint4 *>(orow + col * 2) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        if (valid && col + 16 <= p.Dv)
          *reinterpret_cast<uint4 *>(orow + col * 2 + 16) = make_uint4(w8[4], w8[5], w8[6], w8[7]);
      }
    } else {
      const long total_rows = (long)p.B * p.Hq * p.L;
      float *po = p.part_o + ((long)split * total_rows + grow) * p.Dv;
#pragma unroll 1
      for (int c16 = 0; c16 < DV / 16; ++c16) {
        float o[16];
        if (have_o) {
          tmem_ld16(tmem + lane_base + Cfg::kOCol + c16 * 16, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0.f;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int col = c16 * 16 + q4 * 4;
          if (valid && col + 4 <= p.Dv)
            *reinterpret_cast<float4 *>(po + col) =
                make_float4(o[q4 * 4] * inv, o[q4 * 4 + 1] * inv, o[q4 * 4 + 2] * inv,
                            o[q4 * 4 + 3] * inv);
        }
      }
      if (valid) {
        constexpr float kLn2 = 0.693147180559945309f;
        p.part_lse[(long)split * total_rows + grow] =
            (have_o && l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }

  // ------------------------------ teardown ------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace sdpa
