// Kernel parameter block shared by the attention kernels.
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace sdpa {

// One attention call, as the kernels see it.
//
// Packed rows: for batch b and KV head h, the g = Hq/Hkv query heads that
// read h are consecutive, so their g*L query rows form one contiguous slab of
// R = g*L rows in q and out (row r = j*L + i is query i of head h*g + j).  A
// CTA owns a tile of consecutive slab rows and one range of keys.  Query i
// sits at key position i + off with off = S - L.
struct AttnParams {
  int B, Hq, Hkv, L, S, Dqk, Dv;
  int R;              // packed rows per (b, KV head) = g * L
  int off;            // S - L
  int causal;         // 0/1
  int window;         // 0 = none
  float scale_log2;   // scale * log2(e)
  int row_tiles;      // row tiles per (b, KV head)
  int splits;         // key splits
  int split_base;     // first key of split 0 (a multiple of the key block)
  int keys_per_split; // multiple of the kernel's key block
  void *out;          // [B*Hq*L][Dv] in the I/O type (written when splits == 1)
  float *part_o;      // [splits][B*Hq*L][Dv] fp32, normalised per split
  float *part_lse;    // [splits][B*Hq*L] fp32 natural-log LSE, -inf if empty
  const float *sinks; // optional [Hq] sink logits (natural-log units), applied when splits == 1
  float *lse_out;     // optional [B*Hq*L] natural-log LSE output, written when splits == 1
  Watchdog wd;
};

// Finish one row: fold in the head's sink (one more logit with no value row)
// and return the factor O must be multiplied by; m (log2 units) and l are
// updated to include the sink.  Without a sink the factor is 1/l.
__device__ __forceinline__ float finish_row(const AttnParams &p, long grow, float &m, float &l) {
  if (p.sinks != nullptr) {
    const int hq = (int)((grow / p.L) % p.Hq);
    const float sg = p.sinks[hq] * 1.4426950408889634f;
    const float mf = fmaxf(m, sg);
    const float so = m == -INFINITY ? 0.f : exp2f(m - mf);
    l = l * so + exp2f(sg - mf);
    m = mf;
    return l > 0.f ? so / l : 0.f;
  }
  return l > 0.f ? 1.f / l : 0.f;
}

// Natural-log LSE of a finished row (m in log2 units).
__device__ __forceinline__ float row_lse(float m, float l) {
  return l > 0.f ? (m + log2f(l)) * 0.693147180559945309f : -INFINITY;
}

// Range of positions covered by the valid rows of a tile.
struct TileRows {
  int row0;       // first slab row of the tile
  int nvalid;     // rows of the tile inside the slab
  int pos_min;    // smallest key position of a valid row
  int pos_max;    // largest
};

__device__ __forceinline__ TileRows tile_rows(const AttnParams &p, int row_tile, int rows_per_tile) {
  TileRows t;
  t.row0 = row_tile * rows_per_tile;
  t.nvalid = min(rows_per_tile, p.R - t.row0);
  const int i0 = t.row0 % p.L;
  const int i1 = (t.row0 + t.nvalid - 1) % p.L;
  if (t.nvalid >= p.L || i1 < i0) {  // the tile wraps over a whole head's rows
    t.pos_min = p.off;
    t.pos_max = p.L - 1 + p.off;
  } else {
    t.pos_min = i0 + p.off;
    t.pos_max = i1 + p.off;
  }
  return t;
}

// Key range [k_lo, k_hi) a tile must visit, rounded out to whole key blocks
// of `bn`, then clipped to the split's range [split*kps, (split+1)*kps).
// Causal: keys above the last row's position are skipped (kb_lim).  Window:
// whole blocks left of the first row's window edge are skipped (kb_start)
// (mlx PR #3552, "Implementation").
__device__ __forceinline__ void tile_key_range(const AttnParams &p, const TileRows &t, int bn,
                                               int split, int &k_lo, int &k_hi) {
  const int kend = p.causal ? min(p.S, t.pos_max + 1) : p.S;
  const int kbeg = p.window > 0 ? max(0, t.pos_min - p.window + 1) : 0;
  const int lo = (kbeg / bn) * bn;
  const int hi = ((kend + bn - 1) / bn) * bn;
  const int s_lo = p.split_base + split * p.keys_per_split;
  const int s_hi = s_lo + p.keys_per_split;
  k_lo = max(lo, s_lo);
  k_hi = min(hi, s_hi);
  if (k_hi < k_lo) k_hi = k_lo;
}

// Does key block [k0, k0+bn) need per-element masking for any row of the tile?
__device__ __forceinline__ bool block_needs_mask(const AttnParams &p, const TileRows &t, int k0,
                                                 int bn) {
  if (k0 + bn > p.S) return true;                                  // tail past S
  if (p.causal && k0 + bn - 1 > t.pos_min) return true;            // diagonal
  if (p.window > 0 && k0 <= t.pos_max - p.window) return true;     // window left edge
  return false;
}

__device__ __forceinline__ bool key_visible(const AttnParams &p, int pos, int col) {
  return col < p.S && (!p.causal || col <= pos) && (p.window == 0 || pos - col < p.window);
}

// The keys a row at position pos sees form one interval [lo, hi): the window
// bounds it from below, causality and S from above.  Relative to a block
// starting at key kbase, key kbase + i is visible iff
// (unsigned)(i - (lo - kbase)) < (unsigned)(hi - lo): one subtraction and
// one comparison per key instead of key_visible's three tests.
struct VisibleRange {
  int first;      // lo - kbase
  unsigned span;  // hi - lo (0 when nothing is visible)
  __device__ __forceinline__ bool operator()(int i) const {
    return (unsigned)(i - first) < span;
  }
};

__device__ __forceinline__ VisibleRange visible_range(const AttnParams &p, int pos, int kbase) {
  const int lo = p.window > 0 ? max(0, pos - p.window + 1) : 0;
  const int hi = p.causal ? min(p.S, pos + 1) : p.S;
  VisibleRange v;
  v.first = lo - kbase;
  v.span = hi > lo ? (unsigned)(hi - lo) : 0u;
  return v;
}

// Maximum (or minimum) of a row's N scores of one block, in four chains of
// three-input max (min) operations.
template <int N>
__device__ __forceinline__ float row_reduce_max(const float (&s)[N]) {
  float mr[4];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) mr[q4] = s[q4];
#pragma unroll
  for (int i = 4; i < N; i += 8) {
    mr[0] = fmax3f(mr[0], s[i], s[i + 1]);
    mr[1] = fmax3f(mr[1], s[i + 2], s[i + 3]);
    if (i + 4 < N) {
      mr[2] = fmax3f(mr[2], s[i + 4], s[i + 5]);
      mr[3] = fmax3f(mr[3], s[i + 6], s[i + 7]);
    }
  }
  return fmax3f(mr[0], mr[1], fmaxf(mr[2], mr[3]));
}
template <int N>
__device__ __forceinline__ float row_reduce_min(const float (&s)[N]) {
  float mr[4];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) mr[q4] = s[q4];
#pragma unroll
  for (int i = 4; i < N; i += 8) {
    mr[0] = fmin3f(mr[0], s[i], s[i + 1]);
    mr[1] = fmin3f(mr[1], s[i + 2], s[i + 3]);
    if (i + 4 < N) {
      mr[2] = fmin3f(mr[2], s[i + 4], s[i + 5]);
      mr[3] = fmin3f(mr[3], s[i + 6], s[i + 7]);
    }
  }
  return fmin3f(mr[0], mr[1], fminf(mr[2], mr[3]));
}

}  // namespace sdpa
