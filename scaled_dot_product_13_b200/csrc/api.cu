// C ABI of libsdpa: argument validation, the router (planner), workspace
// handling, TMA descriptor encoding and launch sequencing.
//
// The router never falls back to a non-fused path: a problem either maps to a
// fused kernel instance or the call fails with a message that names the
// violated constraint (mlx PR #4185, "API": force_fused raises with the
// unsupported constraint; "Kernel support": the dispatch-time check that
// prevents silent zero output).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "launch.h"
#include "ptx.cuh"

// Device watchdog word (see sdpa_device_status).
__device__ unsigned int g_sdpa_watchdog_word;

namespace sdpa {

namespace {

thread_local std::string t_last_error;
thread_local cudaEvent_t t_ev_start = nullptr, t_ev_stop = nullptr, t_ev_call = nullptr;
std::atomic<uint64_t> g_wait_limit_ns{0};
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s

sdpa_status fail(sdpa_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

sdpa_status fail_str(sdpa_status st, const std::string &msg) {
  t_last_error = msg;
  return st;
}

// Test-only fault injection on the host, read once when the library loads
// (no device fault is involved; the injected failure is a host-side error
// return, taken before anything is enqueued):
//   SDPA_TEST_FAIL_ALLOC=1      the stream-ordered workspace allocation of the
//                               allocating entry points fails;
//   SDPA_TEST_SMEM_LIMIT=<n>    the pre-launch resource check compares each
//                               kernel's shared memory with n bytes instead of
//                               the device's limit.
struct TestHooks {
  bool fail_alloc = false;
  long long smem_limit = -1;
  TestHooks() {
    const char *a = getenv("SDPA_TEST_FAIL_ALLOC");
    fail_alloc = a != nullptr && a[0] != '\0' && a[0] != '0';
    const char *m = getenv("SDPA_TEST_SMEM_LIMIT");
    if (m != nullptr && m[0] != '\0') smem_limit = atoll(m);
  }
};
const TestHooks g_test_hooks;

uint64_t wait_limit() {
  const uint64_t v = g_wait_limit_ns.load();
  return v ? v : kDefaultWaitLimitNs;
}

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

sdpa_status validate_shape(const Problem &p) {
  if (p.B < 1 || p.Hq < 1 || p.Hkv < 1 || p.L < 1 || p.S < 1)
    return fail(SDPA_ERR_INVALID_ARG,
                "B, Hq, Hkv, L, S must all be >= 1 (got B=%d Hq=%d Hkv=%d L=%d S=%d)", p.B, p.Hq,
                p.Hkv, p.L, p.S);
  if (p.Hq % p.Hkv != 0)
    return fail(SDPA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", p.Hq, p.Hkv);
  if (p.dtype != SDPA_BF16 && p.dtype != SDPA_F16)
    return fail(SDPA_ERR_UNSUPPORTED, "dtype %d is not supported (bf16 = 0, f16 = 1)",
                (int)p.dtype);
  if (p.causal != 0 && p.causal != 1)
    return fail(SDPA_ERR_INVALID_ARG, "causal must be 0 or 1 (got %d)", p.causal);
  if (p.causal && !p.has_q_offset && p.L > p.S)
    return fail(SDPA_ERR_INVALID_ARG,
                "causal attention needs L <= S (got L=%d > S=%d): queries are aligned to the "
                "end of the keys, so the first rows would see no key",
                p.L, p.S);
  if (p.has_q_offset) {
    if (p.q_offset < -(1 << 30) || p.q_offset > (1 << 30))
      return fail(SDPA_ERR_UNSUPPORTED, "q_offset must lie in [-2^30, 2^30] (got %d)", p.q_offset);
    if (p.causal && p.q_offset < 0)
      return fail(SDPA_ERR_INVALID_ARG,
                  "causal attention needs q_offset >= 0 (got %d): query row 0 would see no key",
                  p.q_offset);
  }
  if (p.window < 0)
    return fail(SDPA_ERR_INVALID_ARG, "window_size must be >= 0 (got %d)", p.window);
  if (p.window > 0 && !p.causal)
    return fail(SDPA_ERR_UNSUPPORTED,
                "window_size > 0 is defined only together with causal masking (got causal=0, "
                "window_size=%d)",
                p.window);
  if (p.window > 0 && (long long)p.q_offset + p.L - 1 - (p.window - 1) > (long long)p.S - 1)
    return fail(SDPA_ERR_INVALID_ARG,
                "window_size=%d with q_offset=%d: the last query row (position %d) sees no key "
                "of the %d held",
                p.window, p.q_offset, p.q_offset + p.L - 1, p.S);
  if (!std::isfinite(p.scale))
    return fail(SDPA_ERR_INVALID_ARG, "scale must be finite");
  for (int d : {p.Dqk, p.Dv}) {
    if (d < 8 || d > 512 || d % 8 != 0)
      return fail(SDPA_ERR_UNSUPPORTED,
                  "head dims must be multiples of 8 in [8, 512] (got Dqk=%d, Dv=%d)", p.Dqk,
                  p.Dv);
  }
  const long long rows = (long long)p.B * p.Hq * p.L;
  if (rows > 0x7fffffffLL || (long long)p.B * p.Hkv * p.S > 0x7fffffffLL)
    return fail(SDPA_ERR_UNSUPPORTED,
                "B*Hq*L and B*Hkv*S must each stay below 2^31 (got %lld and %lld)", rows,
                (long long)p.B * p.Hkv * p.S);
  return SDPA_OK;
}

sdpa_status validate_pointers(const Problem &p, const void *q, const void *k, const void *v,
                              const void *out) {
  if (!q || !k || !v || !out)
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL device pointers");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
  const size_t nq = (size_t)p.B * p.Hq * p.L * p.Dqk * 2;
  const size_t nk = (size_t)p.B * p.Hkv * p.S * p.Dqk * 2;
  const size_t nv = (size_t)p.B * p.Hkv * p.S * p.Dv * 2;
  const size_t no = (size_t)p.B * p.Hq * p.L * p.Dv * 2;
  if (overlaps(out, no, q, nq) || overlaps(out, no, k, nk) || overlaps(out, no, v, nv))
    return fail(SDPA_ERR_INVALID_ARG, "out must not overlap q, k or v");
  return SDPA_OK;
}

// ---------------------------------------------------------------------------
// router
// ---------------------------------------------------------------------------
int pick_pair(int dqk, int dv) {
  for (int i = 0; i < kNumDimPairs; ++i)
    if (kDimPairs[i].dqk >= dqk && kDimPairs[i].dv >= dv) return i;
  return -1;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Upper bound on key splits (the combine keeps one weight per split in
// shared memory).
constexpr int kMaxSplits = 4096;

// Packed rows per (batch, KV head) from which the tcgen05 path is taken:
// above two 16-row warp tiles, one 128-row tensor-memory tile costs less
// (measured on the verify sweep: 48 and 64 rows faster there, 32 slower).
constexpr int kTcRowThreshold = 33;
// ... and, at head dims above 256, from which it takes over from the
// column-split warp-tile kernel.
constexpr int kTcRowThresholdWide = 65;
// ... and from which head dims 256/256 and 192/128 take the two-CTA kernel.
constexpr int kTc2RowThreshold = 256;

// A split must cover at least this many key blocks, and problems of at most
// kNoSplitBlocks key blocks are not split: below that the combine launch
// costs more than the parallelism gains.  The split-KV kernel counts in
// 64-key units (128 and 256 keys) whatever its key block.
constexpr int kMinBlocksPerSplit = 2;
constexpr int kMinBlocksPerSplitWide = 8;
constexpr int kNoSplitBlocks = 4;
// Splits the combine merges per round trip (one per lane of a warp).
constexpr int kCombineRound = 32;

// The pair kernel loops over its tiles (SDPA_PATH_TC2_LOOP) when a tile visits
// at most this many key blocks: there a tile's fill and epilogue are a large
// share of its time and the loop hides them under the neighbouring tiles.
constexpr int kLoopMaxTileBlocks = 48;

sdpa_status make_plan(const Problem &pb, int num_sms, int force_path, int force_splits,
                      Plan *out) {
  Plan pl;
  memset(&pl, 0, sizeof(pl));
  pl.col_halves = 1;
  pl.pair = pick_pair(pb.Dqk, pb.Dv);
  if (pl.pair < 0)
    return fail(SDPA_ERR_UNSUPPORTED, "no kernel instance covers Dqk=%d, Dv=%d", pb.Dqk, pb.Dv);
  if (force_path != SDPA_PATH_AUTO && force_path != SDPA_PATH_SPLITKV &&
      force_path != SDPA_PATH_TC && force_path != SDPA_PATH_TC2 && force_path != SDPA_PATH_WIDE &&
      force_path != SDPA_PATH_TC_DUAL && force_path != SDPA_PATH_TC_KSPLIT &&
      force_path != SDPA_PATH_TC2_LOOP)
    return fail(SDPA_ERR_INVALID_ARG, "unknown path %d", force_path);
  // head dims above 256 run on the column-split warp-tile kernel (decode and
  // short verify windows) or on the tcgen05 kernel in column halves; the
  // column-split kernel only on them
  const bool wide = pl.pair == kWidePair;
  if (force_path == SDPA_PATH_WIDE && !wide)
    return fail(SDPA_ERR_UNSUPPORTED,
                "the wide path is built for head dims above 256 (got Dqk=%d, Dv=%d)", pb.Dqk,
                pb.Dv);
  if (wide && force_path != SDPA_PATH_AUTO && force_path != SDPA_PATH_WIDE &&
      force_path != SDPA_PATH_TC && force_path != SDPA_PATH_TC2)
    return fail(SDPA_ERR_UNSUPPORTED,
                "head dims above 256 (got Dqk=%d, Dv=%d) run on the wide path or the tcgen05 "
                "paths (one or two SMs per tile)",
                pb.Dqk, pb.Dv);
  if (force_splits < 0) return fail(SDPA_ERR_INVALID_ARG, "force_splits must be >= 0");
  if (num_sms < 1) num_sms = 148;
  const int g = pb.Hq / pb.Hkv;
  pl.rows = g * pb.L;

  // Route: packed rows that fill a 128-row tensor-core tile go to the
  // tcgen05 kernel; fewer rows (decode, short verify windows) go to the
  // split-KV kernel on 16-row warp tiles.  Both split the keys when the
  // tiles alone do not fill the GPU.
  int path = force_path;
  // head dims above 256: packed rows that fill a 128-row tile take tcgen05;
  // from one 256-row tile, and with at least one pair's work per two SMs
  // (that kernel does not split the keys), an SM pair per tile
  if (path == SDPA_PATH_AUTO && wide) {
    path = pl.rows >= kTcRowThresholdWide ? SDPA_PATH_TC : SDPA_PATH_WIDE;
    const long long pair_units = (long long)pb.B * pb.Hkv * ((pl.rows + 255) / 256) *
                                 ((pb.Dv + kTc2WideHalf - 1) / kTc2WideHalf);
    if (pl.rows >= kTc2RowThreshold && 2 * pair_units >= num_sms) path = SDPA_PATH_TC2;
  }
  if (path == SDPA_PATH_AUTO) {
    path = pl.rows >= kTcRowThreshold ? SDPA_PATH_TC : SDPA_PATH_SPLITKV;
    // wide heads with at least one full 256-row pair tile: two SMs per tile.
    // Causal or windowed tiles see key ranges of different lengths; between
    // one and two of them per SM pair they balance better as twice as many
    // 128-row tiles on the one-SM kernel (2K calls with 128 pair tiles:
    // causal 51.2 against 57.4 us, window 512 43.0 against 49.2).
    if (path == SDPA_PATH_TC && tc2_preferred_pair(pl.pair) && pl.rows >= kTc2RowThreshold) {
      const long long pair_tiles = (long long)pb.B * pb.Hkv * ((pl.rows + 255) / 256);
      const bool uneven = pb.causal || pb.window > 0;
      if (!(uneven && 2 * pair_tiles > num_sms && pair_tiles < num_sms)) path = SDPA_PATH_TC2;
    }
    // head dims <= 80 (where P has TMEM columns of its own): two 128-row
    // tiles per CTA, when the 256-row tiles alone occupy at least half of the
    // SMs (fewer would rather take the one-tile kernel's twice as many CTAs)
    // and no window trims the tiles' key ranges differently (the pair walks
    // the union of both ranges)
    if (path == SDPA_PATH_TC && tc_dual_preferred_pair(pl.pair) && pb.window == 0 &&
        pl.rows >= kTc2RowThreshold &&
        (long long)pb.B * pb.Hkv * ((pl.rows + 255) / 256) * 2 >= num_sms)
      path = SDPA_PATH_TC_DUAL;
  }
  const bool pair_path = path == SDPA_PATH_TC2 || path == SDPA_PATH_TC2_LOOP;
  if (pair_path && !tc2_supports_pair(pl.pair)) {
    // the smallest two-CTA instance that covers the head dims (zero filled)
    for (int i = pl.pair + 1; i < kNumDimPairs; ++i)
      if (tc2_supports_pair(i) && kDimPairs[i].dqk >= pb.Dqk && kDimPairs[i].dv >= pb.Dv) {
        pl.pair = i;
        break;
      }
  }
  if (pair_path && !tc2_supports_pair(pl.pair))
    return fail(SDPA_ERR_UNSUPPORTED,
                "the two-CTA path is built for head dims 256/256, 192/128 and 128/128 (got %d/%d)",
                pb.Dqk, pb.Dv);
  if ((path == SDPA_PATH_TC_DUAL || path == SDPA_PATH_TC_KSPLIT) &&
      !tc_dual_supports_pair(pl.pair))
    return fail(SDPA_ERR_UNSUPPORTED,
                "the two-tile paths are built for head dims up to 128 (got %d/%d)", pb.Dqk, pb.Dv);
  pl.path = path;
  if (path == SDPA_PATH_TC_DUAL) {
    pl.wr = 0; pl.wk = 0;
    pl.row_tile = 2 * kTcRows;
    pl.key_block = tc_pp_key_block(pl.pair, false);
  } else if (path == SDPA_PATH_TC_KSPLIT) {
    pl.wr = 0; pl.wk = 0;
    pl.row_tile = kTcRows;
    pl.key_block = tc_pp_key_block(pl.pair, true);
  } else if (path == SDPA_PATH_WIDE) {
    // one 16-row group (four warps) for decode-sized problems, two otherwise
    pl.wr = pl.rows <= 16 ? 1 : 2;
    pl.wk = 0;
    pl.row_tile = 16 * pl.wr;
    pl.key_block = kWideBN;
  } else if (pair_path) {
    pl.wr = 0; pl.wk = 0;
    pl.row_tile = 2 * kTcRows;
    // head dim 512: 64-key blocks in 256-column halves (grid.y)
    pl.key_block = wide ? 64 : 128;
    if (wide) pl.col_halves = (pb.Dv + kTc2WideHalf - 1) / kTc2WideHalf;
  } else if (path == SDPA_PATH_TC) {
    pl.wr = 0; pl.wk = 0;
    pl.row_tile = kTcRows;
    pl.key_block = tc_key_block(kDimPairs[pl.pair].dqk, kDimPairs[pl.pair].dv);
    if (wide) pl.col_halves = (pb.Dv + kTcWideHalf - 1) / kTcWideHalf;
  } else {
    if (pl.rows <= 16) {
      // one 16-row group: 16 keys per warp of every key block
      pl.wr = 1;
      pl.wk = splitkv_bn(kDimPairs[pl.pair].dqk, kDimPairs[pl.pair].dv) / 16;
      if (pl.wk > 8) pl.wk = 8;
    } else if (pl.rows <= 32) {
      pl.wr = 2; pl.wk = 2;
    } else {
      pl.wr = 4; pl.wk = 1;
    }
    pl.row_tile = 16 * pl.wr;
    pl.key_block = splitkv_bn(kDimPairs[pl.pair].dqk, kDimPairs[pl.pair].dv);
  }
  pl.row_tiles = (pl.rows + pl.row_tile - 1) / pl.row_tile;
  // keys visible to at least one row: [kbeg, kend)
  const int off = pb.q_offset;
  const int kbeg = pb.window > 0 ? std::max(0, off - pb.window + 1) : 0;
  const int kend = pb.causal ? (int)std::min<long long>(pb.S, (long long)off + pb.L) : pb.S;
  const int bn = pl.key_block;
  pl.split_base = (kbeg / bn) * bn;
  const int nkb = std::max(1, (kend + bn - 1) / bn - kbeg / bn);
  // CTAs per split: one per row tile, two per pair tile, two per row tile
  // (one per column half) for the tcgen05 kernel at head dims above 256
  const long long per_tile = pair_path ? 2 : 1;
  const bool tc_wide = path == SDPA_PATH_TC && wide;
  const long long base = (long long)pb.B * pb.Hkv * pl.row_tiles * per_tile * pl.col_halves;
  // resident CTAs per SM (the split-KV kernel runs two where they fit)
  const long long slots =
      (long long)num_sms * (path == SDPA_PATH_SPLITKV
                                ? splitkv_ctas_per_sm(kDimPairs[pl.pair].dqk,
                                                      kDimPairs[pl.pair].dv, pl.wr)
                                : 1);
  int splits;
  if (path == SDPA_PATH_TC2_LOOP || (path == SDPA_PATH_TC2 && wide)) {
    // the looping form, and the pair kernel at head dims above 256, write
    // finished rows only
    if (force_splits > 1)
      return fail(SDPA_ERR_UNSUPPORTED, "this pair path does not split the keys");
    splits = 1;
  } else if (force_splits > 0) {
    splits = std::min(force_splits, nkb);
  } else if (base >= slots || (path == SDPA_PATH_SPLITKV ? nkb * bn <= kNoSplitBlocks * 64
                                : tc_wide              ? nkb * bn <= kNoSplitBlocks * 128
                                                       : nkb <= kNoSplitBlocks)) {
    splits = 1;
  } else {
    // the wide kernel's 32-key blocks are small and its partials wide
    // (Dv up to 512 floats per row and split): give each split more keys.
    // The split-KV kernel's splits cover at least 128 keys whatever its block.
    const int min_blocks = path == SDPA_PATH_WIDE || tc_wide ? kMinBlocksPerSplitWide
                           : path == SDPA_PATH_SPLITKV      ? std::max(1, 128 / bn)
                                                            : kMinBlocksPerSplit;
    splits = (int)std::max(1LL, slots / base);
    splits = std::min(splits, std::max(1, nkb / min_blocks));
    // The combine merges the splits of a row 32 at a time, one round trip
    // to L2 per round: a count just above a multiple of 32 pays a whole
    // extra round for a few splits.  It is rounded down to that multiple
    // when this gives up at most a seventh of the splits (decode with 4 KV
    // heads: 37 -> 32 splits, 14.8 -> 12.6 us at S=16K back to back).
    if (splits > kCombineRound) {
      const int whole = splits / kCombineRound * kCombineRound;
      if ((splits - whole) * 7 <= splits) splits = whole;
    }
  }
  splits = std::min(splits, kMaxSplits);
  const int bps = (nkb + splits - 1) / splits;
  if (force_splits == 0) splits = (nkb + bps - 1) / bps;
  pl.splits = splits;
  pl.keys_per_split = bps * bn;
  pl.ctas = (base / per_tile) * splits;  // all CTAs: grid.x * col_halves
  // Windowed or short unsplit tiles on the pair kernel, more of them than SM
  // pairs: loop over tiles.  A tile visits at most the window's blocks plus
  // its own 256 rows' worth (or all of them without a window).
  if (force_path == SDPA_PATH_AUTO && path == SDPA_PATH_TC2 && !wide && splits == 1 &&
      pl.ctas > num_sms / 2) {
    const int tile_blocks =
        pb.window > 0 ? std::min(nkb, (pb.window + pl.row_tile + bn - 1) / bn + 1) : nkb;
    if (tile_blocks <= kLoopMaxTileBlocks && (pb.window > 0 || !pb.causal))
      path = pl.path = SDPA_PATH_TC2_LOOP;
  }
  if (path == SDPA_PATH_TC2_LOOP)
    pl.loop_pairs = (int)std::min<long long>(pl.ctas, std::max(1, num_sms / 2));
  if (pl.ctas > 0x7fffffffLL)
    return fail(SDPA_ERR_UNSUPPORTED, "problem needs %lld CTAs, above the grid limit", pl.ctas);
  pl.launches = splits > 1 ? 2 : 1;
  if (splits > 1) {
    const size_t rows_total = (size_t)pb.B * pb.Hq * pb.L;
    pl.ws_o_bytes = align256(rows_total * pb.Dv * sizeof(float) * splits);
    pl.ws_lse_bytes = align256(rows_total * sizeof(float) * splits);
  }
  pl.ws_bytes = pl.ws_o_bytes + pl.ws_lse_bytes;
  *out = pl;
  return SDPA_OK;
}

void fill_info(const Plan &pl, sdpa_plan_info *info) {
  info->path = pl.path;
  info->splits = pl.splits;
  info->rows = pl.rows;
  info->row_tile = pl.row_tile;
  info->row_tiles = pl.row_tiles;
  info->key_block = pl.key_block;
  info->keys_per_split = pl.keys_per_split;
  info->ctas = (int)pl.ctas;
  info->launches = pl.launches;
  info->dqk_pad = kDimPairs[pl.pair].dqk;
  info->dv_pad = kDimPairs[pl.pair].dv;
  info->workspace_bytes = pl.ws_bytes;
}

// ---------------------------------------------------------------------------
// device state
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
unsigned int *g_wd_ptr[kMaxDevices];
unsigned long long g_wd_ctx[kMaxDevices];  // context id the address belongs to
int g_num_sms[kMaxDevices];

// cuCtxGetCurrent and cuCtxGetId from the driver (no libcuda link).
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxFns &ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return f;
}

sdpa_status device_state(int *dev_out, int *sms_out, unsigned int **wd_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return fail(SDPA_ERR_CUDA, "no usable CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SDPA_ERR_CUDA, "device index %d too large", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  // A device address looked up in one context is stale once that context is
  // gone (cudaDeviceReset, say): the cache is keyed on the current context's
  // id, which the driver never reuses within a process.
  unsigned long long ctx = 0;
  if (g_wd_ptr[dev] && current_context_id(&ctx) == SDPA_OK && ctx == g_wd_ctx[dev]) {
    *dev_out = dev;
    *sms_out = g_num_sms[dev];
    *wd_out = g_wd_ptr[dev];
    return SDPA_OK;
  }
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess)
    return fail(SDPA_ERR_CUDA, "cudaGetDeviceProperties: %s", cudaGetErrorString(e));
  if (prop.major != 10 || prop.minor != 0)
    return fail(SDPA_ERR_UNSUPPORTED,
                "libsdpa is built for sm_100a (B200); device %d is sm_%d%d", dev, prop.major,
                prop.minor);
  void *ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_sdpa_watchdog_word);
  if (e != cudaSuccess)
    return fail(SDPA_ERR_CUDA, "cudaGetSymbolAddress(watchdog): %s", cudaGetErrorString(e));
  // the lookup made the device's context current
  if (current_context_id(&ctx) != SDPA_OK) ctx = 0;
  g_num_sms[dev] = prop.multiProcessorCount;
  g_wd_ptr[dev] = static_cast<unsigned int *>(ptr);
  g_wd_ctx[dev] = ctx;
  *dev_out = dev;
  *sms_out = g_num_sms[dev];
  *wd_out = g_wd_ptr[dev];
  return SDPA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// ---------------------------------------------------------------------------
// the call
// ---------------------------------------------------------------------------
sdpa_status forward_call(const Problem &pb, const void *q, const void *k, const void *v,
                         void *out, int force_path, int force_splits, void *ws, size_t ws_bytes,
                         bool own_ws, cudaStream_t stream, const float *sinks, float *lse_out) {
  sdpa_status st = validate_shape(pb);
  if (st != SDPA_OK) return st;
  st = validate_pointers(pb, q, k, v, out);
  if (st != SDPA_OK) return st;
  int dev, sms;
  unsigned int *wd;
  st = device_state(&dev, &sms, &wd);
  if (st != SDPA_OK) return st;
  Plan pl;
  st = make_plan(pb, sms, force_path, force_splits, &pl);
  if (st != SDPA_OK) return st;

  bool allocated = false;
  if (pl.ws_bytes > 0) {
    if (own_ws) {
      cudaError_t e = g_test_hooks.fail_alloc ? cudaErrorMemoryAllocation
                                              : cudaMallocAsync(&ws, pl.ws_bytes, stream);
      if (e != cudaSuccess)
        return fail(SDPA_ERR_CUDA, "cudaMallocAsync(%zu bytes) for the split workspace: %s%s",
                    pl.ws_bytes, cudaGetErrorString(e),
                    g_test_hooks.fail_alloc ? " (injected by SDPA_TEST_FAIL_ALLOC)" : "");
      allocated = true;
    } else {
      if (ws == nullptr || ws_bytes < pl.ws_bytes)
        return fail(SDPA_ERR_RESOURCES, "workspace of %zu bytes needed, %zu given", pl.ws_bytes,
                    ws == nullptr ? (size_t)0 : ws_bytes);
      if (!aligned16(ws)) return fail(SDPA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    }
  }
  Launch ln;
  ln.pb = pb;
  ln.plan = pl;
  ln.q = q; ln.k = k; ln.v = v; ln.out = out;
  ln.part_o = static_cast<float *>(ws);
  ln.part_lse = ws ? reinterpret_cast<float *>(static_cast<char *>(ws) + pl.ws_o_bytes) : nullptr;
  ln.lse_out = lse_out;
  ln.sinks = sinks;
  ln.wd_word = wd;
  ln.wd_limit_ns = wait_limit();
  ln.stream = stream;

  std::string err;
  ln.ev_start = t_ev_start;
  ln.ev_stop = t_ev_stop;
  cudaEvent_t ev_call = t_ev_call;
  t_ev_start = t_ev_stop = t_ev_call = nullptr;
  st = pl.path == SDPA_PATH_TC2 || pl.path == SDPA_PATH_TC2_LOOP ? launch_tc2(ln, &err)
       : pl.path == SDPA_PATH_TC      ? launch_tc(ln, &err)
       : pl.path == SDPA_PATH_TC_DUAL || pl.path == SDPA_PATH_TC_KSPLIT ? launch_tc_pp(ln, &err)
       : pl.path == SDPA_PATH_WIDE    ? launch_wide(ln, &err)
                                      : launch_splitkv(ln, &err);
  if (st == SDPA_OK && pl.splits > 1) st = launch_combine(ln, &err);
  if (st == SDPA_OK && ev_call) record_event(ev_call, stream);
  if (allocated) {
    cudaError_t e = cudaFreeAsync(ws, stream);
    if (st == SDPA_OK && e != cudaSuccess) {
      err = std::string("cudaFreeAsync: ") + cudaGetErrorString(e);
      st = SDPA_ERR_CUDA;
    }
  }
  if (st != SDPA_OK) return fail_str(st, err);
  return SDPA_OK;
}

sdpa_status current_context_id(unsigned long long *id) {
  const CtxFns &f = ctx_fns();
  CUcontext ctx = nullptr;
  if (!f.get_current || !f.get_id || f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return SDPA_ERR_CUDA;
  return f.get_id(ctx, id) == CUDA_SUCCESS ? SDPA_OK : SDPA_ERR_CUDA;
}

sdpa_status validate_call(const Problem &pb, const void *q, const void *k, const void *v,
                          const void *out) {
  sdpa_status st = validate_shape(pb);
  if (st != SDPA_OK) return st;
  return validate_pointers(pb, q, k, v, out);
}

sdpa_status plan_call(const Problem &pb, int force_path, int force_splits, Plan *plan) {
  sdpa_status st = validate_shape(pb);
  if (st != SDPA_OK) return st;
  int dev, sms;
  unsigned int *wd;
  st = device_state(&dev, &sms, &wd);
  if (st != SDPA_OK) return st;
  return make_plan(pb, sms, force_path, force_splits, plan);
}

sdpa_status set_error(sdpa_status st, const std::string &msg) { return fail_str(st, msg); }

// ---------------------------------------------------------------------------
// shared helpers declared in launch.h
// ---------------------------------------------------------------------------
namespace {
// Recently encoded tensor maps of this host thread.  A descriptor depends only
// on its arguments (no device state), so an eager loop of calls on the same
// tensors reuses it instead of encoding it again; a few entries cover Q, K
// and V of the last calls.
struct TmaCacheEntry {
  bool used;
  int dt;  // CUtensorMapDataType
  int rank;
  const void *base;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  CUtensorMap map;
};
constexpr int kTmaCacheSize = 12;
thread_local TmaCacheEntry t_tma_cache[kTmaCacheSize];
thread_local int t_tma_next = 0;

bool tma_key_equal(const TmaCacheEntry &e, int dt, int rank, const void *base,
                   const uint64_t *dims, const uint64_t *strides, const uint32_t *box) {
  if (!e.used || e.dt != dt || e.rank != rank || e.base != base) return false;
  for (int i = 0; i < rank; ++i)
    if (e.dims[i] != dims[i] || e.box[i] != box[i]) return false;
  for (int i = 0; i < rank - 1; ++i)
    if (e.strides[i] != strides[i]) return false;
  return true;
}
}  // namespace

namespace {
bool encode_tma_typed(CUtensorMap *map, int dt, int rank, const void *base, const uint64_t *dims,
                      const uint64_t *strides_bytes, const uint32_t *box, std::string *err) {
  if (rank >= 2 && rank <= 3) {
    for (const TmaCacheEntry &e : t_tma_cache)
      if (tma_key_equal(e, dt, rank, base, dims, strides_bytes, box)) {
        *map = e.map;
        return true;
      }
  }
  auto fn = encode_fn();
  if (!fn) {
    *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estr[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gstr[i] = strides_bytes[i];
  CUresult r = fn(map, (CUtensorMapDataType)dt, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstr, bdim, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d, rank %d)", (int)r,
             rank);
    *err = buf;
    return false;
  }
  if (rank >= 2 && rank <= 3) {
    TmaCacheEntry &e = t_tma_cache[t_tma_next];
    t_tma_next = (t_tma_next + 1) % kTmaCacheSize;
    e.used = true;
    e.dt = dt;
    e.rank = rank;
    e.base = base;
    for (int i = 0; i < rank; ++i) {
      e.dims[i] = dims[i];
      e.box[i] = box[i];
    }
    for (int i = 0; i < rank - 1; ++i) e.strides[i] = strides_bytes[i];
    e.map = *map;
  }
  return true;
}
}  // namespace

bool encode_tma(CUtensorMap *map, sdpa_dtype dt, int rank, const void *base,
                const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                std::string *err) {
  return encode_tma_typed(map,
                          dt == SDPA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                          rank, base, dims, strides_bytes, box, err);
}

bool encode_tma_f32(CUtensorMap *map, int rank, const void *base, const uint64_t *dims,
                    const uint64_t *strides_bytes, const uint32_t *box, std::string *err) {
  return encode_tma_typed(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank, base, dims, strides_bytes,
                          box, err);
}

bool encode_out_maps(const Launch &ln, CUtensorMap *to, CUtensorMap *tp, std::string *err) {
  const Problem &pb = ln.pb;
  const Plan &pl = ln.plan;
  const uint64_t slabs = (uint64_t)pb.B * pb.Hkv;
  memset(to, 0, sizeof(*to));
  memset(tp, 0, sizeof(*tp));
  if (pl.splits == 1) {
    const uint64_t dims[3] = {(uint64_t)pb.Dv, (uint64_t)pl.rows, slabs};
    const uint64_t strides[2] = {(uint64_t)pb.Dv * 2, (uint64_t)pl.rows * pb.Dv * 2};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tma(to, pb.dtype, 3, ln.out, dims, strides, box, err);
  }
  const uint64_t dims[3] = {(uint64_t)pb.Dv, (uint64_t)pl.rows, slabs * pl.splits};
  const uint64_t strides[2] = {(uint64_t)pb.Dv * 4, (uint64_t)pl.rows * pb.Dv * 4};
  const uint32_t box[3] = {32, 128, 1};
  return encode_tma_f32(tp, 3, ln.part_o, dims, strides, box, err);
}

sdpa_status prepare_kernel(const void *func, int threads, size_t smem, const char *name,
                           std::string *err) {
  // (device, function) pairs already checked
  static std::mutex mu;
  static const void *done_fn[512];
  static int done_dev[512];
  static int ndone = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < ndone; ++i)
      if (done_fn[i] == func && done_dev[i] == dev) return SDPA_OK;
  }
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, func);
  if (e != cudaSuccess) {
    *err = std::string(name) + ": cudaFuncGetAttributes: " + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  int max_optin = 0;
  cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (g_test_hooks.smem_limit >= 0 && g_test_hooks.smem_limit < max_optin)
    max_optin = (int)g_test_hooks.smem_limit;
  char buf[256];
  if (attr.maxThreadsPerBlock < threads) {
    snprintf(buf, sizeof(buf), "%s: compiled kernel allows %d threads per block, launch needs %d",
             name, attr.maxThreadsPerBlock, threads);
    *err = buf;
    return SDPA_ERR_RESOURCES;
  }
  if ((size_t)attr.sharedSizeBytes + smem > (size_t)max_optin) {
    snprintf(buf, sizeof(buf), "%s: needs %zu bytes of shared memory, device allows %d", name,
             (size_t)attr.sharedSizeBytes + smem, max_optin);
    *err = buf;
    return SDPA_ERR_RESOURCES;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    *err = std::string(name) + ": cudaFuncSetAttribute: " + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (ndone < 512) {
    done_fn[ndone] = func;
    done_dev[ndone] = dev;
    ++ndone;
  }
  return SDPA_OK;
}

// Watchdog self-test kernel: waits on an mbarrier that nothing ever arrives
// on; the bounded wait must expire and record its code.
__global__ void watchdog_selftest_kernel(Watchdog wd, int *result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0, wd, kWdTmaFull);
  if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

// Self-test of the FMA-pipe exp2: evaluates exp2_poly2 and exp2f on n
// points spread evenly over [lo, hi] and writes both results.
__global__ void exp2_selftest_kernel(float lo, float hi, int n, float *poly, float *ref) {
  for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n;
       i += 2 * gridDim.x * blockDim.x) {
    const float step = n > 1 ? (hi - lo) / (float)(n - 1) : 0.f;
    const float x0 = lo + step * (float)i;
    const float x1 = i + 1 < n ? lo + step * (float)(i + 1) : x0;
    const float2 y = exp2_poly2(make_float2(x0, x1));
    poly[i] = y.x;
    ref[i] = exp2f(x0);
    if (i + 1 < n) {
      poly[i + 1] = y.y;
      ref[i + 1] = exp2f(x1);
    }
  }
}

}  // namespace sdpa

// ===========================================================================
// C ABI
// ===========================================================================
using namespace sdpa;

static Problem make_problem(int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv, float scale,
                            int causal, int window, sdpa_dtype dtype) {
  Problem p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.S = S; p.Dqk = Dqk; p.Dv = Dv;
  p.scale = scale; p.causal = causal; p.window = window; p.dtype = dtype;
  p.q_offset = S - L;
  p.has_q_offset = 0;
  return p;
}

extern "C" {

sdpa_status sdpa_forward(const void *q, const void *k, const void *v, void *out, int B, int Hq,
                         int Hkv, int L, int S, int Dqk, int Dv, float scale, int causal,
                         int window_size, sdpa_dtype dtype, sdpa_stream_t stream) {
  t_last_error.clear();
  return forward_call(make_problem(B, Hq, Hkv, L, S, Dqk, Dv, scale, causal, window_size, dtype), q, k, v,
             out, SDPA_PATH_AUTO, 0, nullptr, 0, true, (cudaStream_t)stream);
}

size_t sdpa_workspace_bytes(int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv, int causal,
                            int window_size, sdpa_dtype dtype) {
  t_last_error.clear();
  Problem pb = make_problem(B, Hq, Hkv, L, S, Dqk, Dv, 1.0f, causal, window_size, dtype);
  if (validate_shape(pb) != SDPA_OK) return 0;
  int dev, sms;
  unsigned int *wd;
  if (device_state(&dev, &sms, &wd) != SDPA_OK) return 0;
  Plan pl;
  if (make_plan(pb, sms, SDPA_PATH_AUTO, 0, &pl) != SDPA_OK) return 0;
  return pl.ws_bytes;
}

sdpa_status sdpa_forward_ws(const void *q, const void *k, const void *v, void *out, int B,
                            int Hq, int Hkv, int L, int S, int Dqk, int Dv, float scale,
                            int causal, int window_size, sdpa_dtype dtype, void *workspace,
                            size_t workspace_bytes, sdpa_stream_t stream) {
  t_last_error.clear();
  return forward_call(make_problem(B, Hq, Hkv, L, S, Dqk, Dv, scale, causal, window_size, dtype), q, k, v,
             out, SDPA_PATH_AUTO, 0, workspace, workspace_bytes, false, (cudaStream_t)stream);
}

sdpa_status sdpa_plan(int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv, int causal,
                      int window_size, sdpa_dtype dtype, int num_sms, int force_path,
                      int force_splits, sdpa_plan_info *info) {
  t_last_error.clear();
  if (!info) return fail(SDPA_ERR_INVALID_ARG, "info must be non-NULL");
  Problem pb = make_problem(B, Hq, Hkv, L, S, Dqk, Dv, 1.0f, causal, window_size, dtype);
  sdpa_status st = validate_shape(pb);
  if (st != SDPA_OK) return st;
  Plan pl;
  st = make_plan(pb, num_sms, force_path, force_splits, &pl);
  if (st != SDPA_OK) return st;
  fill_info(pl, info);
  return SDPA_OK;
}

sdpa_status sdpa_forward_planned(const void *q, const void *k, const void *v, void *out, int B,
                                 int Hq, int Hkv, int L, int S, int Dqk, int Dv, float scale,
                                 int causal, int window_size, sdpa_dtype dtype, int force_path,
                                 int force_splits, void *workspace, size_t workspace_bytes,
                                 sdpa_stream_t stream) {
  t_last_error.clear();
  return forward_call(make_problem(B, Hq, Hkv, L, S, Dqk, Dv, scale, causal, window_size, dtype), q, k, v,
             out, force_path, force_splits, workspace, workspace_bytes, false,
             (cudaStream_t)stream);
}

sdpa_status sdpa_forward_ex(const void *q, const void *k, const void *v, void *out, int B, int Hq,
                            int Hkv, int L, int S, int Dqk, int Dv, float scale, int causal,
                            int window_size, sdpa_dtype dtype, const sdpa_options *opt,
                            void *workspace, size_t workspace_bytes, sdpa_stream_t stream) {
  t_last_error.clear();
  Problem pb = make_problem(B, Hq, Hkv, L, S, Dqk, Dv, scale, causal, window_size, dtype);
  int force_path = 0, force_splits = 0;
  const float *sinks = nullptr;
  float *lse = nullptr;
  if (opt != nullptr) {
    if (opt->has_q_offset) {
      pb.has_q_offset = 1;
      pb.q_offset = opt->q_offset;
    }
    sinks = opt->sinks;
    lse = opt->lse;
    force_path = opt->force_path;
    force_splits = opt->force_splits;
    if ((sinks && (reinterpret_cast<uintptr_t>(sinks) & 3u)) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
      return fail(SDPA_ERR_INVALID_ARG, "sinks and lse must be 4-byte aligned");
  }
  const bool own = workspace == nullptr && workspace_bytes == 0;
  return forward_call(pb, q, k, v, out, force_path, force_splits, workspace, workspace_bytes,
                      own, (cudaStream_t)stream, sinks, lse);
}

sdpa_status sdpa_device_status(int clear) {
  t_last_error.clear();
  int dev, sms;
  unsigned int *wd;
  sdpa_status st = device_state(&dev, &sms, &wd);
  if (st != SDPA_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess)
    return fail(SDPA_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpy(&word, wd, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(SDPA_ERR_CUDA, "reading the watchdog word: %s", cudaGetErrorString(e));
  if (clear && word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpy(wd, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail(SDPA_ERR_CUDA, "clearing the watchdog word: %s", cudaGetErrorString(e));
  }
  if (word != 0)
    return fail(SDPA_ERR_TIMEOUT, "a kernel gave up on a bounded wait (watchdog code %u)", word);
  return SDPA_OK;
}

void sdpa_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

void sdpa_time_next_main_kernel(void *start_event, void *stop_event) {
  sdpa_time_next_call(start_event, stop_event, nullptr);
}

void sdpa_time_next_call(void *start_event, void *stop_event, void *call_event) {
  t_ev_start = static_cast<cudaEvent_t>(start_event);
  t_ev_stop = static_cast<cudaEvent_t>(stop_event);
  t_ev_call = static_cast<cudaEvent_t>(call_event);
}

sdpa_status sdpa_watchdog_selftest(uint64_t limit_ns, int *waited_out) {
  t_last_error.clear();
  int dev, sms;
  unsigned int *wd;
  sdpa_status st = device_state(&dev, &sms, &wd);
  if (st != SDPA_OK) return st;
  int *d_res = nullptr;
  cudaError_t e = cudaMalloc(&d_res, sizeof(int));
  if (e != cudaSuccess) return fail(SDPA_ERR_CUDA, "cudaMalloc: %s", cudaGetErrorString(e));
  Watchdog w;
  w.word = wd;
  w.limit_ns = limit_ns ? limit_ns : 100000000ull;
  watchdog_selftest_kernel<<<1, 32>>>(w, d_res);
  e = cudaGetLastError();
  int res = -1;
  if (e == cudaSuccess) e = cudaMemcpy(&res, d_res, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d_res);
  if (e != cudaSuccess) return fail(SDPA_ERR_CUDA, "selftest: %s", cudaGetErrorString(e));
  if (waited_out) *waited_out = res;
  return SDPA_OK;
}

sdpa_status sdpa_exp2_selftest(float lo, float hi, int n, float *poly, float *ref) {
  t_last_error.clear();
  if (n < 1 || !poly || !ref || !(lo <= hi))
    return fail(SDPA_ERR_INVALID_ARG, "exp2 self-test needs n >= 1, lo <= hi and two buffers");
  int dev, sms;
  unsigned int *wd;
  sdpa_status st = device_state(&dev, &sms, &wd);
  if (st != SDPA_OK) return st;
  exp2_selftest_kernel<<<(n + 511) / 512, 256>>>(lo, hi, n, poly, ref);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SDPA_ERR_CUDA, "exp2 self-test: %s", cudaGetErrorString(e));
  return SDPA_OK;
}

const char *sdpa_status_string(sdpa_status s) {
  switch (s) {
    case SDPA_OK: return "SDPA_OK";
    case SDPA_ERR_INVALID_ARG: return "SDPA_ERR_INVALID_ARG";
    case SDPA_ERR_UNSUPPORTED: return "SDPA_ERR_UNSUPPORTED";
    case SDPA_ERR_RESOURCES: return "SDPA_ERR_RESOURCES";
    case SDPA_ERR_CUDA: return "SDPA_ERR_CUDA";
    case SDPA_ERR_TIMEOUT: return "SDPA_ERR_TIMEOUT";
  }
  return "SDPA_ERR_UNKNOWN";
}

const char *sdpa_last_error_message(void) { return t_last_error.c_str(); }

int sdpa_version(void) { return 100; }

}  // extern "C"
