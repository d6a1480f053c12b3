// Host-side declarations shared by the C-ABI layer and the per-kernel launch
// units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

#include "../../include/sdpa.h"

namespace sdpa {

// Head-dim pairs a kernel instance is compiled for.  A problem runs on the
// cheapest pair that covers it; TMA zero-fills the columns in between.
struct DimPair {
  int dqk, dv;
};
constexpr DimPair kDimPairs[] = {{64, 64},   {80, 80},   {128, 128}, {192, 128},
                                 {192, 192}, {256, 256}, {512, 512}};
constexpr int kNumDimPairs = sizeof(kDimPairs) / sizeof(kDimPairs[0]);
// The 512/512 pair is built only for the wide (column-split) kernel.
constexpr int kWidePair = 6;

// Key block of the wide kernel.
constexpr int kWideBN = 32;

// Key block of the split-KV kernel (keys per pipeline stage).
#ifndef SDPA_SK_BN
#define SDPA_SK_BN 64
#endif
constexpr int kSplitKvBN = SDPA_SK_BN;

// Split-KV shared memory: one Q tile of 16*wr rows plus a ring of K/V stages
// (64-column TMA boxes of 128 bytes per row).  With two CTAs per SM each gets
// half of the SM's 228 KB less the 1 KB the hardware reserves per CTA; the
// budgets keep 2 KB for barriers, alignment slack and static shared memory.
constexpr unsigned kSplitKvBudget1 = 232448u - 2048u;
constexpr unsigned kSplitKvBudget2 = 233472u / 2 - 1024u - 2048u;
constexpr unsigned splitkv_stage_bytes(int dqk, int dv, int bn = kSplitKvBN) {
  return (unsigned)(((dqk + 63) / 64 + (dv + 63) / 64) * bn * 128);
}
// Key block of one instance: kSplitKvBN where two stages of it fit next to a
// 64-row Q tile, else 64.
constexpr int splitkv_bn(int dqk, int dv) {
  return 2 * splitkv_stage_bytes(dqk, dv, kSplitKvBN) + ((dqk + 63) / 64) * 64 * 128 <= 232448u - 2048u
             ? kSplitKvBN
             : 64;
}
constexpr unsigned splitkv_q_bytes(int dqk, int wr) {
  return (unsigned)(((dqk + 63) / 64) * 16 * wr * 128);
}
// Stages that fit the budget next to Q, at most 4.
constexpr int splitkv_stages(int dqk, int dv, int wr, unsigned budget) {
  return (int)((budget - splitkv_q_bytes(dqk, wr)) /
               splitkv_stage_bytes(dqk, dv, splitkv_bn(dqk, dv))) > 4
             ? 4
             : (int)((budget - splitkv_q_bytes(dqk, wr)) /
                     splitkv_stage_bytes(dqk, dv, splitkv_bn(dqk, dv)));
}
// CTAs of one instance resident per SM.  The 64-row layout (four warps on
// their own rows, each doing four times the math per key of a slice warp)
// runs two per SM where double buffering fits half the shared memory and the
// registers fit half the file: the second CTA's warps hide the first's
// latencies (verify L=12..16 at S=32K: 44.4 -> 40.3 us).  The 16- and 32-row
// layouts keep one per SM: twice the splits cost more in the combine than
// the pass gains (decode sweep 3234-3245 against 3406-3408 GB/s with the
// warp-per-row combine).
constexpr int splitkv_ctas_per_sm(int dqk, int dv, int wr) {
  return wr == 4 && dqk + dv <= 256 && splitkv_stages(dqk, dv, wr, kSplitKvBudget2) >= 2 ? 2 : 1;
}

// Key block of the tcgen05 kernel: 128 keys while two 128-key score buffers
// plus O fit TMEM and the slots fit shared memory; 64 for head dims > 128;
// 32 for head dims above 256 (a 128 KB Q tile leaves three 32 KB slots).
constexpr int tc_key_block(int dqk, int dv) {
  return (dqk > 256 || dv > 256) ? 32 : (dqk > 128 || dv > 128) ? 64 : 128;
}

// Output columns per CTA of the tcgen05 kernel for head dims above 256: O of
// 128 rows at Dv = 512 would take all of TMEM, so each CTA owns one half of V
// and O (grid.y = 2) and computes the full scores.
constexpr int kTcWideHalf = 256;

// Rows of one tcgen05 tile.
constexpr int kTcRows = 128;

struct Problem {
  int B, Hq, Hkv, L, S, Dqk, Dv;
  float scale;
  int causal, window;
  sdpa_dtype dtype;
  int q_offset;      // key position of query row 0 (S - L unless given)
  int has_q_offset;  // 1 when the caller gave q_offset explicitly
};

struct Plan {
  int path;            // an sdpa_path value other than SDPA_PATH_AUTO
  int pair;            // index into kDimPairs
  int rows;            // g * L
  int wr, wk;          // split-KV warp layout (rows x key slices); wide: row groups
  int row_tile;
  int row_tiles;
  int key_block;
  int split_base;      // first key of split 0 (block aligned)
  int keys_per_split;
  int splits;
  long long ctas;
  int launches;
  int col_halves;      // tcgen05 kernel at head dims above 256: 2 (grid.y), else 1
  int loop_pairs;      // SDPA_PATH_TC2_LOOP: CTA pairs launched (each walks several tiles)
  size_t ws_o_bytes, ws_lse_bytes, ws_bytes;
};

// Everything a kernel launch needs.
struct Launch {
  Problem pb;
  Plan plan;
  const void *q, *k, *v;
  void *out;
  float *part_o, *part_lse;
  float *lse_out;          // optional final LSE [B*Hq*L] (nullptr = not wanted)
  const float *sinks;      // optional [Hq] sink logits
  unsigned int *wd_word;
  uint64_t wd_limit_ns;
  cudaStream_t stream;
  cudaEvent_t ev_start, ev_stop;  // optional, recorded around the main kernel launch
};

// Validate, plan for the current device and enqueue one call (the body of
// every sdpa_forward* entry point).  own_ws: take the split workspace from
// the stream-ordered pool; otherwise use (ws, ws_bytes).
sdpa_status forward_call(const Problem &pb, const void *q, const void *k, const void *v,
                         void *out, int force_path, int force_splits, void *ws, size_t ws_bytes,
                         bool own_ws, cudaStream_t stream, const float *sinks = nullptr,
                         float *lse_out = nullptr);

// Host-side argument checks of every entry point (shape, then pointers); no
// CUDA call.
sdpa_status validate_call(const Problem &pb, const void *q, const void *k, const void *v,
                          const void *out);

// Id of the calling thread's current CUDA context (unique within the process,
// never reused), or SDPA_ERR_CUDA when no context is current.
sdpa_status current_context_id(unsigned long long *id);

// Validate and plan for the current device without enqueuing anything.
sdpa_status plan_call(const Problem &pb, int force_path, int force_splits, Plan *plan);

// Record `msg` as this thread's last error and return `st`.
sdpa_status set_error(sdpa_status st, const std::string &msg);

// Encode a tiled TMA descriptor (128-byte swizzle, zero fill out of bounds).
// rank 2 or 3; dims/strides in elements/bytes as cuTensorMapEncodeTiled wants.
bool encode_tma(CUtensorMap *map, sdpa_dtype dt, int rank, const void *base,
                const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                std::string *err);

// The same for an fp32 tensor (split partials).
bool encode_tma_f32(CUtensorMap *map, int rank, const void *base, const uint64_t *dims,
                    const uint64_t *strides_bytes, const uint32_t *box, std::string *err);

// Tensor maps of a call's output for the TMA-store epilogues, in boxes of 128
// rows: `to` views out as [B*Hkv][R][Dv] (16-bit, 64-column boxes) when the
// call is not split, `tp` views the fp32 partials as [splits*B*Hkv][R][Dv]
// (32-column boxes) when it is; a packed-row slab is contiguous in both, so a
// box never spills into the next slab.  The unused map is zeroed.
bool encode_out_maps(const Launch &ln, CUtensorMap *to, CUtensorMap *tp, std::string *err);

// Per-path launchers (return SDPA_OK or an error with *err set).
sdpa_status launch_splitkv(const Launch &ln, std::string *err);
sdpa_status launch_tc(const Launch &ln, std::string *err);
sdpa_status launch_tc2(const Launch &ln, std::string *err);
sdpa_status launch_wide(const Launch &ln, std::string *err);
sdpa_status launch_tc_pp(const Launch &ln, std::string *err);

// Head-dim pairs the two-tile kernel is built for (index into kDimPairs).
constexpr bool tc_dual_supports_pair(int pair) { return pair <= 2; }
// ... and those the router sends to it by itself: at head dims 128 the
// one-tile kernel measured faster (P shares the scores' columns there)
constexpr bool tc_dual_preferred_pair(int pair) { return pair <= 1; }
// Key block of the two-tile kernel: 96 keys for row pairs at head dims 80
// (score, P and O columns of a tile then fit its 256 TMEM columns apart),
// 128 otherwise.
constexpr int tc_pp_key_block(int pair, bool key_split) { return (!key_split && pair == 1) ? 96 : 128; }

// Head-dim pairs the two-CTA kernel is built for (index into kDimPairs), and
// those the router sends to it by itself (where it measured faster than one
// SM per 128-row tile).
constexpr bool tc2_supports_pair(int pair) {
  return pair == 2 || pair == 3 || pair == 5 || pair == kWidePair;
}
// Output columns per launch column of the two-CTA kernel at head dim 512.
constexpr int kTc2WideHalf = 256;
constexpr bool tc2_preferred_pair(int pair) { return pair == 3 || pair == 5; }
sdpa_status launch_combine(const Launch &ln, std::string *err);

// Record a timing event on `stream`.  Inside stream capture a plain
// cudaEventRecord only orders work within the graph; an external record node
// is needed for the event to carry a timestamp when the graph is replayed.
inline void record_event(cudaEvent_t ev, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, stream);
}

// Checks that a kernel fits the device (threads, shared memory) before its
// first launch, and raises its dynamic shared-memory limit.  Cached per
// device and kernel.
sdpa_status prepare_kernel(const void *func, int threads, size_t smem, const char *name,
                           std::string *err);

}  // namespace sdpa
