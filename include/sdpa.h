/*
 * libsdpa: fused scaled-dot-product attention forward pass for NVIDIA B200
 * (sm_100a).
 *
 *   O = softmax(scale * Q K^T + mask) V
 *
 * computed tile by tile with an online (running max / running sum) softmax,
 * so the [L, S] score matrix never exists in memory.  The method and its
 * cases come from the pages on MLX's fused attention:
 *   - online-softmax flash attention with GQA and causal masking
 *     (mlx-rs issue #339, "Context");
 *   - causal masking with the queries aligned to the end of the keys, and a
 *     sliding window that skips whole key blocks below its left edge
 *     (mlx PR #3552, "Summary" and "Implementation": qL_off = kL - qL,
 *     kb_start / kb_lim, left-edge rule row - col >= W masked);
 *   - asymmetric head dims Dqk != Dv, e.g. 192/128 (mlx PR #3637);
 *   - head dims outside the usual fused sets: 72, 192, 256 (mlx-rs issue
 *     #339 finding 1; mlx PR #4185 "Kernel support"), and 512, where the
 *     pages' kernels stop (mlx PR #4185, "Kernel support");
 *   - decode and short "verify" queries processed as a split over the keys
 *     with a log-sum-exp merge, so the work stays parallel over S
 *     (mlx issue #3826, routing analysis and the 2-pass extension);
 *   - a call either runs a fused kernel or fails with a message naming the
 *     violated constraint; never a silent fallback or silent zeros
 *     (mlx PR #4185, "API" and "Kernel support": force_fused and the
 *     dispatch-time threadgroup check).
 *
 * Conventions for every entry point below
 * ---------------------------------------
 * Tensors are dense, row-major, in device memory, all of one 16-bit type:
 *   q   [B][Hq ][L][Dqk]     k [B][Hkv][S][Dqk]     v [B][Hkv][S][Dv]
 *   out [B][Hq ][L][Dv]
 * Query head hq reads KV head hq / (Hq / Hkv): each KV head serves Hq/Hkv
 * consecutive query heads.  Query row i sits at key position i + S - L.
 *   causal       row i sees keys j <= i + S - L.
 *   window_size  W > 0 (with causal): row i sees only keys with
 *                i + S - L - j < W (the last W positions, its own included).
 *                W = 0 means no window.  W >= S equals plain causal.
 * Accumulation and softmax are fp32; out is rounded to nearest even.
 *
 * Ownership: the caller owns q, k, v, out and any workspace.  Every pointer
 * must be 16-byte aligned; out must not overlap q, k or v.  The library keeps
 * no pointer after a call returns.
 *
 * Asynchrony: a call validates its arguments on the host, enqueues its
 * kernels on `stream` and returns; it never synchronises the stream.  Errors
 * found on the host are returned before anything is enqueued.  Launch errors
 * are returned as SDPA_ERR_CUDA.  Faults inside a kernel surface later, like
 * any CUDA error, and sdpa_device_status() reports a watchdog expiry.
 * Stream order holds as for plain launches.  The split-KV pass and the
 * combine are launched with programmatic stream serialization: their setup
 * (and, for the split pass, an L2 prefetch of its first inputs) may overlap
 * the previous kernel on the stream, but neither reads nor writes global
 * memory before that kernel has completed.  A kernel the caller launches
 * after a call with the same attribute must likewise wait
 * (griddepcontrol.wait / cudaGridDependencySynchronize) before it reads `out`.
 *
 * Thread safety: calls from several host threads are safe; the last error
 * message is kept per thread.
 */
#ifndef SDPA_H_
#define SDPA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SDPA_API __attribute__((visibility("default")))
#else
#define SDPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *sdpa_stream_t;

typedef enum { SDPA_BF16 = 0, SDPA_F16 = 1 } sdpa_dtype;

typedef enum {
  SDPA_OK = 0,
  SDPA_ERR_INVALID_ARG = 1, /* the arguments break a stated constraint        */
  SDPA_ERR_UNSUPPORTED = 2, /* valid attention, but no fused kernel covers it */
  SDPA_ERR_RESOURCES = 3,   /* workspace too small, or a kernel does not fit  */
  SDPA_ERR_CUDA = 4,        /* a CUDA runtime call failed                     */
  SDPA_ERR_TIMEOUT = 5      /* a kernel's bounded wait expired (device flag)  */
} sdpa_status;

/* Execution paths the router picks from (see sdpa_plan). */
typedef enum {
  SDPA_PATH_AUTO = 0,
  SDPA_PATH_SPLITKV = 1, /* split-KV pass over packed (head-in-group, query)
                            rows on warp-level tensor-core tiles, then the
                            log-sum-exp combine when split                   */
  SDPA_PATH_TC = 2,      /* 128-row tiles on tcgen05 with TMEM accumulators,
                            TMA-staged K/V, optional key splits + combine    */
  SDPA_PATH_TC2 = 3,     /* 256-row tiles on a pair of SMs (tcgen05
                            cta_group::2): each SM loads half of every K/V
                            block; head dims 256/256, 192/128 (routed) and
                            128/128 (on request)                             */
  SDPA_PATH_WIDE = 4,    /* head dims above 256 (up to 512): 16-row groups
                            whose four warps split the output columns, key
                            splits + combine as on SDPA_PATH_SPLITKV; the
                            only path for those head dims                    */
  SDPA_PATH_TC_DUAL = 5, /* head dims up to 128: two 128-row tiles per CTA
                            share each K/V block, their softmax phases
                            interleaved with each other's MMAs (tcgen05)     */
  SDPA_PATH_TC_KSPLIT = 6, /* head dims up to 128: one 128-row tile per CTA
                            whose two softmax groups take alternate key
                            blocks, merged in the epilogue (tcgen05)        */
  SDPA_PATH_TC2_LOOP = 7  /* the SDPA_PATH_TC2 kernel with at most one CTA
                            pair per two SMs, each walking several 256-row
                            tiles: the next tile's Q and first scores run
                            under the current tile's end.  Never splits the
                            keys; routed for windows and short key ranges  */
} sdpa_path;

/*
 * sdpa_forward: the whole forward pass.
 *   scale        multiplies Q K^T (commonly Dqk^-0.5); must be finite.
 *   causal       0 or 1.
 *   window_size  0 (none) or >= 1, only together with causal = 1.
 *   dtype        type of q, k, v and out.
 * When the chosen plan splits the keys, the call takes its fp32 workspace
 * stream-ordered from the device's default memory pool
 * (cudaMallocAsync/cudaFreeAsync on `stream`); use sdpa_forward_ws to pass
 * your own.
 * Errors:
 *   SDPA_ERR_INVALID_ARG  a NULL or unaligned pointer; B, Hq, Hkv, L, S < 1;
 *                         Hq not a multiple of Hkv; causal with L > S (no key
 *                         would be visible to the first rows); window_size <
 *                         0; a non-finite scale; out overlapping an input.
 *   SDPA_ERR_UNSUPPORTED  Dqk or Dv not a multiple of 8 or above 512 (for
 *                         example 576); an unknown dtype; window_size > 0
 *                         with causal = 0; sizes whose element offsets
 *                         exceed 2^31 rows of 2^31 bytes.
 *   SDPA_ERR_CUDA         no usable CUDA device, or a launch failed.
 */
SDPA_API sdpa_status sdpa_forward(const void *q, const void *k, const void *v, void *out,
                         int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                         float scale, int causal, int window_size,
                         sdpa_dtype dtype, sdpa_stream_t stream);

/*
 * Bytes of workspace sdpa_forward_ws needs for this problem on the current
 * device (0 when the plan does not split the keys).  Returns 0 and sets the
 * last error message when the arguments are invalid.
 */
SDPA_API size_t sdpa_workspace_bytes(int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                            int causal, int window_size, sdpa_dtype dtype);

/*
 * sdpa_forward_ws: as sdpa_forward, with caller-owned device workspace of
 * workspace_bytes >= sdpa_workspace_bytes(...) bytes (NULL allowed when that
 * is 0).  No allocation happens inside the call.  The workspace must not be
 * used by other work until the call's kernels have finished on `stream`.
 * Extra error: SDPA_ERR_RESOURCES when the workspace is too small.
 */
SDPA_API sdpa_status sdpa_forward_ws(const void *q, const void *k, const void *v, void *out,
                            int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                            float scale, int causal, int window_size,
                            sdpa_dtype dtype, void *workspace, size_t workspace_bytes,
                            sdpa_stream_t stream);

/*
 * sdpa_forward_noalloc: as sdpa_forward, for callers that cannot allocate
 * device memory.  (This entry point has no counterpart in the pages; it is
 * a service of this library.)
 *
 * Who needs it: code that must not call cudaMalloc or cudaMallocAsync, for
 * example a runtime whose device memory is owned by an allocator it cannot
 * reach at the point of the call, or a latency-critical loop where an
 * allocation could synchronise the device or grow a memory pool mid-run.
 * sdpa_forward allocates its split workspace and sdpa_forward_ws needs the
 * caller to provide one; this call does neither.
 *
 * How: when the router splits the keys, the fp32 partial outputs and
 * log-sum-exp values go to one fixed scratch array of 16 MiB that the library
 * keeps in each GPU's memory from load until process exit.  The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 * The caller still passes q, k, v and out.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  If the device's context is replaced later
 *     (cudaDeviceReset), the next call looks the address up again.
 *   - Problems whose split workspace (sdpa_workspace_bytes) exceeds 16 MiB
 *     are rejected with SDPA_ERR_RESOURCES and a message; use sdpa_forward or
 *     sdpa_forward_ws for them.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  Nothing in it needs clearing: each call writes every element
 *     it later reads.  Calls whose kernels overlap on the GPU (different
 *     streams, or several host threads) race on the array and may return
 *     wrong results; order them on one stream or use sdpa_forward_ws.
 * Other arguments, validation and errors as sdpa_forward.
 */
SDPA_API sdpa_status sdpa_forward_noalloc(const void *q, const void *k, const void *v, void *out,
                                          int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                                          float scale, int causal, int window_size,
                                          sdpa_dtype dtype, sdpa_stream_t stream);

/*
 * Options of sdpa_forward_ex (zero-initialise, then set what is needed).
 *   has_q_offset / q_offset  key position of query row 0.  Without it the
 *       queries end at the last key (q_offset = S - L).  With it a query block
 *       can sit anywhere: chunked prefill (queries [c0, c1) over keys [0, c1)
 *       with q_offset = c0), or keys held in a rotating window cache and
 *       addressed relative to the first held key (mlx PR #3552,
 *       "Implementation": K-relative coordinates).  Causal needs q_offset >= 0;
 *       with a window the last row must still see a held key.
 *   sinks  optional device array [Hq] of fp32 sink logits (natural-log units):
 *       one more logit per query head that joins the softmax normalisation
 *       with no value row (the `sinks` argument of mlx PR #4185 "API" and mlx
 *       PR #3552 "Public API"):  O = sum_j e^{s_j} V_j / (e^{sink} + sum_j e^{s_j}).
 *   lse    optional device array [B][Hq][L] of fp32, written with each row's
 *       natural-log log-sum-exp (sink included), e.g. for a later merge of
 *       results computed over disjoint key ranges.
 *   force_path / force_splits  as in sdpa_plan (0 = the router's choice).
 */
typedef struct {
  int has_q_offset;
  int q_offset;
  const float *sinks;
  float *lse;
  int force_path;
  int force_splits;
} sdpa_options;

/*
 * sdpa_forward_ex: sdpa_forward with sdpa_options (opt may be NULL).
 * workspace: as sdpa_forward_ws; when workspace is NULL and workspace_bytes
 * is 0 the call takes it stream-ordered from the pool like sdpa_forward.
 * Extra errors: SDPA_ERR_INVALID_ARG for a misaligned sinks/lse pointer or a
 * q_offset that leaves a row without keys.
 */
SDPA_API sdpa_status sdpa_forward_ex(const void *q, const void *k, const void *v, void *out,
                                     int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                                     float scale, int causal, int window_size, sdpa_dtype dtype,
                                     const sdpa_options *opt, void *workspace,
                                     size_t workspace_bytes, sdpa_stream_t stream);

/* What the router decides for one problem.  Host-only, no CUDA call. */
typedef struct {
  int path;          /* sdpa_path actually taken (never AUTO)               */
  int splits;        /* key splits per row tile (1 = no combine launch)     */
  int rows;          /* packed rows per (batch, KV head): (Hq/Hkv) * L      */
  int row_tile;      /* rows one CTA (one CTA pair on SDPA_PATH_TC2) owns   */
  int row_tiles;     /* row tiles per (batch, KV head)                      */
  int key_block;     /* keys per pipeline stage                             */
  int keys_per_split;/* keys one split covers (a multiple of key_block)     */
  int ctas;          /* CTAs of the main launch (CTA pairs on SDPA_PATH_TC2;
                        256-row tiles on SDPA_PATH_TC2_LOOP, whose pairs
                        walk them)                                          */
  int launches;      /* kernel launches one call makes (1 or 2)             */
  int dqk_pad;       /* head dims the kernel instance is built for          */
  int dv_pad;
  size_t workspace_bytes;
} sdpa_plan_info;

/*
 * sdpa_plan: the router on its own.  num_sms is the SM count to plan for
 * (148 on B200).  force_path / force_splits = 0 let the router choose;
 * otherwise they pin the path or the split count (test and bench use: every
 * choice gives the same result up to rounding).  Validates like sdpa_forward.
 */
SDPA_API sdpa_status sdpa_plan(int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                      int causal, int window_size, sdpa_dtype dtype, int num_sms,
                      int force_path, int force_splits, sdpa_plan_info *info);

/*
 * sdpa_forward_planned: sdpa_forward_ws with the router's path and split
 * count pinned as in sdpa_plan (0 = router's choice).  For tests of
 * path/split invariance and for the bench.
 */
SDPA_API sdpa_status sdpa_forward_planned(const void *q, const void *k, const void *v, void *out,
                                 int B, int Hq, int Hkv, int L, int S, int Dqk, int Dv,
                                 float scale, int causal, int window_size,
                                 sdpa_dtype dtype, int force_path, int force_splits,
                                 void *workspace, size_t workspace_bytes,
                                 sdpa_stream_t stream);

/*
 * Device watchdog.  Every wait inside the kernels (on an mbarrier or a
 * tensor-core completion) gives up after a bounded time, records a code in a
 * device word and lets the kernel exit cleanly instead of hanging.
 * sdpa_device_status synchronises the current device, returns
 * SDPA_ERR_TIMEOUT if any kernel gave up since the last clear (and
 * SDPA_ERR_CUDA if synchronisation itself failed), and clears the word when
 * `clear` is non-zero.
 */
SDPA_API sdpa_status sdpa_device_status(int clear);

/*
 * Test hook for the watchdog: limit (nanoseconds) on each bounded wait of
 * later calls on this host process; 0 restores the default (about 2 s).
 */
SDPA_API void sdpa_set_wait_limit_ns(uint64_t ns);

/*
 * Watchdog self-test: launches one CTA whose bounded wait is on an mbarrier
 * that nothing ever arrives on, with limit `limit_ns` (0 = 100 ms).  The wait
 * must expire, record its code in the watchdog word and let the kernel exit;
 * no GPU fault is involved.  Synchronises the device.  *waited_out is 0 when
 * the wait expired as designed, 1 if it (wrongly) completed.  Afterwards
 * sdpa_device_status reports SDPA_ERR_TIMEOUT until cleared.
 */
SDPA_API sdpa_status sdpa_watchdog_selftest(uint64_t limit_ns, int *waited_out);

/*
 * Profiling hook: the next sdpa_forward* call made by this host thread
 * records `start_event` on its stream right before its main attention kernel
 * and `stop_event` right after it (before any combine launch), then disarms.
 * Both are cudaEvent_t handles owned by the caller; NULL, NULL disarms.
 */
SDPA_API void sdpa_time_next_main_kernel(void *start_event, void *stop_event);

/*
 * As sdpa_time_next_main_kernel, plus `call_event` recorded after the last
 * launch of the call (after the combine, when there is one).  NULL events
 * are skipped.
 */
SDPA_API void sdpa_time_next_call(void *start_event, void *stop_event, void *call_event);

/*
 * Self-test of the kernels' FMA-pipe exp2 (a Cody-Waite range reduction with
 * a fitted minimax polynomial, used for part of the softmax exponentials):
 * writes that function's value and exp2f's for n points spread evenly over
 * [lo, hi] into the device arrays poly[n] and ref[n] (caller-owned, fp32),
 * asynchronously on the legacy default stream.  For tests; no counterpart in
 * the pages.
 */
SDPA_API sdpa_status sdpa_exp2_selftest(float lo, float hi, int n, float *poly, float *ref);

SDPA_API const char *sdpa_status_string(sdpa_status status);
/* Message of the last failed call on this thread ("" if none). */
SDPA_API const char *sdpa_last_error_message(void);
/* Library version, major*10000 + minor*100 + patch. */
SDPA_API int sdpa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SDPA_H_ */
