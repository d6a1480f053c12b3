// Launch unit of the split-KV kernel and the log-sum-exp combine.
#include <cmath>

#include "launch.h"
#include "combine.cuh"
#include "splitkv.cuh"

namespace sdpa {

namespace {

template <bool kBF16, int DQK, int DV, int WR, int WK>
sdpa_status run_splitkv(const Launch &ln, std::string *err) {
  constexpr int kBN = splitkv_bn(DQK, DV);
  // one or two CTAs per SM; stages: as many as fit next to Q, at most 4
  constexpr int kMinB = splitkv_ctas_per_sm(DQK, DV, WR);
  constexpr int kNST =
      splitkv_stages(DQK, DV, WR, kMinB == 2 ? kSplitKvBudget2 : kSplitKvBudget1);
  static_assert(kNST >= 2, "at least double buffering");
  using Cfg = SplitKvCfg<DQK, DV, kBN, WR, WK, kNST>;
  static_assert(kMinB == 1 || Cfg::kSmemBytes + 1024 <= 233472u / 2, "two CTAs per SM");
  auto kern = splitkv_kernel<kBF16, DQK, DV, kBN, WR, WK, kNST, kMinB>;
  sdpa_status st = prepare_kernel((const void *)kern, Cfg::kThreads, Cfg::kSmemBytes,
                                  "splitkv_kernel", err);
  if (st != SDPA_OK) return st;

  const Problem &pb = ln.pb;
  const Plan &pl = ln.plan;
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[2] = {(uint64_t)pb.Dqk, (uint64_t)pb.B * pb.Hq * pb.L};
    const uint64_t strides[1] = {(uint64_t)pb.Dqk * 2};
    const uint32_t box[2] = {64, (uint32_t)Cfg::kRT};
    if (!encode_tma(&tq, pb.dtype, 2, ln.q, dims, strides, box, err)) return SDPA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)pb.Dqk, (uint64_t)pb.S, (uint64_t)pb.B * pb.Hkv};
    const uint64_t strides[2] = {(uint64_t)pb.Dqk * 2, (uint64_t)pb.S * pb.Dqk * 2};
    const uint32_t box[3] = {64, (uint32_t)kBN, 1};
    if (!encode_tma(&tk, pb.dtype, 3, ln.k, dims, strides, box, err)) return SDPA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)pb.Dv, (uint64_t)pb.S, (uint64_t)pb.B * pb.Hkv};
    const uint64_t strides[2] = {(uint64_t)pb.Dv * 2, (uint64_t)pb.S * pb.Dv * 2};
    const uint32_t box[3] = {64, (uint32_t)kBN, 1};
    if (!encode_tma(&tv, pb.dtype, 3, ln.v, dims, strides, box, err)) return SDPA_ERR_CUDA;
  }
  AttnParams p;
  p.B = pb.B; p.Hq = pb.Hq; p.Hkv = pb.Hkv; p.L = pb.L; p.S = pb.S; p.Dqk = pb.Dqk; p.Dv = pb.Dv;
  p.R = pl.rows;
  p.off = pb.q_offset;
  p.causal = pb.causal;
  p.window = pb.window;
  p.scale_log2 = pb.scale * 1.4426950408889634f;
  p.row_tiles = pl.row_tiles;
  p.splits = pl.splits;
  p.split_base = pl.split_base;
  p.keys_per_split = pl.keys_per_split;
  p.out = ln.out;
  p.part_o = ln.part_o;
  p.part_lse = ln.part_lse;
  p.sinks = ln.sinks;
  p.lse_out = ln.lse_out;
  p.wd.word = ln.wd_word;
  p.wd.limit_ns = ln.wd_limit_ns;
  if (ln.ev_start) record_event(ln.ev_start, ln.stream);
  // programmatic stream serialization: the kernel's setup may overlap the
  // previous grid on the stream; it waits (griddepcontrol.wait) before any
  // global memory access
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.ctas);
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = ln.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
  if (ln.ev_stop) record_event(ln.ev_stop, ln.stream);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = std::string("splitkv_kernel launch failed: ") + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  return SDPA_OK;
}

template <bool kBF16, int DQK, int DV>
sdpa_status run_layout(const Launch &ln, std::string *err) {
  const Plan &pl = ln.plan;
  if constexpr (splitkv_bn(DQK, DV) >= 128) {
    // 128-key blocks: eight warps of 16 keys each for one 16-row group
    if (pl.wr == 1 && pl.wk == 8) return run_splitkv<kBF16, DQK, DV, 1, 8>(ln, err);
  }
  if (pl.wr == 1 && pl.wk == 4) return run_splitkv<kBF16, DQK, DV, 1, 4>(ln, err);
  if (pl.wr == 2 && pl.wk == 2) return run_splitkv<kBF16, DQK, DV, 2, 2>(ln, err);
  if (pl.wr == 4 && pl.wk == 1) return run_splitkv<kBF16, DQK, DV, 4, 1>(ln, err);
  *err = "internal: no split-KV warp layout for this plan";
  return SDPA_ERR_UNSUPPORTED;
}

template <bool kBF16>
sdpa_status run_dtype(const Launch &ln, std::string *err) {
  switch (ln.plan.pair) {
    case 0: return run_layout<kBF16, 64, 64>(ln, err);
    case 1: return run_layout<kBF16, 80, 80>(ln, err);
    case 2: return run_layout<kBF16, 128, 128>(ln, err);
    case 3: return run_layout<kBF16, 192, 128>(ln, err);
    case 4: return run_layout<kBF16, 192, 192>(ln, err);
    case 5: return run_layout<kBF16, 256, 256>(ln, err);
  }
  *err = "internal: no split-KV instance for this head-dim pair";
  return SDPA_ERR_UNSUPPORTED;
}

}  // namespace

sdpa_status launch_splitkv(const Launch &ln, std::string *err) {
  return ln.pb.dtype == SDPA_BF16 ? run_dtype<true>(ln, err) : run_dtype<false>(ln, err);
}

sdpa_status launch_combine(const Launch &ln, std::string *err) {
  // Launched as a programmatic dependent of the attention pass: its CTAs may
  // be scheduled before that grid finishes and wait (griddepcontrol.wait) for
  // it, which hides the second launch's latency.
  const long total = (long)ln.pb.B * ln.pb.Hq * ln.pb.L;
  cudaLaunchConfig_t cfg = {};
  // one warp per output row and 128 columns, kCombineRowsPerCta rows per CTA
  cfg.gridDim = dim3((unsigned)((total + kCombineRowsPerCta - 1) / kCombineRowsPerCta),
                     (unsigned)((ln.pb.Dv + 127) / 128));
  cfg.blockDim = dim3(32 * kCombineRowsPerCta);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = ln.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = ln.pb.dtype == SDPA_BF16 ? combine_kernel<true> : combine_kernel<false>;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, (const float *)ln.part_o,
                                     (const float *)ln.part_lse, ln.out, ln.lse_out, ln.sinks,
                                     total, ln.pb.Dv, ln.plan.splits, ln.pb.L, ln.pb.Hq);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = std::string("combine_kernel launch failed: ") + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  return SDPA_OK;
}

}  // namespace sdpa
