// Launch unit of the two-CTA (cta_group::2) attention kernel.
#include "launch.h"
#include "tc2.cuh"

namespace sdpa {

namespace {

// kLoop: the looping form (two Q buffers, so fewer K/V slots), grid of
// plan.loop_pairs pairs; otherwise one pair per 256-row tile.  DV is the
// output columns of one launch column (grid.y = plan.col_halves); kBN the
// key block.
template <bool kBF16, int DQK, int DV, bool kLoop, int kBN = 128>
sdpa_status run_tc2(const Launch &ln, std::string *err) {
  constexpr uint32_t kQ = (DQK / 64) * 128 * 128;
  constexpr uint32_t kK = (DQK / 64) * (kBN / 2) * 128;
  constexpr uint32_t kV = (DV / 128) * kBN * 128;  // this CTA's DV/2 columns
  constexpr uint32_t kSlot = kK > kV ? kK : kV;
  constexpr uint32_t kBudget = 232448u - 48u * 8u - 16u;
  constexpr int kFit = (int)((kBudget - (kLoop ? 2u : 1u) * kQ) / kSlot);
  constexpr int kNSlot = kFit > 8 ? 8 : kFit;
  static_assert(kNSlot >= 3, "at least three K/V slots");
  using Cfg = Tc2Cfg<DQK, DV, kBN, kNSlot, kLoop>;
  auto kern = tc2_attn_kernel<kBF16, DQK, DV, kBN, kNSlot, kLoop>;
  if (!Cfg::kSplitStage && ln.plan.splits != 1) {
    *err = "internal: this two-CTA instance does not split the keys";
    return SDPA_ERR_UNSUPPORTED;
  }
  sdpa_status st =
      prepare_kernel((const void *)kern, Cfg::kThreads, Cfg::kSmemBytes, "tc2_attn_kernel", err);
  if (st != SDPA_OK) return st;

  const Problem &pb = ln.pb;
  const Plan &pl = ln.plan;
  CUtensorMap tq, tk, tv, to, tp;
  {
    const uint64_t dims[2] = {(uint64_t)pb.Dqk, (uint64_t)pb.B * pb.Hq * pb.L};
    const uint64_t strides[1] = {(uint64_t)pb.Dqk * 2};
    const uint32_t box[2] = {64, 128};
    if (!encode_tma(&tq, pb.dtype, 2, ln.q, dims, strides, box, err)) return SDPA_ERR_CUDA;
  }
  {  // each CTA loads half of a key block: BN/2 keys
    const uint64_t dims[3] = {(uint64_t)pb.Dqk, (uint64_t)pb.S, (uint64_t)pb.B * pb.Hkv};
    const uint64_t strides[2] = {(uint64_t)pb.Dqk * 2, (uint64_t)pb.S * pb.Dqk * 2};
    const uint32_t box[3] = {64, (uint32_t)(kBN / 2), 1};
    if (!encode_tma(&tk, pb.dtype, 3, ln.k, dims, strides, box, err)) return SDPA_ERR_CUDA;
  }
  {  // and half of a value block's columns, all BN keys
    const uint64_t dims[3] = {(uint64_t)pb.Dv, (uint64_t)pb.S, (uint64_t)pb.B * pb.Hkv};
    const uint64_t strides[2] = {(uint64_t)pb.Dv * 2, (uint64_t)pb.S * pb.Dv * 2};
    const uint32_t box[3] = {64, (uint32_t)kBN, 1};
    if (!encode_tma(&tv, pb.dtype, 3, ln.v, dims, strides, box, err)) return SDPA_ERR_CUDA;
  }
  if (!encode_out_maps(ln, &to, &tp, err)) return SDPA_ERR_CUDA;
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

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * (kLoop ? (long long)pl.loop_pairs : pl.ctas / pl.col_halves)),
                     (unsigned)pl.col_halves);
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = ln.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic stream serialization: the set-up overlaps the previous
  // grid's tail
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (ln.ev_start) record_event(ln.ev_start, ln.stream);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, tp, p);
  if (ln.ev_stop) record_event(ln.ev_stop, ln.stream);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = std::string("tc2_attn_kernel launch failed: ") + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  return SDPA_OK;
}

template <bool kBF16, bool kLoop>
sdpa_status run_dtype(const Launch &ln, std::string *err) {
  switch (ln.plan.pair) {
    case 2: return run_tc2<kBF16, 128, 128, kLoop>(ln, err);
    case 3: return run_tc2<kBF16, 192, 128, kLoop>(ln, err);
    case 5: return run_tc2<kBF16, 256, 256, kLoop>(ln, err);
    case kWidePair:
      // head dim 512 in two 256-column halves, 64-key blocks (the 128 KB Q
      // tile leaves room for three 32 KB K/V slots and no second Q buffer)
      if constexpr (!kLoop) return run_tc2<kBF16, 512, kTc2WideHalf, false, 64>(ln, err);
      break;
  }
  *err = "internal: no two-CTA instance for this head-dim pair";
  return SDPA_ERR_UNSUPPORTED;
}

}  // namespace

sdpa_status launch_tc2(const Launch &ln, std::string *err) {
  const bool bf16 = ln.pb.dtype == SDPA_BF16;
  if (ln.plan.path == SDPA_PATH_TC2_LOOP)
    return bf16 ? run_dtype<true, true>(ln, err) : run_dtype<false, true>(ln, err);
  return bf16 ? run_dtype<true, false>(ln, err) : run_dtype<false, false>(ln, err);
}

}  // namespace sdpa
