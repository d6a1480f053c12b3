// Launch unit of the two-tile (ping-pong) tcgen05 kernel: two 128-row tiles
// per CTA (SDPA_PATH_TC_DUAL) or one tile whose two softmax groups take
// alternate key blocks (SDPA_PATH_TC_KSPLIT).
#include "launch.h"
#include "tc_pp.cuh"

namespace sdpa {

namespace {

template <bool kBF16, int DQK, int DV, bool kKSplit>
sdpa_status run_tc_pp(const Launch &ln, std::string *err) {
  constexpr int kPair = DQK == 64 ? 0 : DQK == 80 ? 1 : 2;
  constexpr int kBN = tc_pp_key_block(kPair, kKSplit);
  if (ln.plan.key_block != kBN) {
    *err = "internal: the plan's key block does not match the two-tile instance";
    return SDPA_ERR_UNSUPPORTED;
  }
  constexpr uint32_t kQ = (kKSplit ? 1u : 2u) * ((DQK + 63) / 64) * 128 * 128;
  constexpr uint32_t kK = ((DQK + 63) / 64) * kBN * 128;
  constexpr uint32_t kV = ((DV + 63) / 64) * kBN * 128;
  constexpr uint32_t kSlot = kK > kV ? kK : kV;
  constexpr uint32_t kBudget =
      232448u - (2u * 8u + 14u) * 8u - 16u - (kKSplit ? 2u * 128u * 8u : 0u);
  constexpr int kFit = (int)((kBudget - kQ) / kSlot);
  constexpr int kNSlot = kFit > 8 ? 8 : kFit;
  static_assert(kNSlot >= 2, "at least two K/V slots");
  using Cfg = PpCfg<DQK, DV, kBN, kNSlot, kKSplit>;
  auto kern = tc_pp_attn_kernel<kBF16, DQK, DV, kBN, kNSlot, kKSplit>;
  sdpa_status st = prepare_kernel((const void *)kern, Cfg::kThreads, Cfg::kSmemBytes,
                                  "tc_pp_attn_kernel", err);
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
  if (ln.ev_start) record_event(ln.ev_start, ln.stream);
  // programmatic stream serialization: the set-up overlaps the previous
  // grid's tail
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, tp, p);
  if (ln.ev_stop) record_event(ln.ev_stop, ln.stream);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = std::string("tc_pp_attn_kernel launch failed: ") + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  return SDPA_OK;
}

template <bool kBF16>
sdpa_status run_dtype(const Launch &ln, std::string *err) {
  const bool ks = ln.plan.path == SDPA_PATH_TC_KSPLIT;
  switch (ln.plan.pair) {
    case 0: return ks ? run_tc_pp<kBF16, 64, 64, true>(ln, err) : run_tc_pp<kBF16, 64, 64, false>(ln, err);
    case 1: return ks ? run_tc_pp<kBF16, 80, 80, true>(ln, err) : run_tc_pp<kBF16, 80, 80, false>(ln, err);
    case 2:
      return ks ? run_tc_pp<kBF16, 128, 128, true>(ln, err)
                : run_tc_pp<kBF16, 128, 128, false>(ln, err);
  }
  *err = "internal: no two-tile instance for this head-dim pair";
  return SDPA_ERR_UNSUPPORTED;
}

}  // namespace

sdpa_status launch_tc_pp(const Launch &ln, std::string *err) {
  return ln.pb.dtype == SDPA_BF16 ? run_dtype<true>(ln, err) : run_dtype<false>(ln, err);
}

}  // namespace sdpa
