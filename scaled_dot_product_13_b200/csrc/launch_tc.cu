// Launch unit of the tcgen05 attention kernel.
#include "launch.h"
#include "tc.cuh"

// upper bound on K/V ring slots (shared memory allowing)
#ifndef SDPA_TC_MAX_SLOTS
#define SDPA_TC_MAX_SLOTS 8
#endif

namespace sdpa {

namespace {

template <bool kBF16, int DQK, int DV>
sdpa_status run_tc(const Launch &ln, std::string *err) {
  constexpr int kBN = tc_key_block(DQK, DV);
  constexpr uint32_t kQ = ((DQK + 63) / 64) * 128 * 128;
  constexpr uint32_t kK = ((DQK + 63) / 64) * kBN * 128;
  constexpr uint32_t kV = ((DV + 63) / 64) * kBN * 128;
  constexpr uint32_t kSlot = kK > kV ? kK : kV;
  // everything but Q and the slots: row-max exchange and the barriers
  constexpr uint32_t kBudget =
      232448u - 2u * SDPA_TC_PARTS * 128u * 4u - (2u * SDPA_TC_MAX_SLOTS + 17u) * 8u - 16u;
  constexpr int kFit = (int)((kBudget - kQ) / kSlot);
  constexpr int kNSlot = kFit > SDPA_TC_MAX_SLOTS ? SDPA_TC_MAX_SLOTS : kFit;
  static_assert(kNSlot >= 2, "at least two K/V slots");
  using Cfg = TcCfg<DQK, DV, kBN, kNSlot>;
  auto kern = tc_attn_kernel<kBF16, DQK, DV, kBN, kNSlot>;
  sdpa_status st =
      prepare_kernel((const void *)kern, Cfg::kThreads, Cfg::kSmemBytes, "tc_attn_kernel", err);
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
  // head dims above 256: one CTA per half of V and O (grid.y); programmatic
  // stream serialization: the set-up overlaps the previous grid's tail
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(pl.ctas / pl.col_halves), (unsigned)pl.col_halves);
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
    *err = std::string("tc_attn_kernel launch failed: ") + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  return SDPA_OK;
}

template <bool kBF16>
sdpa_status run_dtype(const Launch &ln, std::string *err) {
  switch (ln.plan.pair) {
    case 0: return run_tc<kBF16, 64, 64>(ln, err);
    case 1: return run_tc<kBF16, 80, 80>(ln, err);
    case 2: return run_tc<kBF16, 128, 128>(ln, err);
    case 3: return run_tc<kBF16, 192, 128>(ln, err);
    case 4: return run_tc<kBF16, 192, 192>(ln, err);
    case 5: return run_tc<kBF16, 256, 256>(ln, err);
    case 6: return run_tc<kBF16, 512, kTcWideHalf>(ln, err);
  }
  *err = "internal: no tcgen05 instance for this head-dim pair";
  return SDPA_ERR_UNSUPPORTED;
}

}  // namespace

sdpa_status launch_tc(const Launch &ln, std::string *err) {
  return ln.pb.dtype == SDPA_BF16 ? run_dtype<true>(ln, err) : run_dtype<false>(ln, err);
}

}  // namespace sdpa
