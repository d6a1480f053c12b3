// Launch unit of the wide (column-split) kernel for head dims above 256.
#include "launch.h"
#include "wide.cuh"

namespace sdpa {

namespace {

template <bool kBF16, int WR>
sdpa_status run_wide(const Launch &ln, std::string *err) {
  constexpr int kDqk = 512, kDv = 512, kBN = kWideBN;
  // stages: as many as fit next to Q, P and the exchange buffer, at most 4
  constexpr uint32_t kStage = (kDqk / 64 + kDv / 64) * kBN * 128;
  constexpr uint32_t kFixed = (kDqk / 64) * 16 * WR * 128 + 16 * WR * kBN * 2 + WR * 4 * 16 * 4 +
                              9 * 8;
  constexpr int kFit = (int)((232448u - kFixed) / kStage);
  constexpr int kNST = kFit > 4 ? 4 : kFit;
  static_assert(kNST >= 2, "at least double buffering");
  using Cfg = WideCfg<kDqk, kDv, kBN, WR, kNST>;
  auto kern = wide_kernel<kBF16, kDqk, kDv, kBN, WR, kNST>;
  sdpa_status st =
      prepare_kernel((const void *)kern, Cfg::kThreads, Cfg::kSmemBytes, "wide_kernel", err);
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
  kern<<<(unsigned)pl.ctas, Cfg::kThreads, Cfg::kSmemBytes, ln.stream>>>(tq, tk, tv, p);
  if (ln.ev_stop) record_event(ln.ev_stop, ln.stream);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = std::string("wide_kernel launch failed: ") + cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
  }
  return SDPA_OK;
}

template <bool kBF16>
sdpa_status run_dtype(const Launch &ln, std::string *err) {
  if (ln.plan.pair != kWidePair) {
    *err = "internal: the wide kernel is built for head dims 512/512 only";
    return SDPA_ERR_UNSUPPORTED;
  }
  if (ln.plan.wr == 1) return run_wide<kBF16, 1>(ln, err);
  if (ln.plan.wr == 2) return run_wide<kBF16, 2>(ln, err);
  *err = "internal: no wide row-group layout for this plan";
  return SDPA_ERR_UNSUPPORTED;
}

}  // namespace

sdpa_status launch_wide(const Launch &ln, std::string *err) {
  return ln.pb.dtype == SDPA_BF16 ? run_dtype<true>(ln, err) : run_dtype<false>(ln, err);
}

}  // namespace sdpa
