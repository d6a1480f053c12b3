// Log-sum-exp combine of split partials (mlx issue #3826: split over S, then
// a log-sum-exp merge; mlx PR #3637: the 2-pass kernel's aggregation).
//   LSE = max_s LSE_s + ln sum_s exp(LSE_s - max),  O = sum_s exp(LSE_s - LSE) O_s
// Splits that saw no visible key carry LSE_s = -inf and weight 0.  A head's
// sink (when given) joins as one more term with weight exp(sink - LSE) and
// no value row.
//
// One warp per output row and 128 output columns, four rows per CTA: each
// lane owns four adjacent columns (one 16-byte load per split) and holds the
// LSE of split `lane` of each round of 32.  The first round's partials and
// LSEs are requested together, so up to 32 splits cost one round trip to L2
// before the reductions; the LSE max and the weight sum are warp shuffles
// (no shared memory, no block barrier), and each split's weight reaches the
// lanes by one more shuffle.
// Launched as a programmatic dependent of the split pass: it waits for that
// grid (griddepcontrol.wait) before touching the partials.
#pragma once

#include "params.cuh"

namespace sdpa {

constexpr int kCombineRowsPerCta = 4;

template <bool kBF16>
__global__ void __launch_bounds__(32 * kCombineRowsPerCta)
    combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                   void *__restrict__ out, float *lse_out, const float *__restrict__ sinks,
                   long total_rows, int Dv, int splits, int L, int Hq) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next split pass on the stream may start its setup now; it waits for
  // this grid before it reads or writes global memory
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long row = (long)blockIdx.x * kCombineRowsPerCta + (threadIdx.x >> 5);
  if (row >= total_rows) return;  // whole warps
  const int col = blockIdx.y * 128 + lane * 4;  // this lane's four output columns
  const bool live = col < Dv;                   // Dv is a multiple of 8
  const long stride = total_rows * Dv;          // floats between two splits' partials
  const float *src = part_o + row * Dv + col;
  const float *lse = part_lse + row;

  // ---- first round: the partials of splits 0..31 and their LSEs (lane s
  // holds split s's) go out together, before any reduction ----
  float4 v[32];
#pragma unroll
  for (int k = 0; k < 32; ++k)
    v[k] = (live && k < splits)
               ? __ldcg(reinterpret_cast<const float4 *>(src + (long)k * stride))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  const float lse0 = lane < splits ? __ldcg(lse + (long)lane * total_rows) : -INFINITY;
  // the LSE max over all splits (and the sink)
  float mx = lse0;
  for (int s = lane + 32; s < splits; s += 32) mx = fmaxf(mx, __ldcg(lse + (long)s * total_rows));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float sink = sinks != nullptr ? sinks[(int)((row / L) % Hq)] : -INFINITY;
  mx = fmaxf(mx, sink);
  const float ref = mx == -INFINITY ? 0.f : mx;

  // ---- weighted sum: lane s's weight is shuffled out to every lane ----
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float w_own = lane < splits ? __expf(lse0 - ref) : 0.f;
  float den = w_own;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float w = __shfl_sync(0xffffffffu, w_own, k);
    acc.x += w * v[k].x;
    acc.y += w * v[k].y;
    acc.z += w * v[k].z;
    acc.w += w * v[k].w;
  }
  // further rounds of 32 splits
  for (int s0 = 32; s0 < splits; s0 += 32) {
    const int s = s0 + lane;
#pragma unroll
    for (int k = 0; k < 32; ++k)
      v[k] = (live && s0 + k < splits)
                 ? __ldcg(reinterpret_cast<const float4 *>(src + (long)(s0 + k) * stride))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    w_own = s < splits ? __expf(__ldcg(lse + (long)s * total_rows) - ref) : 0.f;
    den += w_own;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float w = __shfl_sync(0xffffffffu, w_own, k);
      acc.x += w * v[k].x;
      acc.y += w * v[k].y;
      acc.z += w * v[k].z;
      acc.w += w * v[k].w;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (sinks != nullptr) den += __expf(sink - ref);

  const float inv = den > 0.f ? 1.f / den : 0.f;
  if (live) {
    uint2 w;
    w.x = pack2<kBF16>(acc.x * inv, acc.y * inv);
    w.y = pack2<kBF16>(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(out) + row * Dv + col) = w;
  }
  if (lse_out != nullptr && blockIdx.y == 0 && lane == 0)
    lse_out[row] = den > 0.f ? ref + logf(den) : -INFINITY;
}

}  // namespace sdpa
