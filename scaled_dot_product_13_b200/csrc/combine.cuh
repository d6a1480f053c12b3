// Log-sum-exp combine of split partials (mlx issue #3826: split over S, then
// a log-sum-exp merge; mlx PR #3637: the 2-pass kernel's aggregation).
// One CTA of 128 threads per output row and 128 output columns:
//   LSE = max_s LSE_s + ln sum_s exp(LSE_s - max),  O = sum_s exp(LSE_s - LSE) O_s
// Splits that saw no visible key carry LSE_s = -inf and weight 0.  A head's
// sink (when given) joins as one more term with weight exp(sink - LSE) and
// no value row.  Warp 0 forms the weights in shared memory while every
// thread already has its column's partials of the first splits in flight;
// after one barrier each thread accumulates its output column.
// Launched as a programmatic dependent of the split pass: it waits for that
// grid (griddepcontrol.wait) before touching the partials.
#pragma once

#include "params.cuh"

// splits loaded per round trip to L2 after the first kPre
#ifndef SDPA_COMBINE_BATCH
#define SDPA_COMBINE_BATCH 8
#endif

namespace sdpa {

template <bool kBF16>
__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ part_o,
                                                      const float *__restrict__ part_lse,
                                                      void *__restrict__ out, float *lse_out,
                                                      const float *__restrict__ sinks,
                                                      long total_rows, int Dv, int splits, int L,
                                                      int Hq) {
  extern __shared__ float s_w[];  // [splits]
  __shared__ float s_res[2];      // 1 / denominator, LSE
  constexpr int kPre = 32;        // splits whose partials are loaded before the weights exist
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int col = blockIdx.y * 128 + tid;  // this thread's output column
  const bool live = col < Dv;
  const long stride = total_rows * Dv;
  const float *src = part_o + row * Dv + col;
  // the partial loads go out first, in flight while warp 0 forms the weights
  float v[kPre];
#pragma unroll
  for (int t = 0; t < kPre; ++t) v[t] = (t < splits && live) ? __ldcg(src + (long)t * stride) : 0.f;
  if (tid < 32) {
    // warp 0: max of the split LSEs (and the sink), weights, denominator
    float mx = -INFINITY;
    for (int s = lane; s < splits; s += 32) {
      const float x = __ldcg(part_lse + (long)s * total_rows + row);
      s_w[s] = x;
      mx = fmaxf(mx, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float sink = sinks != nullptr ? sinks[(int)((row / L) % Hq)] : -INFINITY;
    mx = fmaxf(mx, sink);
    const float ref = mx == -INFINITY ? 0.f : mx;
    float den = 0.f;
    for (int s = lane; s < splits; s += 32) {  // each lane rereads its own entries
      const float w = __expf(s_w[s] - ref);
      s_w[s] = w;
      den += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (sinks != nullptr) den += __expf(sink - ref);
    if (lane == 0) {
      s_res[0] = den > 0.f ? 1.f / den : 0.f;
      s_res[1] = den > 0.f ? ref + logf(den) : -INFINITY;
    }
  }
  __syncthreads();
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < kPre; ++t)
    if (t < splits) acc += s_w[t] * v[t];
  // the remaining splits, kBatch per round trip to L2
  constexpr int kBatch = SDPA_COMBINE_BATCH;
  for (int s0 = kPre; s0 < splits; s0 += kBatch) {
    float x[kBatch];
#pragma unroll
    for (int t = 0; t < kBatch; ++t)
      x[t] = (s0 + t < splits && live) ? __ldcg(src + (long)(s0 + t) * stride) : 0.f;
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const float w = s0 + t < splits ? s_w[s0 + t] : 0.f;
      acc += w * x[t];
    }
  }
  if (live) {
    const float o = acc * s_res[0];
    if constexpr (kBF16)
      reinterpret_cast<__nv_bfloat16 *>(out)[row * Dv + col] = __float2bfloat16_rn(o);
    else
      reinterpret_cast<__half *>(out)[row * Dv + col] = __float2half_rn(o);
  }
  if (lse_out != nullptr && blockIdx.y == 0 && tid == 0) lse_out[row] = s_res[1];
}

}  // namespace sdpa
