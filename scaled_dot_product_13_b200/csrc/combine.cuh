// Log-sum-exp combine of split partials (mlx issue #3826: split over S, then
// a log-sum-exp merge; mlx PR #3637: the 2-pass kernel's aggregation).
// One CTA of 128 threads per output row and 128 output columns:
//   LSE = max_s LSE_s + ln sum_s exp(LSE_s - max),  O = sum_s exp(LSE_s - LSE) O_s
// Splits that saw no visible key carry LSE_s = -inf and weight 0.  A head's
// sink (when given) joins as one more term with weight exp(sink - LSE) and
// no value row.  Every thread loads its column's partials of the first 64
// splits and one split LSE in the same round trip to L2; two block
// reductions (max, then the weight sum) form the weights in shared memory,
// and each thread accumulates its output column.
// Launched as a programmatic dependent of the split pass: it waits for that
// grid (griddepcontrol.wait) before touching the partials.
#pragma once

#include "params.cuh"

// splits loaded per round trip to L2 after the first kPre
#ifndef SDPA_COMBINE_BATCH
#define SDPA_COMBINE_BATCH 16
#endif

namespace sdpa {

template <bool kBF16>
__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ part_o,
                                                      const float *__restrict__ part_lse,
                                                      void *__restrict__ out, float *lse_out,
                                                      const float *__restrict__ sinks,
                                                      long total_rows, int Dv, int splits, int L,
                                                      int Hq) {
  extern __shared__ float s_w[];  // [splits]: the split LSEs, then their weights
  __shared__ float s_red[2][4];   // per-warp max, per-warp weight sum
  constexpr int kPre = 64;        // splits whose partials go out in the first round trip
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next split pass on the stream may start its setup now; it waits for
  // this grid before it reads or writes global memory
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col = blockIdx.y * 128 + tid;  // this thread's output column
  const bool live = col < Dv;
  const long stride = total_rows * Dv;
  const float *src = part_o + row * Dv + col;
  // One round trip to L2: each thread's partials of the first kPre splits and
  // one split LSE per thread (up to 128 splits; more take further rounds).
  float v[kPre];
#pragma unroll
  for (int t = 0; t < kPre; ++t) v[t] = (t < splits && live) ? __ldcg(src + (long)t * stride) : 0.f;
  float mx = -INFINITY;
  for (int s = tid; s < splits; s += 128) {
    const float x = __ldcg(part_lse + (long)s * total_rows + row);
    s_w[s] = x;
    mx = fmaxf(mx, x);
  }
  // block max of the split LSEs and the sink
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[0][warp] = mx;
  __syncthreads();
  const float sink = sinks != nullptr ? sinks[(int)((row / L) % Hq)] : -INFINITY;
  mx = fmaxf(fmaxf(fmaxf(s_red[0][0], s_red[0][1]), fmaxf(s_red[0][2], s_red[0][3])), sink);
  const float ref = mx == -INFINITY ? 0.f : mx;
  // weights exp(LSE_s - ref); each thread rereads the entries it wrote
  float den = 0.f;
  for (int s = tid; s < splits; s += 128) {
    const float w = __expf(s_w[s] - ref);
    s_w[s] = w;
    den += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane == 0) s_red[1][warp] = den;
  __syncthreads();
  den = (s_red[1][0] + s_red[1][1]) + (s_red[1][2] + s_red[1][3]);
  if (sinks != nullptr) den += __expf(sink - ref);
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < kPre; ++t) {
    const float w = t < splits ? s_w[t] : 0.f;
    acc += w * v[t];
  }
  // splits past kPre, kBatch per round trip
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
    const float o = den > 0.f ? acc / den : 0.f;
    if constexpr (kBF16)
      reinterpret_cast<__nv_bfloat16 *>(out)[row * Dv + col] = __float2bfloat16_rn(o);
    else
      reinterpret_cast<__half *>(out)[row * Dv + col] = __float2half_rn(o);
  }
  if (lse_out != nullptr && blockIdx.y == 0 && tid == 0)
    lse_out[row] = den > 0.f ? ref + logf(den) : -INFINITY;
}

}  // namespace sdpa
