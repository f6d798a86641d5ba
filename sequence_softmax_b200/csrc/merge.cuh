// merge.cuh -- lse-weighted merge of n partial attention states (HBM-bandwidth bound).
//
// From the associativity lse(x) = lse([lse(x1), lse(x2)]) ([LECTURE] log-sum-exp passage):
// per row, L = max_i lse_i + log sum_i exp(lse_i - max) and O = sum_i exp(lse_i - L) O_i.
// Every partial byte is read exactly once and the output written once, so the roofline is
// HBM bandwidth. One warp owns a row at a time: lane i < n loads lse_i (weights are then
// broadcast by shuffle) and every lane streams 16-byte float4 chunks of the n partial rows
// with cache-streaming loads; rows are walked grid-stride, two per warp iteration so that
// each lane keeps 2n independent 16-byte loads in flight.
#pragma once

#include "common.cuh"

namespace ra {

constexpr int MERGE_THREADS = 256;

template <bool OUT_BF16>
__device__ __forceinline__ void merge_store4(void* out, int64_t idx4, float a, float b, float c, float e) {
  if (OUT_BF16) {
    uint2 w;
    w.x = pack_bf16x2(a, b);
    w.y = pack_bf16x2(c, e);
    __stcs(reinterpret_cast<uint2*>(out) + idx4, w);
  } else {
    __stcs(reinterpret_cast<float4*>(out) + idx4, make_float4(a, b, c, e));
  }
}

// At most 64 parts: lane i holds the weights of parts i and i + 32.
constexpr int MERGE_MAX_PARTS = 64;

// Weight of part i (warp-uniform i), broadcast from the lane that holds it.
__device__ __forceinline__ float weight_of(const float (&w)[2], int i) {
  return __shfl_sync(0xffffffffu, i < 32 ? w[0] : w[1], i & 31);
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(MERGE_THREADS)
merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int n, int64_t rows, int d,
             void* __restrict__ o_out, float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * MERGE_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * MERGE_THREADS) >> 5;
  const int d4 = d >> 2;
  const float4* op4 = reinterpret_cast<const float4*>(o_parts);
  const int64_t part_stride4 = rows * d4;

  for (int64_t r0 = warp_global * 2; r0 < rows; r0 += nwarps * 2) {
    const int nr = (r0 + 1 < rows) ? 2 : 1;
    float w[2][2];  // weights of parts lane and lane + 32, for the two rows
    float L[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int64_t r = r0 + q;
      float x0 = -INFINITY, x1 = -INFINITY;
      if (q < nr) {
        if (lane < n) x0 = __ldcs(lse_parts + (int64_t)lane * rows + r);
        if (lane + 32 < n) x1 = __ldcs(lse_parts + (int64_t)(lane + 32) * rows + r);
      }
      float mx = fmaxf(x0, x1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float sh = (mx == -INFINITY) ? 0.f : mx;
      float e0 = expf(x0 - sh), e1 = expf(x1 - sh);
      float tot = e0 + e1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
      const float inv = tot > 0.f ? 1.f / tot : 0.f;
      w[q][0] = e0 * inv;
      w[q][1] = e1 * inv;
      L[q] = tot > 0.f ? sh + logf(tot) : -INFINITY;
    }
    // Uniform trip count so that every lane takes part in the weight shuffles.
    for (int c0 = 0; c0 < d4; c0 += 32) {
      const int c = c0 + lane;
      const bool act = c < d4;
      const int cc = act ? c : 0;  // inactive lanes read a valid address and store nothing
      float4 acc[2];
      acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      int i = 0;
      for (; i + 2 <= n; i += 2) {
        const float wa0 = weight_of(w[0], i), wb0 = weight_of(w[0], i + 1);
        const float wa1 = weight_of(w[1], i), wb1 = weight_of(w[1], i + 1);
        const float4 a0 = __ldcs(op4 + i * part_stride4 + r0 * d4 + cc);
        const float4 b0 = __ldcs(op4 + (i + 1) * part_stride4 + r0 * d4 + cc);
        float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = a1;
        if (nr == 2) {
          a1 = __ldcs(op4 + i * part_stride4 + (r0 + 1) * d4 + cc);
          b1 = __ldcs(op4 + (i + 1) * part_stride4 + (r0 + 1) * d4 + cc);
        }
        acc[0].x = fmaf(wa0, a0.x, fmaf(wb0, b0.x, acc[0].x));
        acc[0].y = fmaf(wa0, a0.y, fmaf(wb0, b0.y, acc[0].y));
        acc[0].z = fmaf(wa0, a0.z, fmaf(wb0, b0.z, acc[0].z));
        acc[0].w = fmaf(wa0, a0.w, fmaf(wb0, b0.w, acc[0].w));
        acc[1].x = fmaf(wa1, a1.x, fmaf(wb1, b1.x, acc[1].x));
        acc[1].y = fmaf(wa1, a1.y, fmaf(wb1, b1.y, acc[1].y));
        acc[1].z = fmaf(wa1, a1.z, fmaf(wb1, b1.z, acc[1].z));
        acc[1].w = fmaf(wa1, a1.w, fmaf(wb1, b1.w, acc[1].w));
      }
      for (; i < n; ++i) {
        const float wa0 = weight_of(w[0], i), wa1 = weight_of(w[1], i);
        const float4 a0 = __ldcs(op4 + i * part_stride4 + r0 * d4 + cc);
        float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (nr == 2) a1 = __ldcs(op4 + i * part_stride4 + (r0 + 1) * d4 + cc);
        acc[0].x = fmaf(wa0, a0.x, acc[0].x);
        acc[0].y = fmaf(wa0, a0.y, acc[0].y);
        acc[0].z = fmaf(wa0, a0.z, acc[0].z);
        acc[0].w = fmaf(wa0, a0.w, acc[0].w);
        acc[1].x = fmaf(wa1, a1.x, acc[1].x);
        acc[1].y = fmaf(wa1, a1.y, acc[1].y);
        acc[1].z = fmaf(wa1, a1.z, acc[1].z);
        acc[1].w = fmaf(wa1, a1.w, acc[1].w);
      }
      if (act) {
        merge_store4<OUT_BF16>(o_out, r0 * d4 + c, acc[0].x, acc[0].y, acc[0].z, acc[0].w);
        if (nr == 2) merge_store4<OUT_BF16>(o_out, (r0 + 1) * d4 + c, acc[1].x, acc[1].y, acc[1].z, acc[1].w);
      }
    }
    if (lse_out != nullptr && lane == 0) {
      lse_out[r0] = L[0];
      if (nr == 2) lse_out[r0 + 1] = L[1];
    }
  }
}

}  // namespace ra
