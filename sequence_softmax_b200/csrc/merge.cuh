// merge.cuh -- lse-weighted merge of n partial attention states (HBM-bandwidth bound).
//
// From the associativity lse(x) = lse([lse(x1), lse(x2)]) ([LECTURE] log-sum-exp passage):
// per row, L = max_i lse_i + log sum_i exp(lse_i - max) and O = sum_i exp(lse_i - L) O_i.
// Every partial byte is read exactly once and the output written once, so the roofline is
// HBM bandwidth.
//
// Eight lanes own one row: each lane streams float4 chunks sub, sub + 8, sub + 16, ... of the
// n partial rows with cache-streaming loads, so one warp-wide load instruction covers four
// contiguous 128-byte segments. Every lane computes the row's weights itself from the n lse
// values (the same addresses for the eight lanes: one broadcast load each), so there are no
// shuffles; all CPL loads of a part are issued before they are used.
#pragma once

#include "common.cuh"

namespace ra {

constexpr int MERGE_THREADS = 256;
constexpr int MERGE_LANES_PER_ROW = 8;
constexpr int MERGE_MAX_PARTS = 64;

// CPL > 0: d == 4 * 8 * CPL, chunks fully unrolled. CPL == 0: any d % 4 == 0 (runtime loop).
template <bool OUT_BF16, int CPL>
__global__ void __launch_bounds__(MERGE_THREADS)
merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int n, int64_t rows, int d,
             void* __restrict__ o_out, float* __restrict__ lse_out) {
  const int sub = threadIdx.x & (MERGE_LANES_PER_ROW - 1);
  const int64_t group = ((int64_t)blockIdx.x * MERGE_THREADS + threadIdx.x) / MERGE_LANES_PER_ROW;
  const int64_t ngroups = ((int64_t)gridDim.x * MERGE_THREADS) / MERGE_LANES_PER_ROW;
  const int d4 = d >> 2;
  const float4* op4 = reinterpret_cast<const float4*>(o_parts);

  for (int64_t r = group; r < rows; r += ngroups) {
    // Weights of the n parts of row r (identical in the eight lanes).
    float mx = -INFINITY;
    for (int i = 0; i < n; ++i) mx = fmaxf(mx, __ldg(lse_parts + (int64_t)i * rows + r));
    const float sh = (mx == -INFINITY) ? 0.f : mx;
    float tot = 0.f;
    for (int i = 0; i < n; ++i) tot += expf(__ldg(lse_parts + (int64_t)i * rows + r) - sh);
    const bool empty = !(tot > 0.f);
    const float L = empty ? -INFINITY : sh + logf(tot);

    if (CPL > 0) {
      constexpr int NC = CPL > 0 ? CPL : 1;
      float4 acc[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int i = 0; i < n; ++i) {
        const float w = empty ? 0.f : expf(__ldg(lse_parts + (int64_t)i * rows + r) - L);
        const float4* src = op4 + ((int64_t)i * rows + r) * d4 + sub;
        float4 x[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) x[c] = __ldcs(src + c * MERGE_LANES_PER_ROW);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          acc[c].x = fmaf(w, x[c].x, acc[c].x);
          acc[c].y = fmaf(w, x[c].y, acc[c].y);
          acc[c].z = fmaf(w, x[c].z, acc[c].z);
          acc[c].w = fmaf(w, x[c].w, acc[c].w);
        }
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int64_t idx4 = r * d4 + sub + c * MERGE_LANES_PER_ROW;
        if (OUT_BF16) {
          uint2 v;
          v.x = pack_bf16x2(acc[c].x, acc[c].y);
          v.y = pack_bf16x2(acc[c].z, acc[c].w);
          __stcs(reinterpret_cast<uint2*>(o_out) + idx4, v);
        } else {
          __stcs(reinterpret_cast<float4*>(o_out) + idx4, acc[c]);
        }
      }
    } else {
      for (int c = sub; c < d4; c += MERGE_LANES_PER_ROW) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < n; ++i) {
          const float w = empty ? 0.f : expf(__ldg(lse_parts + (int64_t)i * rows + r) - L);
          const float4 x = __ldcs(op4 + ((int64_t)i * rows + r) * d4 + c);
          acc.x = fmaf(w, x.x, acc.x);
          acc.y = fmaf(w, x.y, acc.y);
          acc.z = fmaf(w, x.z, acc.z);
          acc.w = fmaf(w, x.w, acc.w);
        }
        const int64_t idx4 = r * d4 + c;
        if (OUT_BF16) {
          uint2 v;
          v.x = pack_bf16x2(acc.x, acc.y);
          v.y = pack_bf16x2(acc.z, acc.w);
          __stcs(reinterpret_cast<uint2*>(o_out) + idx4, v);
        } else {
          __stcs(reinterpret_cast<float4*>(o_out) + idx4, acc);
        }
      }
    }
    if (lse_out != nullptr && sub == 0) lse_out[r] = L;
  }
}

}  // namespace ra
