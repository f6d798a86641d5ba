// keybound.cuh -- the per-head key-norm bound that lets the forward skip row maxima.
//
// For a query row q and any key k of its head, the scaled score obeys
//   s * scale * log2(e) <= |q| max_k |k| * scale * log2(e)          (Cauchy-Schwarz).
// When that bound is within MAXSKIP_LOG2 of a row's running max m, no score of any tile can
// make exp2(s * scale * log2(e) - m) exceed 2^MAXSKIP_LOG2, so the forward may keep m without
// taking the tile's row max (the online update stays exact; only the size of the
// exponentials, not their ratios, depends on m). The forward computes |q| of its own rows
// from the Q tile in shared memory; this file computes max |k| per head, in two passes, and
// leaves it in every lse slot of the head. The forward thread that owns a row reads that
// slot once, before it overwrites it with the row's lse.
//   pass 1 (key_norm_chunk_kernel): block (c, bh) reduces key rows [c R, min(N, (c + 1) R))
//           of head bh to their largest norm and writes it into the first 4 bytes of O row c
//           of head bh (O is scratch until the forward's epilogue writes it);
//   pass 2 (key_norm_spread_kernel): every lse slot of head bh gets the largest of the C
//           chunk values.
// Pass 2 reads O and writes lse only, so its blocks never race with one another. NaN or inf
// in K propagates into the bound, and the forward then never skips.
//
// ra_key_norm_max (key_norm_max_kernel) writes the same per-head maximum into a caller array
// instead, for ra_partial_fold: every block folds its chunk's maximum in with an integer
// atomicMax on the float's bits (the order of non-negative floats, +inf and a positive NaN
// is that of their bit patterns), after a memset of the array to +0.
#pragma once

#include "common.cuh"

namespace ra {

constexpr int KB_MAX_CHUNKS = 1024;  // key chunks per head in pass 1 (at most the head's rows)
constexpr int KB_TARGET_BLOCKS = 4096;  // pass 1 grid: enough blocks to keep HBM busy
constexpr int KB_THREADS = 256;

// NaN-propagating maximum: once a NaN is seen the result stays NaN.
__device__ __forceinline__ float kb_max(float best, float x) { return (x > best || x != x) ? x : best; }

// Sum of squares of the 8 bf16 values in u (bf16 -> fp32 is exact).
__device__ __forceinline__ float kb_sq8(uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
    ss = fmaf(lo, lo, ss);
    ss = fmaf(hi, hi, ss);
  }
  return ss;
}

// The largest squared norm of key rows [c R, min(rows, (c + 1) R)) of head bh (R = ceil(rows / C)),
// NaN-propagating; valid in thread 0 of the block. Every thread of the block calls it.
template <int D>
__device__ __forceinline__ float kb_block_max_sq(const __nv_bfloat16* __restrict__ k, int64_t rows, int C, int c,
                                                 int bh) {
  constexpr int LPR = D / 8;     // lanes per key row, 16 bytes each
  constexpr int RPW = 32 / LPR;  // key rows per warp step
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, part = lane % LPR;
  const int64_t R = (rows + C - 1) / C;
  const int64_t r0 = (int64_t)c * R, r1 = min(rows, r0 + R);
  const uint4* kb = reinterpret_cast<const uint4*>(k + (int64_t)bh * rows * D);
  float best = 0.f;
  // warp-uniform trip count: every lane runs every step and shuffles
  for (int64_t rw = r0 + (int64_t)warp * RPW; rw < r1; rw += (int64_t)(KB_THREADS / 32) * RPW) {
    const int64_t r = rw + sub;
    float ss = 0.f;
    if (r < r1) ss = kb_sq8(kb[r * (D / 8) + part]);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    best = kb_max(best, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) best = kb_max(best, __shfl_xor_sync(0xffffffffu, best, off));
  __shared__ float s_best[KB_THREADS / 32];
  if (lane == 0) s_best[warp] = best;
  __syncthreads();
  float b = 0.f;
  if (threadIdx.x == 0)
    for (int w = 0; w < KB_THREADS / 32; ++w) b = kb_max(b, s_best[w]);
  return b;
}

// Grids are one-dimensional (any number of heads): block i takes chunk i % C of head i / C.
template <int D>
__global__ void __launch_bounds__(KB_THREADS) key_norm_chunk_kernel(const __nv_bfloat16* __restrict__ k, int64_t rows,
                                                                    int C, void* o, int64_t o_row_bytes) {
  const int c = (int)(blockIdx.x % (unsigned)C), bh = (int)(blockIdx.x / (unsigned)C);
  const float b = kb_block_max_sq<D>(k, rows, C, c, bh);
  if (threadIdx.x == 0)
    *reinterpret_cast<float*>(static_cast<char*>(o) + ((int64_t)bh * rows + c) * o_row_bytes) = sqrtf(b);
}

// kmax[bh] = max(kmax[bh], largest key norm of chunk c); kmax starts at +0. A NaN becomes +inf,
// so that the bound of a head with a non-finite key is +inf whatever the NaN's sign bit.
template <int D>
__global__ void __launch_bounds__(KB_THREADS) key_norm_max_kernel(const __nv_bfloat16* __restrict__ k, int64_t rows,
                                                                  int C, float* __restrict__ kmax) {
  const int c = (int)(blockIdx.x % (unsigned)C), bh = (int)(blockIdx.x / (unsigned)C);
  const float b = kb_block_max_sq<D>(k, rows, C, c, bh);
  if (threadIdx.x == 0) {
    const float n = (b != b) ? INFINITY : sqrtf(b);
    atomicMax(reinterpret_cast<int*>(kmax + bh), __float_as_int(n));
  }
}

// Block i writes part i % G of head i / G's lse slots.
__global__ void __launch_bounds__(KB_THREADS) key_norm_spread_kernel(const void* o, int64_t o_row_bytes, int64_t rows,
                                                                     int C, int G, float* __restrict__ lse) {
  const int bh = (int)(blockIdx.x / (unsigned)G), part = (int)(blockIdx.x % (unsigned)G);
  __shared__ float s_kmax;
  if (threadIdx.x < 32) {
    float b = 0.f;
    for (int c = threadIdx.x; c < C; c += 32)
      b = kb_max(b, *reinterpret_cast<const float*>(static_cast<const char*>(o) + ((int64_t)bh * rows + c) * o_row_bytes));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) b = kb_max(b, __shfl_xor_sync(0xffffffffu, b, off));
    if (threadIdx.x == 0) s_kmax = b;
  }
  __syncthreads();
  const float kmax = s_kmax;
  float* dst = lse + (int64_t)bh * rows;
  for (int64_t r = (int64_t)part * KB_THREADS + threadIdx.x; r < rows; r += (int64_t)G * KB_THREADS)
    dst[r] = kmax;
}

}  // namespace ra
