// attn_simt.cuh -- fp32 ring-attention forward on the CUDA cores.
//
// fp32 inputs must match the definition within 1e-5 (the glossary's 4-device toy check),
// which rules out tensor-core tf32. One warp owns one query row of one virtual ring
// position and walks the same ring order as the tensor-core kernel ([BLOG]
// ring_attention_forward: position (p - s) mod P at step s), 32 keys at a time:
// each lane scores one key (full-d dot product in fp32), the warp reduces the group max,
// and the running state (m, l, o) is updated with expf ([BLOG] blockwise_attention;
// [CARD] online softmax). Lane e owns output columns e, e + 32, e + 64, e + 96.
#pragma once

#include "common.cuh"

namespace ra {

constexpr int SIMT_WARPS = 4;
constexpr int SIMT_DMAX = 128;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// grid: x = ceil(rows per position / SIMT_WARPS), y = P, z = B*H.
__global__ void __launch_bounds__(SIMT_WARPS * 32)
attn_fwd_simt_f32_kernel(const Plan pl, int64_t rows_per_pos) {
  __shared__ float sq[SIMT_WARPS][SIMT_DMAX];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t li = (int64_t)blockIdx.x * SIMT_WARPS + warp;  // local query row of the position
  const int p = blockIdx.y;
  const int bh = blockIdx.z;
  if (li >= rows_per_pos) return;  // whole warp exits together
  const int d = pl.d;
  const int si = (int)(li / pl.q_seg_len);
  const Seg qs = segment_of(pl.layout, pl.P, pl.q_seg_len, p, si);
  const int64_t qrow = qs.row0 + qs.stride * (li - (int64_t)si * pl.q_seg_len);
  if (!in_bounds(qrow < pl.q_rows && bh < pl.BH)) return;  // whole warp: qrow is warp-uniform
  const int64_t tq = pl.q_tok0 + pl.q_tok_stride * qrow;
  const float* qp = static_cast<const float*>(pl.q) + ((int64_t)bh * pl.q_rows + qrow) * d;
  const float* kb = static_cast<const float*>(pl.k) + (int64_t)bh * pl.k_rows * d;
  const float* vb = static_cast<const float*>(pl.v) + (int64_t)bh * pl.k_rows * d;
  for (int e = lane; e < d; e += 32) sq[warp][e] = qp[e];
  __syncwarp();

  float m = -INFINITY, l = 0.f;
  float acc[SIMT_DMAX / 32];
#pragma unroll
  for (int t = 0; t < SIMT_DMAX / 32; ++t) acc[t] = 0.f;

  const int nks = num_segments(pl.layout);
  for (int s = 0; s < pl.P; ++s) {
    int c = p - s;
    if (c < 0) c += pl.P;
    for (int sk = 0; sk < nks; ++sk) {
      const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
      const int64_t nvis = visible_prefix(pl, ks, tq);
      for (int64_t j0 = 0; j0 < nvis; j0 += 32) {
        const int64_t j = j0 + lane;
        const int64_t krow = ks.row0 + ks.stride * j;
        const bool vis = j < nvis && in_bounds(krow < pl.k_rows) &&
                         (!pl.causal || pl.k_tok0 + pl.k_tok_stride * krow <= tq);
        float sc = -INFINITY;
        if (vis) {
          const float* kp = kb + krow * d;
          float dot = 0.f;
          for (int e = 0; e < d; ++e) dot = fmaf(sq[warp][e], kp[e], dot);
          sc = dot * pl.scale;
        }
        const float m_new = fmaxf(m, warp_max(sc));
        if (m_new == -INFINITY) continue;  // nothing visible yet
        const float corr = expf(m - m_new);
        const float pj = vis ? expf(sc - m_new) : 0.f;
        l = l * corr + warp_sum(pj);
#pragma unroll
        for (int t = 0; t < SIMT_DMAX / 32; ++t) acc[t] *= corr;
        const int64_t nj = min((int64_t)32, nvis - j0);
        for (int jj = 0; jj < nj; ++jj) {
          const float pb = __shfl_sync(0xffffffffu, pj, jj);
          if (pb == 0.f) continue;  // uniform across the warp
          const float* vp = vb + (ks.row0 + ks.stride * (j0 + jj)) * d;
#pragma unroll
          for (int t = 0; t < SIMT_DMAX / 32; ++t) {
            const int e = lane + 32 * t;
            if (e < d) acc[t] = fmaf(pb, vp[e], acc[t]);
          }
        }
        m = m_new;
      }
    }
  }
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  const float lse_row = l > 0.f ? m + logf(l) : -INFINITY;
  const int64_t orow = (int64_t)bh * pl.q_rows + qrow;
  float* op = static_cast<float*>(pl.o) + orow * d;
  // Folding into a running state: every lane reads the state's lse before any lane writes it.
  FoldWeights fw{lse_row, 0.f, 1.f};
  if (pl.fold) {
    fw = fold_weights(pl.lse[orow], lse_row);
    __syncwarp();
  }
#pragma unroll
  for (int t = 0; t < SIMT_DMAX / 32; ++t) {
    const int e = lane + 32 * t;
    if (e < d) {
      const float o_new = acc[t] * inv_l;
      op[e] = pl.fold ? fmaf(fw.w_new, o_new, fmaf(fw.w_state, op[e], 0.f)) : o_new;
    }
  }
  if (lane == 0 && pl.lse != nullptr) pl.lse[orow] = fw.L;
}

// Writes the empty state (O = 0, lse = -inf) for every row: ra_partial with Lk == 0 (the
// folding variant leaves the running state as it is instead).
__global__ void fill_empty_kernel(float* o, float* lse, int64_t rows, int d) {
  const int64_t n = rows * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    o[i] = 0.f;
    if (i % d == 0) lse[i / d] = -INFINITY;
  }
}

}  // namespace ra
