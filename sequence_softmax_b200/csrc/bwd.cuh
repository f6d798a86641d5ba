// bwd.cuh -- backward pass of ring attention: the problem plan, the key-tile / query-tile
// walk, the row term D, helpers of the tensor-core kernels and the fp32 CUDA-core kernels.
//
// Gradients of O = softmax(S) V with S = Q K^T * scale ([BLOG] ring_attention_backward):
//   P = exp(S - lse)            recomputed from the forward's log-sum-exp, no max pass
//   dV = P^T dO                 dP = dO V^T
//   D_i = sum_e dO_ie O_ie      (= sum_j P_ij dP_ij)
//   dS = P * (dP - D) * scale   dQ = dS K      dK = dS^T Q
// with the causal mask of the forward (key token j visible to query token i iff j <= i),
// which that listing leaves out. In the ring, position p keeps Q_p, dO_p, O_p and lse_p;
// at step s it receives KV chunk (p - s) mod P, adds dS K to its own dQ_p and hands the
// chunk's dK, dV contributions back to the chunk's owner, where they are summed (the
// listing's reduce to a per-rank root is read as that sum). Equivalently, KV chunk c meets
// the query positions c, c + 1, ... (mod P) in turn: that is the order the kernels here walk.
#pragma once

#include "common.cuh"
#include "attn_simt.cuh"

namespace ra {

struct BwdPlan {
  const void* q;
  const void* k;
  const void* v;
  const void* d_o;
  const float* lse;     // [BH, q_rows] natural-log lse of the forward
  const float* delta;   // [BH, q_rows] D = rowsum(dO * O)
  void* dq;             // [BH, q_rows, d]
  void* dk;             // [BH, k_rows, d]
  void* dv;             // [BH, k_rows, d]
  int BH;
  int d;
  int P;
  int layout;
  int causal;
  int accumulate;       // 1: dq, dk, dv are fp32 accumulators (+=); 0: written in the input dtype
  int64_t q_rows, k_rows, q_seg_len, k_seg_len;
  int64_t q_tok0, q_tok_stride, k_tok0, k_tok_stride;
  float scale;
  float scale_log2;
};

constexpr int BWD_TILE = 128;  // keys per key tile and query rows per query tile

// The key tile a CTA owns: tile j0 / 128 of segment `seg` of position c.
struct KTile {
  int c;
  Seg seg;
  int64_t j0;
};

// Units within one head, earliest tokens first: under the causal mask the earliest keys are
// seen by the most queries, so the longest-running CTAs start first.
__device__ __forceinline__ KTile decode_ktile(const BwdPlan& pl, int unit) {
  KTile t;
  const int P = pl.P;
  const int64_t nkt = (pl.k_seg_len + BWD_TILE - 1) / BWD_TILE;
  int si = 0;
  int64_t jt;
  if (pl.layout == RA_LAYOUT_STRIPED) {
    jt = unit / P;
    t.c = unit % P;
  } else if (pl.layout == RA_LAYOUT_ZIGZAG) {
    const int gc = (int)(unit / nkt);  // global chunk
    jt = unit % nkt;
    if (gc < P) { t.c = gc; si = 0; } else { t.c = 2 * P - 1 - gc; si = 1; }
  } else {
    t.c = (int)(unit / nkt);
    jt = unit % nkt;
  }
  t.seg = segment_of(pl.layout, P, pl.k_seg_len, t.c, si);
  t.j0 = jt * BWD_TILE;
  return t;
}

__device__ __forceinline__ int64_t ktile_token_min(const BwdPlan& pl, const KTile& kt) {
  return pl.k_tok0 + pl.k_tok_stride * (kt.seg.row0 + kt.seg.stride * kt.j0);
}

// First local row of query segment qs that sees a key of token >= tk_min (causal), else 0.
__host__ __device__ __forceinline__ int64_t first_seeing_row(const BwdPlan& pl, const Seg& qs, int64_t tk_min) {
  if (!pl.causal) return 0;
  const int64_t tq0 = pl.q_tok0 + pl.q_tok_stride * qs.row0;
  const int64_t tqs = pl.q_tok_stride * qs.stride;
  if (tk_min <= tq0) return 0;
  return (tk_min - tq0 + tqs - 1) / tqs;
}

// Calls f(qs, i0) for every 128-row query tile (local rows i0 .. i0 + 127 of segment qs)
// that can see a key of the tile, in ring order: positions c, c + 1, ... (mod P).
// Stops when f returns false.
template <class F>
__device__ __forceinline__ void walk_q_tiles(const BwdPlan& pl, const KTile& kt, F&& f) {
  const int64_t tk_min = ktile_token_min(pl, kt);
  const int nqs = num_segments(pl.layout);
  for (int s = 0; s < pl.P; ++s) {
    int p = kt.c + s;
    if (p >= pl.P) p -= pl.P;
    for (int si = 0; si < nqs; ++si) {
      const Seg qs = segment_of(pl.layout, pl.P, pl.q_seg_len, p, si);
      const int64_t first = first_seeing_row(pl, qs, tk_min);
      if (first >= qs.count) continue;
      const int64_t ntile = (qs.count + BWD_TILE - 1) / BWD_TILE;
      for (int64_t qt = first / BWD_TILE; qt < ntile; ++qt)
        if (!f(qs, qt * BWD_TILE)) return;
    }
  }
}

// ------------------------------------------------------------------------------------
// D_i = sum_e dO_ie O_ie, one group of 8 lanes per row.
// ------------------------------------------------------------------------------------
constexpr int DELTA_THREADS = 256;

template <bool BF16>
__global__ void __launch_bounds__(DELTA_THREADS)
bwd_delta_kernel(const void* __restrict__ o, const void* __restrict__ d_o, int64_t rows, int d,
                 float* __restrict__ delta) {
  const int g = threadIdx.x & 7;
  const int64_t groups = (int64_t)gridDim.x * (DELTA_THREADS / 8);
  for (int64_t r = (int64_t)blockIdx.x * (DELTA_THREADS / 8) + (threadIdx.x >> 3); r < rows; r += groups) {
    float acc = 0.f;
    if (BF16) {
      // d is a multiple of 8: 16-byte chunks of 8 bf16
      const uint4* a = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + r * d);
      const uint4* b = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(d_o) + r * d);
      for (int c = g; c < d / 8; c += 8) {
        const uint4 x = __ldcs(a + c), y = __ldcs(b + c);
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[t]));
          const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[t]));
          acc = fmaf(xf.x, yf.x, acc);
          acc = fmaf(xf.y, yf.y, acc);
        }
      }
    } else {
      const float* a = static_cast<const float*>(o) + r * d;
      const float* b = static_cast<const float*>(d_o) + r * d;
      for (int e = g; e < d; e += 8) acc = fmaf(a[e], b[e], acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (g == 0) delta[r] = acc;
  }
}

// ------------------------------------------------------------------------------------
// Helpers of the tensor-core backward kernels (one thread = one TMEM lane, 64 columns).
// ------------------------------------------------------------------------------------

// p[j] = exp2(s_j * sl2 + nl2_j) for the 64 fp32 TMEM columns at taddr, where nl2_j is
// -lse_j log2(e): nl2col[j] (a per-column value in shared memory) when PER_COL, else nl2row.
// With `masked` (warp-uniform), columns outside [lo, hi) are 0. Paired f32x2 FMAs form the
// exponents; MUFU ex2 evaluates them.
template <bool PER_COL>
__device__ __forceinline__ void bwd_exp_row64(uint32_t taddr, const float* nl2col, float nl2row, float sl2, bool masked,
                                              int lo, int hi, float (&p)[64]) {
  uint32_t sr[64];
  RA_TMEM_LD32(taddr, sr);
  RA_TMEM_LD32(taddr + 32, (sr + 32));
  tmem_wait_ld();
  RA_REG_FENCE32(sr);
  RA_REG_FENCE32((sr + 32));
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
#pragma unroll
  for (int j = 0; j < 64; j += 4) {
    float4 L = make_float4(nl2row, nl2row, nl2row, nl2row);
    if (PER_COL) L = *reinterpret_cast<const float4*>(nl2col + j);
    float x0, x1, x2, x3;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), sl2x2, f2_pack(L.x, L.y)), x0, x1);
    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), sl2x2, f2_pack(L.z, L.w)), x2,
              x3);
    p[j + 0] = ex2_approx(x0);
    p[j + 1] = ex2_approx(x1);
    p[j + 2] = ex2_approx(x2);
    p[j + 3] = ex2_approx(x3);
  }
  if (masked) {
#pragma unroll
    for (int j = 0; j < 64; ++j) p[j] = (j >= lo && j < hi) ? p[j] : 0.f;
  }
}

// ds = bf16 pairs of p_j (dP_j scale + nds_j) = p_j (dP_j - D_j) scale for 64 fp32 dP
// values dr; nds_j = -D_j scale is ndscol[j] (per column, shared memory) when PER_COL, else
// ndsrow. Two paired f32x2 operations per two scores.
template <bool PER_COL>
__device__ __forceinline__ void bwd_ds_regs64(const uint32_t (&dr)[64], const float (&p)[64], const float* ndscol,
                                              float ndsrow, float scale, uint32_t (&ds)[32]) {
  const uint64_t sc2 = f2_pack(scale, scale), z2 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 64; j += 4) {
    float4 N = make_float4(ndsrow, ndsrow, ndsrow, ndsrow);
    if (PER_COL) N = *reinterpret_cast<const float4*>(ndscol + j);
    const uint64_t t01 = f2_fma(f2_pack(__uint_as_float(dr[j]), __uint_as_float(dr[j + 1])), sc2, f2_pack(N.x, N.y));
    const uint64_t t23 =
        f2_fma(f2_pack(__uint_as_float(dr[j + 2]), __uint_as_float(dr[j + 3])), sc2, f2_pack(N.z, N.w));
    float a, b, c, d;
    f2_unpack(f2_fma(f2_pack(p[j], p[j + 1]), t01, z2), a, b);
    f2_unpack(f2_fma(f2_pack(p[j + 2], p[j + 3]), t23, z2), c, d);
    ds[j / 2] = pack_bf16x2(a, b);
    ds[j / 2 + 1] = pack_bf16x2(c, d);
  }
}

// As bwd_ds_regs64, with the 64 dP values loaded from the TMEM columns at taddr.
template <bool PER_COL>
__device__ __forceinline__ void bwd_ds_row64(uint32_t taddr, const float (&p)[64], const float* ndscol, float ndsrow,
                                             float scale, uint32_t (&ds)[32]) {
  uint32_t dr[64];
  RA_TMEM_LD32(taddr, dr);
  RA_TMEM_LD32(taddr + 32, (dr + 32));
  tmem_wait_ld();
  RA_REG_FENCE32(dr);
  RA_REG_FENCE32((dr + 32));
  bwd_ds_regs64<PER_COL>(dr, p, ndscol, ndsrow, scale, ds);
}

// bwd_exp_row64 for the 32 columns [OFF, OFF + 32) of the thread's 64, loaded from the TMEM
// columns at taddr + OFF; fills p[OFF .. OFF + 32).
template <bool PER_COL, int OFF>
__device__ __forceinline__ void bwd_exp_part32(uint32_t taddr, const float* nl2col, float nl2row, float sl2,
                                               bool masked, int lo, int hi, float (&p)[64]) {
  uint32_t sr[32];
  RA_TMEM_LD32(taddr + OFF, sr);
  tmem_wait_ld();
  RA_REG_FENCE32(sr);
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    float4 L = make_float4(nl2row, nl2row, nl2row, nl2row);
    if (PER_COL) L = *reinterpret_cast<const float4*>(nl2col + OFF + j);
    float x0, x1, x2, x3;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), sl2x2, f2_pack(L.x, L.y)), x0, x1);
    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), sl2x2, f2_pack(L.z, L.w)), x2,
              x3);
    p[OFF + j + 0] = ex2_approx(x0);
    p[OFF + j + 1] = ex2_approx(x1);
    p[OFF + j + 2] = ex2_approx(x2);
    p[OFF + j + 3] = ex2_approx(x3);
  }
  if (masked) {
#pragma unroll
    for (int j = OFF; j < OFF + 32; ++j) p[j] = (j >= lo && j < hi) ? p[j] : 0.f;
  }
}

// bwd_ds_row64 for the 32 columns [OFF, OFF + 32): 16 bf16 pairs from the dP columns at
// taddr + OFF and p[OFF .. OFF + 32).
template <bool PER_COL, int OFF>
__device__ __forceinline__ void bwd_ds_part32(uint32_t taddr, const float (&p)[64], const float* ndscol,
                                              float ndsrow, float scale, uint32_t (&ds)[16]) {
  uint32_t dr[32];
  RA_TMEM_LD32(taddr + OFF, dr);
  tmem_wait_ld();
  RA_REG_FENCE32(dr);
  const uint64_t sc2 = f2_pack(scale, scale), z2 = f2_pack(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    float4 N = make_float4(ndsrow, ndsrow, ndsrow, ndsrow);
    if (PER_COL) N = *reinterpret_cast<const float4*>(ndscol + OFF + j);
    const uint64_t t01 = f2_fma(f2_pack(__uint_as_float(dr[j]), __uint_as_float(dr[j + 1])), sc2, f2_pack(N.x, N.y));
    const uint64_t t23 =
        f2_fma(f2_pack(__uint_as_float(dr[j + 2]), __uint_as_float(dr[j + 3])), sc2, f2_pack(N.z, N.w));
    float a, b, c, d;
    f2_unpack(f2_fma(f2_pack(p[OFF + j], p[OFF + j + 1]), t01, z2), a, b);
    f2_unpack(f2_fma(f2_pack(p[OFF + j + 2], p[OFF + j + 3]), t23, z2), c, d);
    ds[j / 2] = pack_bf16x2(a, b);
    ds[j / 2 + 1] = pack_bf16x2(c, d);
  }
}

// ceil(num / den) clamped to [0, cap] for num > 0, den >= 1, with a 32-bit division when the
// result is below the cap (the per-tile causal bound; 64-bit division is slow on the GPU).
__device__ __forceinline__ int ceil_div_clamped(int64_t num, int64_t den, int cap) {
  if (num > (int64_t)cap * den) return cap;
  if (den < (1 << 23)) return (int)(((uint32_t)num + (uint32_t)den - 1u) / (uint32_t)den);
  return (int)((num + den - 1) / den);
}

// Epilogue of an fp32 TMEM accumulator row: NC columns at taddr (all lanes of the warp load;
// `have` false means the accumulator was never written and reads as 0). Valid rows are
// written to dst + off as bf16, or added to the fp32 values there when `accumulate`.
template <int NC>
__device__ __forceinline__ void bwd_store_acc_row(uint32_t taddr, bool have, bool valid, void* dst, int64_t off,
                                                  bool accumulate) {
#pragma unroll
  for (int cc = 0; cc < NC / 32; ++cc) {
    uint32_t r[32];
    if (have) {
      RA_TMEM_LD32(taddr + cc * 32, r);
      tmem_wait_ld();
      RA_REG_FENCE32(r);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = 0u;
    }
    if (!valid) continue;
    if (accumulate) {
      float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(dst) + off + cc * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 a = o4[j];
        a.x += __uint_as_float(r[4 * j]);
        a.y += __uint_as_float(r[4 * j + 1]);
        a.z += __uint_as_float(r[4 * j + 2]);
        a.w += __uint_as_float(r[4 * j + 3]);
        o4[j] = a;
      }
    } else {
      uint4* o16 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + off + cc * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        o16[j] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                            pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                            pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                            pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])));
    }
  }
}

// ------------------------------------------------------------------------------------
// fp32 backward on the CUDA cores (the fp32 path must match the definition within 1e-5,
// which rules out tf32 tensor cores). Two kernels, no atomics:
//   dkdv: one warp per key row, walking the query rows that see it in ring order;
//         lane l scores query row i0 + l (full-d dot products), then the warp
//         accumulates dV_j += P_ij dO_i and dK_j += dS_ij Q_i over those 32 rows.
//   dq:   one warp per query row, walking the visible keys in the forward's ring order.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ float bwd_prob(float s_scaled, float lse) {
  return lse == -INFINITY ? 0.f : expf(s_scaled - lse);
}

// grid: x = ceil(key rows per position / SIMT_WARPS), y = P, z = B*H.
__global__ void __launch_bounds__(SIMT_WARPS * 32)
bwd_dkdv_simt_f32_kernel(const BwdPlan pl, int64_t rows_per_pos) {
  __shared__ float sk[SIMT_WARPS][SIMT_DMAX];
  __shared__ float sv[SIMT_WARPS][SIMT_DMAX];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t lj = (int64_t)blockIdx.x * SIMT_WARPS + warp;
  const int c = blockIdx.y;
  const int bh = blockIdx.z;
  if (lj >= rows_per_pos) return;
  const int d = pl.d;
  const int sk_i = (int)(lj / pl.k_seg_len);
  const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk_i);
  const int64_t krow = ks.row0 + ks.stride * (lj - (int64_t)sk_i * pl.k_seg_len);
  if (!in_bounds(krow < pl.k_rows && bh < pl.BH)) return;  // whole warp: krow is warp-uniform
  const int64_t tk = pl.k_tok0 + pl.k_tok_stride * krow;
  const float* kp = static_cast<const float*>(pl.k) + ((int64_t)bh * pl.k_rows + krow) * d;
  const float* vp = static_cast<const float*>(pl.v) + ((int64_t)bh * pl.k_rows + krow) * d;
  for (int e = lane; e < d; e += 32) {
    sk[warp][e] = kp[e];
    sv[warp][e] = vp[e];
  }
  __syncwarp();
  const float* qb = static_cast<const float*>(pl.q) + (int64_t)bh * pl.q_rows * d;
  const float* ob = static_cast<const float*>(pl.d_o) + (int64_t)bh * pl.q_rows * d;
  const float* lb = pl.lse + (int64_t)bh * pl.q_rows;
  const float* db = pl.delta + (int64_t)bh * pl.q_rows;
  float dk[SIMT_DMAX / 32], dv[SIMT_DMAX / 32];
#pragma unroll
  for (int t = 0; t < SIMT_DMAX / 32; ++t) dk[t] = dv[t] = 0.f;

  const int nqs = num_segments(pl.layout);
  for (int s = 0; s < pl.P; ++s) {
    int p = c + s;
    if (p >= pl.P) p -= pl.P;
    for (int si = 0; si < nqs; ++si) {
      const Seg qs = segment_of(pl.layout, pl.P, pl.q_seg_len, p, si);
      for (int64_t i0 = first_seeing_row(pl, qs, tk); i0 < qs.count; i0 += 32) {
        const int64_t i = i0 + lane;
        const int64_t qrow = qs.row0 + qs.stride * i;
        float pij = 0.f, dsij = 0.f;
        if (i < qs.count && in_bounds(qrow < pl.q_rows) && (!pl.causal || tk <= pl.q_tok0 + pl.q_tok_stride * qrow)) {
          const float* qp = qb + qrow * d;
          const float* op = ob + qrow * d;
          float dot = 0.f, dpd = 0.f;
          for (int e = 0; e < d; ++e) {
            dot = fmaf(qp[e], sk[warp][e], dot);
            dpd = fmaf(op[e], sv[warp][e], dpd);
          }
          pij = bwd_prob(dot * pl.scale, lb[qrow]);
          dsij = pij * (dpd - db[qrow]) * pl.scale;
        }
        const int64_t nj = min((int64_t)32, qs.count - i0);
        for (int jj = 0; jj < nj; ++jj) {
          const float pb = __shfl_sync(0xffffffffu, pij, jj);
          const float db2 = __shfl_sync(0xffffffffu, dsij, jj);
          if (pb == 0.f && db2 == 0.f) continue;  // uniform across the warp
          const int64_t r = qs.row0 + qs.stride * (i0 + jj);
          const float* qp = qb + r * d;
          const float* op = ob + r * d;
#pragma unroll
          for (int t = 0; t < SIMT_DMAX / 32; ++t) {
            const int e = lane + 32 * t;
            if (e < d) {
              dv[t] = fmaf(pb, op[e], dv[t]);
              dk[t] = fmaf(db2, qp[e], dk[t]);
            }
          }
        }
      }
    }
  }
  float* dkp = static_cast<float*>(pl.dk) + ((int64_t)bh * pl.k_rows + krow) * d;
  float* dvp = static_cast<float*>(pl.dv) + ((int64_t)bh * pl.k_rows + krow) * d;
#pragma unroll
  for (int t = 0; t < SIMT_DMAX / 32; ++t) {
    const int e = lane + 32 * t;
    if (e < d) {
      if (pl.accumulate) {
        dkp[e] += dk[t];
        dvp[e] += dv[t];
      } else {
        dkp[e] = dk[t];
        dvp[e] = dv[t];
      }
    }
  }
}

// grid: x = ceil(query rows per position / SIMT_WARPS), y = P, z = B*H.
__global__ void __launch_bounds__(SIMT_WARPS * 32)
bwd_dq_simt_f32_kernel(const BwdPlan pl, int64_t rows_per_pos) {
  __shared__ float sq[SIMT_WARPS][SIMT_DMAX];
  __shared__ float so[SIMT_WARPS][SIMT_DMAX];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t li = (int64_t)blockIdx.x * SIMT_WARPS + warp;
  const int p = blockIdx.y;
  const int bh = blockIdx.z;
  if (li >= rows_per_pos) return;
  const int d = pl.d;
  const int si = (int)(li / pl.q_seg_len);
  const Seg qs = segment_of(pl.layout, pl.P, pl.q_seg_len, p, si);
  const int64_t qrow = qs.row0 + qs.stride * (li - (int64_t)si * pl.q_seg_len);
  if (!in_bounds(qrow < pl.q_rows && bh < pl.BH)) return;  // whole warp: qrow is warp-uniform
  const int64_t tq = pl.q_tok0 + pl.q_tok_stride * qrow;
  const float* qp = static_cast<const float*>(pl.q) + ((int64_t)bh * pl.q_rows + qrow) * d;
  const float* op = static_cast<const float*>(pl.d_o) + ((int64_t)bh * pl.q_rows + qrow) * d;
  for (int e = lane; e < d; e += 32) {
    sq[warp][e] = qp[e];
    so[warp][e] = op[e];
  }
  __syncwarp();
  const float lse = pl.lse[(int64_t)bh * pl.q_rows + qrow];
  const float Di = pl.delta[(int64_t)bh * pl.q_rows + qrow];
  const float* kb = static_cast<const float*>(pl.k) + (int64_t)bh * pl.k_rows * d;
  const float* vb = static_cast<const float*>(pl.v) + (int64_t)bh * pl.k_rows * d;
  float dq[SIMT_DMAX / 32];
#pragma unroll
  for (int t = 0; t < SIMT_DMAX / 32; ++t) dq[t] = 0.f;

  // The key-side visibility test of the forward (keys of token <= tq), on the key plan.
  Plan kp{};
  kp.causal = pl.causal;
  kp.k_tok0 = pl.k_tok0;
  kp.k_tok_stride = pl.k_tok_stride;
  const int nks = num_segments(pl.layout);
  for (int s = 0; s < pl.P; ++s) {
    int c = p - s;
    if (c < 0) c += pl.P;
    for (int sk_i = 0; sk_i < nks; ++sk_i) {
      const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk_i);
      const int64_t nvis = visible_prefix(kp, ks, tq);
      for (int64_t j0 = 0; j0 < nvis; j0 += 32) {
        const int64_t j = j0 + lane;
        const int64_t krow = ks.row0 + ks.stride * j;
        float dsij = 0.f;
        if (j < nvis && in_bounds(krow < pl.k_rows) && (!pl.causal || pl.k_tok0 + pl.k_tok_stride * krow <= tq)) {
          const float* kr = kb + krow * d;
          const float* vr = vb + krow * d;
          float dot = 0.f, dpd = 0.f;
          for (int e = 0; e < d; ++e) {
            dot = fmaf(sq[warp][e], kr[e], dot);
            dpd = fmaf(so[warp][e], vr[e], dpd);
          }
          dsij = bwd_prob(dot * pl.scale, lse) * (dpd - Di) * pl.scale;
        }
        const int64_t nj = min((int64_t)32, nvis - j0);
        for (int jj = 0; jj < nj; ++jj) {
          const float db2 = __shfl_sync(0xffffffffu, dsij, jj);
          if (db2 == 0.f) continue;
          const float* kr = kb + (ks.row0 + ks.stride * (j0 + jj)) * d;
#pragma unroll
          for (int t = 0; t < SIMT_DMAX / 32; ++t) {
            const int e = lane + 32 * t;
            if (e < d) dq[t] = fmaf(db2, kr[e], dq[t]);
          }
        }
      }
    }
  }
  float* dqp = static_cast<float*>(pl.dq) + ((int64_t)bh * pl.q_rows + qrow) * d;
#pragma unroll
  for (int t = 0; t < SIMT_DMAX / 32; ++t) {
    const int e = lane + 32 * t;
    if (e < d) {
      if (pl.accumulate) dqp[e] += dq[t];
      else dqp[e] = dq[t];
    }
  }
}

}  // namespace ra
