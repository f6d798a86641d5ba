// attn_tc.cuh -- bf16 ring-attention forward on the 5th-generation tensor cores (sm_100a).
//
// One CTA owns a query block of two 128-row tiles of one virtual ring position and walks
// that position's KV tiles in ring order ([BLOG] ring_attention_forward: position p visits
// position (p - s) mod P at step s; [GLOSSARY] "How Ring Attention works"), folding each
// 128-key tile into a running online-softmax state (m, l, o) ([BLOG] blockwise_attention;
// [CARD] online softmax). Causal tiles wholly in the future are never visited; tiles that
// straddle the diagonal are masked elementwise ([BLOG] ring_attention_causal_step).
//
// Warp roles (384 threads, 3 warpgroups; setmaxnreg moves registers to the softmax):
//   warps 0-3  softmax for query tile 0 (thread i owns row i = TMEM lane i)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q tiles once, then K/V tiles into an NSTAGE ring of shared
//              memory stages (the single-GPU counterpart of the ring's overlap of the next
//              chunk's transfer with the current chunk's compute)
//   warp  9    MMA issuer (one thread): S_t = Q_t K^T (both operands from 128B-swizzled
//              shared memory) and O_t += P_t V (P from tensor memory, V from shared memory)
//   warps 10-11 idle
//
// Tensor memory (512 columns x 128 lanes of fp32): S_0 | S_1 | O_0 | O_1. P_t (bf16 pairs)
// overwrites the first 64 columns of S_t. The MMA warp issues, per KV tile n,
//   PV_0(n-1), S_0(n), PV_1(n-1), S_1(n)
// so the tensor core computes one tile's GEMMs while the other tile's softmax runs. MMAs
// issued by one thread execute in order, so S_t(n) cannot overwrite P_t(n-1) before
// PV_t(n-1) has read it, and the commit that signals S_t(n) also covers PV_t(n-1): when a
// softmax warpgroup sees S_t(n), its O_t is stable and may be rescaled.
//
// Rescaling is conditional: the running max used for exponentials only moves when the
// true row max exceeds it by more than RESCALE_LOG2 (in log2 units); until then exp2 values
// stay <= 2^RESCALE_LOG2 and l and O keep sharing the same stale max, so the result is
// exact up to rounding.
//
// With a key-norm bound (keybound.cuh), a warp also skips the row max of a tile when, for
// each of its rows, |q| max|k| scale log2(e) <= m + MAXSKIP_LOG2: no score of the tile can then
// take an exponential above 2^MAXSKIP_LOG2, and m is kept as it is.
#pragma once

#include "common.cuh"

namespace ra {

constexpr int TC_BM = 128;          // query rows per tile
constexpr int TC_BN = 128;          // keys per KV tile
constexpr int TC_THREADS = 384;     // 3 warpgroups
constexpr int TC_REGS_SOFTMAX = 216;  // per thread, after setmaxnreg (launch: 168)
constexpr int TC_REGS_OTHER = 72;     // 2 x 216 + 72 = 504 = 168 * 384 / 128
constexpr int TC_WARP_PRODUCER = 8;
constexpr int TC_WARP_MMA = 9;
constexpr int TC_TMEM_COLS = 512;
constexpr float RESCALE_LOG2 = 8.0f;
// Exponentials stay <= 2^MAXSKIP_LOG2 on tiles whose max is skipped: l <= 2^55 for 2^31 keys,
// and O stays finite in fp32 while |V| < 2^72.
constexpr float MAXSKIP_LOG2 = 24.0f;

template <int D>
struct TcCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int BOX_BYTES = TC_BM * 64 * 2;         // one TMA box: 128 rows x 64 bf16
  static constexpr int NBOX = D / 64;                      // boxes per tile (d split in 64s)
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;      // one Q, K or V tile
  static constexpr int NSTAGE = (D == 128) ? 4 : 8;        // K/V ring depth (in tiles)
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSTAGE * TILE_BYTES;
  static constexpr int NBAR = 2 + 2 * NSTAGE + 2 + 2 + 2 + 1 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr int COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(TC_BM, TC_BN, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(TC_BM, D, true);
};

// Query block owned by the CTA with index `unit` within its head, heaviest (latest tokens) first.
struct QBlock {
  int p;      // virtual position
  Seg seg;    // the position's segment that holds the block
  int64_t i0; // local row of tile 0 inside the segment
};

__device__ __forceinline__ QBlock decode_unit(const Plan& pl, int unit) {
  QBlock b;
  const int P = pl.P;
  const int64_t nb = (pl.q_seg_len + 2 * TC_BM - 1) / (2 * TC_BM);
  int si = 0;
  int64_t qb;
  if (pl.layout == RA_LAYOUT_STRIPED) {
    qb = nb - 1 - unit / P;
    b.p = P - 1 - unit % P;
  } else if (pl.layout == RA_LAYOUT_ZIGZAG) {
    const int gc = 2 * P - 1 - (int)(unit / nb);  // global chunk, latest first
    qb = nb - 1 - unit % nb;
    if (gc >= P) { b.p = 2 * P - 1 - gc; si = 1; } else { b.p = gc; si = 0; }
  } else {
    b.p = P - 1 - (int)(unit / nb);
    qb = nb - 1 - unit % nb;
  }
  b.seg = segment_of(pl.layout, P, pl.q_seg_len, b.p, si);
  b.i0 = qb * (2 * TC_BM);
  return b;
}

__device__ __forceinline__ int64_t q_token(const Plan& pl, const Seg& s, int64_t i) {
  return pl.q_tok0 + pl.q_tok_stride * (s.row0 + s.stride * i);
}

// P = exp2(s * sl2 - shift) for the 64 scores of keys 64h .. 64h + 63 of one row: P as 32
// bf16 pairs in pk, and the sums of the even and odd pairs added into sum2a / sum2b. The
// exponentials run on the MUFU (ex2.approx); the scale and shift are one paired FMA.
__device__ __forceinline__ void exp_half(const uint32_t (&sr)[TC_BN], int h, uint64_t sl2x2, uint64_t negm2,
                                         uint32_t (&pk)[32], uint64_t& sum2a, uint64_t& sum2b) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint64_t x2 =
        f2_fma(f2_pack(__uint_as_float(sr[h * 64 + 2 * j]), __uint_as_float(sr[h * 64 + 2 * j + 1])), sl2x2, negm2);
    float x0, x1;
    f2_unpack(x2, x0, x1);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    if (j & 1) sum2b = f2_add(sum2b, f2_pack(p0, p1));
    else sum2a = f2_add(sum2a, f2_pack(p0, p1));
    pk[j] = pack_bf16x2(p0, p1);
  }
}

// Maximum of one row's 128 raw scores: eight independent chains of three-input max.
__device__ __forceinline__ float row_max(const uint32_t (&sr)[TC_BN]) {
#define SV(j) __uint_as_float(sr[(j)])
  float mxc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mxc[c] = fmax3(SV(2 * c), SV(2 * c + 1), SV(16 + 2 * c));
#pragma unroll
  for (int j = 32; j < TC_BN; j += 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c) mxc[c] = fmax3(mxc[c], SV(j + 2 * c), SV(j + 2 * c + 1));
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) mxc[c] = fmaxf(mxc[c], SV(17 + 2 * c));
#undef SV
  return fmaxf(fmax3(mxc[0], mxc[1], mxc[2]), fmax3(mxc[3], mxc[4], fmax3(mxc[5], mxc[6], mxc[7])));
}

// O_t *= corr for this thread's row (D columns of fp32 in TMEM), 32 columns at a time.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float corr) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t orr[32];
    RA_TMEM_LD32(tO + cc * 32, orr);
    tmem_wait_ld();
    RA_REG_FENCE32(orr);
#pragma unroll
    for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * corr);
    RA_TMEM_ST32(tO + cc * 32, orr);
  }
}


// Index (0..127) of the last key of KV tile jt of segment (c, sk) that query token tq may
// see: the segment's end and, when causal, the query's own token bound it; -1 if none.
__device__ __forceinline__ int last_visible_key(const Plan& pl, int c, int sk, int jt, int64_t tq) {
  const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
  const int64_t j0 = (int64_t)jt * TC_BN;
  int lim = (int)min((int64_t)TC_BN, ks.count - j0) - 1;
  if (pl.causal) {
    const int64_t tks = pl.k_tok_stride * ks.stride;
    const int64_t tk0 = pl.k_tok0 + pl.k_tok_stride * (ks.row0 + ks.stride * j0);
    const int64_t jl = tq < tk0 ? -1 : (tq - tk0) / tks;
    if (jl < lim) lim = (int)jl;
  }
  return lim;
}

// P ready: this thread's tcgen05.st of P are complete; every softmax thread of the tile
// arrives (one arrival per warp measured slower).
__device__ __forceinline__ void arrive_p_ready(uint32_t bar) {
  tmem_wait_st();
  tc_fence_before_sync();
  mbar_arrive(bar);
}

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Plan pl) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::Q_OFF;
  const uint32_t sKV = sbase + C::KV_OFF;
  const uint32_t bar0 = sbase + C::BAR_OFF;
  auto bar_q_full = [&](int t) { return bar0 + 8u * t; };
  auto bar_kv_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto bar_kv_empty = [&](int s) { return bar0 + 8u * (2 + C::NSTAGE + s); };
  auto bar_s_full = [&](int t) { return bar0 + 8u * (2 + 2 * C::NSTAGE + t); };
  auto bar_p_full = [&](int t) { return bar0 + 8u * (4 + 2 * C::NSTAGE + t); };
  auto bar_o_done = [&](int t) { return bar0 + 8u * (6 + 2 * C::NSTAGE + t); };
  const uint32_t bar_drain = bar0 + 8u * (8 + 2 * C::NSTAGE);
  auto bar_p_half = [&](int t) { return bar0 + 8u * (9 + 2 * C::NSTAGE + t); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Head-major order: the CTAs running at the same time belong to one (batch, head) and
  // walk the same KV chunks in the same ring order, so the K/V tiles they stream are
  // shared through L2 (measured on the 1M-token workload: 86x less DRAM traffic than
  // interleaving heads). Within a head, query blocks go heaviest first.
  const int units_per_head = (int)(gridDim.x / pl.BH);
  const int bh = blockIdx.x / units_per_head;
  const int unit = blockIdx.x % units_per_head;
  const QBlock qb = decode_unit(pl, unit);
  const int64_t q_last = min(qb.i0 + 2 * TC_BM, qb.seg.count) - 1;  // last valid local row
  const int64_t tq_max = q_token(pl, qb.seg, q_last);
  const int nks = num_segments(pl.layout);

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full(0), 1);
    mbar_init(bar_q_full(1), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full(t), 1);
      mbar_init(bar_p_full(t), TC_BM);
      mbar_init(bar_p_half(t), TC_BM);
      mbar_init(bar_o_done(t), 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == TC_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), TC_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TC_WARP_PRODUCER && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Number of KV tiles this block visits (identical walk in every role).
  int T = 0;
  for (int s = 0; s < pl.P; ++s) {
    int c = qb.p - s;
    if (c < 0) c += pl.P;
    for (int sk = 0; sk < nks; ++sk) {
      const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
      T += (int)((visible_prefix(pl, ks, tq_max) + TC_BN - 1) / TC_BN);
    }
  }

  if (warp >= 8) {
    // Warpgroup 2 (TMA producer, MMA issuer, two idle warps) gives registers to the softmax.
    regs_decrease<TC_REGS_OTHER>();
  }
  if (warp == TC_WARP_PRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int qy = (int)(qb.seg.row0 % qb.seg.stride);
      const int64_t qz0 = qb.seg.row0 / qb.seg.stride + qb.i0;
      // the block starts inside its segment and the segment lies inside the tensor
      in_bounds(qb.i0 < qb.seg.count && qb.seg.row0 + qb.seg.stride * (qb.seg.count - 1) < pl.q_rows &&
                bh < pl.BH);
      for (int t = 0; t < 2; ++t) {
        mbar_arrive_expect_tx(bar_q_full(t), C::TILE_BYTES);
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_4d(sQ + t * C::TILE_BYTES + b * C::BOX_BYTES, &tm_q, bar_q_full(t), 64 * b, qy,
                      (int)(qz0 + t * TC_BM), bh);
      }
      uint32_t use = 0;
      bool ok = true;
      for (int s = 0; s < pl.P && ok; ++s) {
        int c = qb.p - s;
        if (c < 0) c += pl.P;
        for (int sk = 0; sk < nks && ok; ++sk) {
          const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
          const int ntiles = (int)((visible_prefix(pl, ks, tq_max) + TC_BN - 1) / TC_BN);
          const int ky = (int)(ks.row0 % ks.stride);
          const int64_t kz0 = ks.row0 / ks.stride;
          for (int jt = 0; jt < ntiles && ok; ++jt) {
            in_bounds((int64_t)jt * TC_BN < ks.count && ks.row0 + ks.stride * (ks.count - 1) < pl.k_rows);
            for (int kv = 0; kv < 2; ++kv, ++use) {
              const int st = use % C::NSTAGE;
              const uint32_t ph = (use / C::NSTAGE) & 1u;
              if (!mbar_wait(bar_kv_empty(st), ph ^ 1u, abort_flag)) { ok = false; break; }
              mbar_arrive_expect_tx(bar_kv_full(st), C::TILE_BYTES);
              const CUtensorMap* map = kv == 0 ? &tm_k : &tm_v;
              for (int b = 0; b < C::NBOX; ++b)
                tma_load_4d(sKV + st * C::TILE_BYTES + b * C::BOX_BYTES, map, bar_kv_full(st), 64 * b, ky,
                            (int)(kz0 + (int64_t)jt * TC_BN), bh);
            }
          }
        }
      }
      // Drain: every load issued must land before the CTA's shared memory goes away.
      const uint32_t first = use > (uint32_t)C::NSTAGE ? use - C::NSTAGE : 0u;
      for (uint32_t u = first; u < use; ++u) mbar_wait_drain(bar_kv_full(u % C::NSTAGE), (u / C::NSTAGE) & 1u);
      mbar_wait_drain(bar_q_full(0), 0);
      mbar_wait_drain(bar_q_full(1), 0);
    }
  } else if (warp == TC_WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (converged) and one elected lane issues: tcgen05.mma
    // issued from a converged warp streams much faster than from a lone diverged thread.
    if (T > 0) {
      const uint32_t tS[2] = {tmem + C::COL_S0, tmem + C::COL_S1};
      const uint32_t tO[2] = {tmem + C::COL_O0, tmem + C::COL_O1};
      // Descriptors are built once; per k-step only the start-address field (the low 14
      // bits, in 16-byte units) moves, by a constant. Addresses stay below 256 KB, so the
      // add never carries into the neighbouring fields.
      const uint32_t hi_sw128 = (1024u >> 4) | (1u << 14) | (2u << 29);  // SBO 1 KB, sm_100 version, 128B swizzle
      const uint32_t lo_q[2] = {((sQ & 0x3FFFFu) >> 4) | (1u << 16),
                                (((sQ + C::TILE_BYTES) & 0x3FFFFu) >> 4) | (1u << 16)};
      const uint32_t lo_k = ((sKV & 0x3FFFFu) >> 4) | (1u << 16);                     // K-major, LBO 16 B
      const uint32_t lo_v = ((sKV & 0x3FFFFu) >> 4) | ((uint32_t)(C::BOX_BYTES >> 4) << 16);  // MN-major, LBO one box
      auto desc = [&](uint32_t lo) { return ((uint64_t)hi_sw128 << 32) | lo; };
      auto issue_s = [&](int t, int st) {
        const uint32_t kb = lo_k + (uint32_t)st * (C::TILE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
          mma_bf16_ss(tS[t], desc(lo_q[t] + off), desc(kb + off), C::IDESC_S, kk > 0);
        }
      };
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
      };
      // PV over keys 64h .. 64h + 63 (k-steps 4h .. 4h + 3).
      auto issue_pv_half = [&](int t, int st, bool acc, int h) {
        const uint32_t vb = lo_v + (uint32_t)st * (C::TILE_BYTES >> 4);
#pragma unroll
        for (int k4 = 0; k4 < TC_BN / 32; ++k4) {
          const int kk = h * (TC_BN / 32) + k4;
          mma_bf16_ts(tO[t], tS[t] + kk * 8, desc(vb + kk * (2048 >> 4)), C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // PV of tile t: waits for each half of P separately.
      auto pv_tile = [&](int t, int st, bool acc, uint32_t parity) {
        if (!wait_all(bar_p_half(t), parity)) return false;
        tc_fence_after_sync();
        if (elect_one()) issue_pv_half(t, st, acc, 0);
        __syncwarp();
        if (!wait_all(bar_p_full(t), parity)) return false;
        tc_fence_after_sync();
        if (elect_one()) issue_pv_half(t, st, acc, 1);
        __syncwarp();
        return true;
      };
      bool ok = wait_all(bar_q_full(0), 0) && wait_all(bar_q_full(1), 0);
      // tile 0: K_0
      if (ok) ok = wait_all(bar_kv_full(0), 0);
      if (ok) {
        tc_fence_after_sync();
        if (elect_one()) {
          issue_s(0, 0);
          tc_commit(bar_s_full(0));
          issue_s(1, 0);
          tc_commit(bar_s_full(1));
          tc_commit(bar_kv_empty(0));
        }
        __syncwarp();
      }
      for (int n = 1; n < T && ok; ++n) {
        const uint32_t uv = 2u * (n - 1) + 1u, uk = 2u * n;
        const int sv = uv % C::NSTAGE, sk = uk % C::NSTAGE;
        const uint32_t pv = (uv / C::NSTAGE) & 1u, pk = (uk / C::NSTAGE) & 1u;
        const uint32_t pp = (uint32_t)(n - 1) & 1u;
        if (!(ok = wait_all(bar_kv_full(sv), pv))) break;
        if (!(ok = pv_tile(0, sv, n - 1 > 0, pp))) break;
        if (!(ok = wait_all(bar_kv_full(sk), pk))) break;
        tc_fence_after_sync();
        if (elect_one()) {
          issue_s(0, sk);
          tc_commit(bar_s_full(0));
        }
        __syncwarp();
        if (!(ok = pv_tile(1, sv, n - 1 > 0, pp))) break;
        if (elect_one()) {
          tc_commit(bar_kv_empty(sv));
          issue_s(1, sk);
          tc_commit(bar_s_full(1));
          tc_commit(bar_kv_empty(sk));
        }
        __syncwarp();
      }
      if (ok) {
        const uint32_t uv = 2u * (T - 1) + 1u;
        const int sv = uv % C::NSTAGE;
        const uint32_t pv = (uv / C::NSTAGE) & 1u, pp = (uint32_t)(T - 1) & 1u;
        ok = wait_all(bar_kv_full(sv), pv) && pv_tile(0, sv, T - 1 > 0, pp);
        if (ok) {
          if (elect_one()) tc_commit(bar_o_done(0));
          __syncwarp();
          ok = pv_tile(1, sv, T - 1 > 0, pp);
        }
        if (ok) {
          if (elect_one()) {
            tc_commit(bar_o_done(1));
            tc_commit(bar_kv_empty(sv));
          }
          __syncwarp();
        }
      }
      // Drain: all MMAs issued by the elected lane complete before TMEM is released.
      if (elect_one()) {
        tc_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    regs_increase<TC_REGS_SOFTMAX>();
    const int t = warp >> 2;                 // query tile 0 or 1
    const int row = threadIdx.x & 127;       // row inside the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + (t == 0 ? C::COL_S0 : C::COL_S1) + lane_off;
    const uint32_t tO = tmem + (t == 0 ? C::COL_O0 : C::COL_O1) + lane_off;
    const int64_t li = qb.i0 + (int64_t)t * TC_BM + row;   // local row in the segment
    const bool row_valid = li < qb.seg.count;
    const int64_t tq = q_token(pl, qb.seg, li);
    const int64_t tq_tile_min = q_token(pl, qb.seg, qb.i0 + (int64_t)t * TC_BM);
    const float sl2 = pl.scale_log2;
    float m = -INFINITY;   // running max (scaled, log2 units) used for the exponentials
    float l = 0.f;         // running sum of exp2(s * sl2 - m)
    int n = 0;
    bool ok = true;
    // Upper bound of this row's scaled scores (log2 units): |q| max|k| sl2, rounded up by a
    // relative 2^-8 and an absolute 2^-8 that cover the fp32 rounding of the norms and of S.
    // +inf (never skip) without a key bound and for rows past the segment's end.
    float bq = INFINITY;
    if (pl.kbound || pl.kmax_head) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_q_full(t), 0, abort_flag));
      const int64_t mrow = qb.seg.row0 + qb.seg.stride * li;
      if (ok && row_valid && in_bounds(mrow < pl.q_rows)) {
        // |q| of this row from the Q tile (the 128B swizzle permutes 16-byte chunks within
        // the row, which a sum of squares ignores; the rotation by `row` spreads the banks).
        const uint8_t* qrow = smem + C::Q_OFF + t * C::TILE_BYTES + row * 128;
        float ss = 0.f;
#pragma unroll
        for (int b = 0; b < C::NBOX; ++b)
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            const uint4 u = *reinterpret_cast<const uint4*>(qrow + b * C::BOX_BYTES + ((c8 + row) & 7) * 16);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
              ss = fmaf(lo, lo, fmaf(hi, hi, ss));
            }
          }
        const float kmax = pl.kmax_head ? pl.kmax_head[bh] : pl.lse[(int64_t)bh * pl.q_rows + mrow];
        bq = fmaf(sqrtf(ss) * kmax * sl2, 1.00390625f, 0.00390625f);
        if (!(bq >= 0.f)) bq = INFINITY;  // NaN from non-finite inputs: never skip
      }
    }
    for (int s = 0; s < pl.P && ok; ++s) {
      int c = qb.p - s;
      if (c < 0) c += pl.P;
      for (int sk = 0; sk < nks && ok; ++sk) {
        int ntiles, nfull;
        {
          const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
          ntiles = (int)((visible_prefix(pl, ks, tq_max) + TC_BN - 1) / TC_BN);
          // Leading tiles with all 128 keys present and (causal) visible to every row of the
          // query tile: key token of the tile's last key <= the tile's first query token.
          int64_t nf = ks.count / TC_BN;
          if (pl.causal) {
            const int64_t tks = pl.k_tok_stride * ks.stride;
            const int64_t t0 = pl.k_tok0 + pl.k_tok_stride * ks.row0;
            const int64_t slack = tq_tile_min - t0 - tks * (TC_BN - 1);
            const int64_t vis = slack < 0 ? 0 : slack / (tks * TC_BN) + 1;
            if (vis < nf) nf = vis;
          }
          nfull = (int)min(nf, (int64_t)ntiles);
        }
        for (int jt = 0; jt < ntiles; ++jt, ++n) {
          const bool full = jt < nfull;
          if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full(t), (uint32_t)n & 1u, abort_flag))) { ok = false; break; }
          tc_fence_after_sync();
          uint32_t sr[TC_BN];
          // S_t of this row from tensor memory; keys after this row's last visible one are
          // masked on a tile that straddles the causal diagonal or the segment's end.
          RA_TMEM_LD32(tS + 0, (sr + 0));
          RA_TMEM_LD32(tS + 32, (sr + 32));
          RA_TMEM_LD32(tS + 64, (sr + 64));
          RA_TMEM_LD32(tS + 96, (sr + 96));
          tmem_wait_ld();
          RA_REG_FENCE32((sr + 0));
          RA_REG_FENCE32((sr + 32));
          RA_REG_FENCE32((sr + 64));
          RA_REG_FENCE32((sr + 96));
          if (!full) {
            const int lim = last_visible_key(pl, c, sk, jt, tq);
#pragma unroll
            for (int j = 0; j < TC_BN; ++j) sr[j] = (j <= lim) ? sr[j] : __float_as_uint(-INFINITY);
          }
          const uint64_t sl2x2 = f2_pack(sl2, sl2);
          uint64_t sum2a = f2_pack(0.f, 0.f), sum2b = sum2a;
          uint32_t pk[32];
          // Running max update (conditional rescale, see the file comment): m moves only
          // when the tile's max exceeds it by more than RESCALE_LOG2; O and l are then
          // scaled by corr.
          auto update_max = [&](float mx) {
            float corr = 1.f;
            bool rescale = false;
            if (m == -INFINITY) {
              m = mx;  // first visible keys of this row: O and l are still 0
            } else if (mx > m + RESCALE_LOG2) {
              corr = ex2_approx(m - mx);
              m = mx;
              l *= corr;
              rescale = true;
            }
            if (__any_sync(0xffffffffu, rescale) && n > 0) rescale_o<D>(tO, corr);
          };
          // The online update as the pages state it: the tile's row max first, then the
          // exponentials with the (conditionally) updated running max.
          if (!__all_sync(0xffffffffu, bq <= m + MAXSKIP_LOG2)) update_max(row_max(sr) * sl2);
          exp_half(sr, 0, sl2x2, f2_pack(m == -INFINITY ? 0.f : -m, m == -INFINITY ? 0.f : -m), pk, sum2a, sum2b);
          // P of keys 0-63 is complete: the MMA warp may start PV on it while the second half
          // is computed.
          RA_TMEM_ST32(tS, pk);
          arrive_p_ready(bar_p_half(t));
          {
            const float shift = m == -INFINITY ? 0.f : m;
            exp_half(sr, 1, sl2x2, f2_pack(-shift, -shift), pk, sum2a, sum2b);
          }
          RA_TMEM_ST32(tS + 32, pk);
          float sa0, sa1, sb0, sb1;
          f2_unpack(sum2a, sa0, sa1);
          f2_unpack(sum2b, sb0, sb1);
          l += (sa0 + sb0) + (sa1 + sb1);
          arrive_p_ready(bar_p_full(t));
        }
      }
    }
    // ---- epilogue: O = O / l, lse = (m + log2 l) * ln 2
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done(t), 0, abort_flag));
    if (ok) {
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const int64_t mrow = qb.seg.row0 + qb.seg.stride * li;
      const int64_t orow = (int64_t)bh * pl.q_rows + mrow;
      const bool row_ok = row_valid && in_bounds(mrow < pl.q_rows);
      const float lse_row = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      // Folding into a caller's running state (fp32 output only): this row's weights, with
      // the merge kernel's arithmetic; the thread owns the row, so it reads the state before
      // writing it.
      FoldWeights fw{lse_row, 0.f, 1.f};
      if (pl.fold && row_ok) fw = fold_weights(pl.lse[orow], lse_row);
      if (T > 0) tc_fence_after_sync();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t orr[32];
        if (T > 0) {
          RA_TMEM_LD32(tO + cc * 32, orr);
          tmem_wait_ld();
          RA_REG_FENCE32(orr);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) orr[j] = 0u;
        }
        if (row_ok) {
          if (pl.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(pl.o) + orow * D + cc * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float4 o = make_float4(__uint_as_float(orr[4 * j]) * inv_l, __uint_as_float(orr[4 * j + 1]) * inv_l,
                                     __uint_as_float(orr[4 * j + 2]) * inv_l, __uint_as_float(orr[4 * j + 3]) * inv_l);
              if (pl.fold) {
                const float4 st = dst[j];
                o.x = fmaf(fw.w_new, o.x, fmaf(fw.w_state, st.x, 0.f));
                o.y = fmaf(fw.w_new, o.y, fmaf(fw.w_state, st.y, 0.f));
                o.z = fmaf(fw.w_new, o.z, fmaf(fw.w_state, st.z, 0.f));
                o.w = fmaf(fw.w_new, o.w, fmaf(fw.w_state, st.w, 0.f));
              }
              dst[j] = o;
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(pl.o) + orow * D + cc * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(orr[8 * j + 0]) * inv_l, __uint_as_float(orr[8 * j + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(orr[8 * j + 2]) * inv_l, __uint_as_float(orr[8 * j + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(orr[8 * j + 4]) * inv_l, __uint_as_float(orr[8 * j + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(orr[8 * j + 6]) * inv_l, __uint_as_float(orr[8 * j + 7]) * inv_l);
              dst[j] = w;
            }
          }
        }
      }
      if (row_ok && pl.lse != nullptr) pl.lse[orow] = fw.L;
    }
  }

  // ---- teardown: TMEM is released only after every tcgen05 operation has finished.
  tc_fence_before_sync();
  __syncthreads();
  if (warp == TC_WARP_MMA) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
}

}  // namespace ra
