// bwd_dq_tc.cuh -- bf16 ring-attention backward, dQ, on the 5th-generation tensor cores
// (sm_100a).
//
// Query-stationary: one CTA owns a tile of 128 query rows of one virtual ring position and
// walks the KV tiles its queries can see in the forward's ring order (position p visits
// position (p - s) mod P at step s). Its dQ stays in tensor memory for the whole walk and
// is written once, so each query row's dQ is produced by exactly one CTA. This is the
// ring backward's "add dS K to the position's own dQ at every step"; the KV side (dK, dV)
// is the key-stationary kernel of bwd_tc.cuh.
//
// Per KV tile n (K_n into a 3-stage ring, V_n into a 2-stage ring by TMA; Q, dO loaded once):
//   S    = Q K_n^T             (M = queries, N = keys, K = d; both operands K-major)
//   dP   = dO V_n^T            (same form)
//   P    = exp2(S scale log2e - lse log2e), masked    (lse and D are per thread: one row)
//   dS   = P (dP - D) scale, bf16 into the S columns of TMEM just read
//   dQ  += dS K_n              (A = dS from TMEM, B = K_n MN-major)
// Three 128 x 128 x d GEMMs and one exponential per score.
//
// Warp roles (384 threads): warps 0-7 math (thread t of warpgroup g owns query row t =
// TMEM lane t and key columns 64g .. 64g + 63; dQ columns g d/2 .. in the epilogue), warp 8
// TMA producer, warp 9 MMA issuer. S is double-buffered so that S(n+1) runs while tile n's
// exponentials are computed: MMA order S(n+1), dQ(n), dP(n+1).
//
// Tensor memory (512 columns at d = 128): S_0 [0,128) | S_1 [128,256) | dP [256,384) | dQ.
#pragma once

#include "bwd.cuh"

namespace ra {

constexpr int BQ_THREADS = 384;
constexpr int BQ_WARP_PRODUCER = 8;
constexpr int BQ_WARP_MMA = 9;
constexpr int BQ_REGS_MATH = 216;
constexpr int BQ_REGS_OTHER = 72;
constexpr int BQ_TMEM_COLS = 512;

template <int D>
struct BqCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int BOX_BYTES = BWD_TILE * 64 * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
  // K feeds S(n+1), issued before dQ(n) frees K(n): three K stages give its load two tiles of
  // lead. V is last read by dP, earlier: two stages suffice.
  static constexpr int NK = (D == 128) ? 3 : 4;
  static constexpr int NV = (D == 128) ? 2 : 4;
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = TILE_BYTES;
  static constexpr int K_OFF = 2 * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NK * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + NV * TILE_BYTES;
  static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 6;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static constexpr int COL_S0 = 0, COL_S1 = 128, COL_DP = 256, COL_DQ = 384;
  static constexpr uint32_t IDESC_SS = idesc_bf16_f32_ab(128, 128, false, false);
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32_ab(128, D, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(COL_DQ + D <= BQ_TMEM_COLS, "tensor memory columns");
};

// The query tile a CTA owns: local rows i0 .. i0 + 127 of segment `seg` of position p.
struct QTile {
  int p;
  Seg seg;
  int64_t i0;
};

// Units within one head, latest tokens first: under the causal mask the latest queries see
// the most keys, so the longest-running CTAs start first.
__device__ __forceinline__ QTile decode_qtile(const BwdPlan& pl, int unit) {
  QTile t;
  const int P = pl.P;
  const int64_t nqt = (pl.q_seg_len + BWD_TILE - 1) / BWD_TILE;
  int si = 0;
  int64_t qt;
  if (pl.layout == RA_LAYOUT_STRIPED) {
    qt = nqt - 1 - unit / P;
    t.p = P - 1 - unit % P;
  } else if (pl.layout == RA_LAYOUT_ZIGZAG) {
    const int gc = 2 * P - 1 - (int)(unit / nqt);  // global chunk, latest first
    qt = nqt - 1 - unit % nqt;
    if (gc >= P) { t.p = 2 * P - 1 - gc; si = 1; } else { t.p = gc; si = 0; }
  } else {
    t.p = P - 1 - (int)(unit / nqt);
    qt = nqt - 1 - unit % nqt;
  }
  t.seg = segment_of(pl.layout, P, pl.q_seg_len, t.p, si);
  t.i0 = qt * BWD_TILE;
  return t;
}

// Keys of segment ks (from its start) that can be visible to a query of token <= tq_max.
__device__ __forceinline__ int64_t bwd_visible_prefix(const BwdPlan& pl, const Seg& ks, int64_t tq_max) {
  if (!pl.causal) return ks.count;
  const int64_t t0 = pl.k_tok0 + pl.k_tok_stride * ks.row0;
  const int64_t ts = pl.k_tok_stride * ks.stride;
  if (tq_max < t0) return 0;
  const int64_t n = (tq_max - t0) / ts + 1;
  return n < ks.count ? n : ks.count;
}

// Calls f(ks, j0) for every 128-key tile (local keys j0 .. j0 + 127 of segment ks) that a
// query of token <= tq_max can see, in the forward's ring order. Stops when f returns false.
template <class F>
__device__ __forceinline__ void walk_k_tiles(const BwdPlan& pl, int p, int64_t tq_max, F&& f) {
  const int nks = num_segments(pl.layout);
  for (int s = 0; s < pl.P; ++s) {
    int c = p - s;
    if (c < 0) c += pl.P;
    for (int sk = 0; sk < nks; ++sk) {
      const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
      const int64_t nt = (bwd_visible_prefix(pl, ks, tq_max) + BWD_TILE - 1) / BWD_TILE;
      for (int64_t jt = 0; jt < nt; ++jt)
        if (!f(ks, jt * BWD_TILE)) return;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(BQ_THREADS, 1)
attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdPlan pl) {
  using C = BqCfg<D>;
  extern __shared__ __align__(1024) uint8_t bq_smem[];
  uint8_t* smem = bq_smem;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) record_error(DEVERR_BOUNDS);
    return;
  }
  const uint32_t sQ = sbase + C::Q_OFF, sDO = sbase + C::DO_OFF;
  auto sK = [&](int st) { return sbase + C::K_OFF + (uint32_t)st * C::TILE_BYTES; };
  auto sV = [&](int st) { return sbase + C::V_OFF + (uint32_t)st * C::TILE_BYTES; };
  const uint32_t bar0 = sbase + C::BAR_OFF;
  const uint32_t bar_qo_full = bar0;
  auto bar_k_full = [&](int st) { return bar0 + 8u * (1 + st); };
  auto bar_k_empty = [&](int st) { return bar0 + 8u * (1 + C::NK + st); };
  auto bar_v_full = [&](int st) { return bar0 + 8u * (1 + 2 * C::NK + st); };
  auto bar_v_empty = [&](int st) { return bar0 + 8u * (1 + 2 * C::NK + C::NV + st); };
  // One "S ready" barrier per S buffer: S(n+2) reuses buffer n & 1 only after every math
  // thread has arrived on ds_ready(n), i.e. after it has seen S(n), so a waiter never sees
  // two phases of its barrier complete (with one barrier for both buffers, S(n+2) could
  // complete before a slow thread had seen S(n+1)).
  auto bar_s_full = [&](int b) { return bar0 + 8u * (1 + 2 * C::NK + 2 * C::NV + b); };
  const uint32_t bar_dp_full = bar0 + 8u * (3 + 2 * C::NK + 2 * C::NV), bar_ds_ready = bar_dp_full + 8u,
                 bar_acc_done = bar_dp_full + 16u, bar_drain = bar_dp_full + 24u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units_per_head = (int)(gridDim.x / pl.BH);
  const int bh = blockIdx.x / units_per_head;
  const QTile qt = decode_qtile(pl, blockIdx.x % units_per_head);
  const int64_t q_last = min(qt.i0 + BWD_TILE, qt.seg.count) - 1;  // last valid local row
  const int64_t tq_max = pl.q_tok0 + pl.q_tok_stride * (qt.seg.row0 + qt.seg.stride * q_last);

  if (threadIdx.x == 0) {
    mbar_init(bar_qo_full, 1);
    for (int st = 0; st < C::NK; ++st) {
      mbar_init(bar_k_full(st), 1);
      mbar_init(bar_k_empty(st), 1);
    }
    for (int st = 0; st < C::NV; ++st) {
      mbar_init(bar_v_full(st), 1);
      mbar_init(bar_v_empty(st), 1);
    }
    mbar_init(bar_s_full(0), 1);
    mbar_init(bar_s_full(1), 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_ready, 256);
    mbar_init(bar_acc_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == BQ_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), BQ_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == BQ_WARP_PRODUCER && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  int T = 0;  // KV tiles this CTA visits (the same walk in every role)
  walk_k_tiles(pl, qt.p, tq_max, [&](const Seg&, int64_t) { ++T; return true; });

  if (warp >= 8) regs_decrease<BQ_REGS_OTHER>();
  if (warp == BQ_WARP_PRODUCER) {
    // ------------------------------------------------------------------ producer
    if (T > 0 && lane == 0) {
      in_bounds(qt.i0 < qt.seg.count && qt.seg.row0 + qt.seg.stride * (qt.seg.count - 1) < pl.q_rows &&
                bh < pl.BH);
      mbar_arrive_expect_tx(bar_qo_full, 2 * C::TILE_BYTES);
      const int qy = (int)(qt.seg.row0 % qt.seg.stride);
      const int qz = (int)(qt.seg.row0 / qt.seg.stride + qt.i0);
      for (int b = 0; b < C::NBOX; ++b) {
        tma_load_4d(sQ + b * C::BOX_BYTES, &tm_q, bar_qo_full, 64 * b, qy, qz, bh);
        tma_load_4d(sDO + b * C::BOX_BYTES, &tm_do, bar_qo_full, 64 * b, qy, qz, bh);
      }
      int issued = 0;
      walk_k_tiles(pl, qt.p, tq_max, [&](const Seg& ks, int64_t j0) {
        const int n = issued, sk = n % C::NK, sv = n % C::NV;
        const int ky = (int)(ks.row0 % ks.stride);
        const int kz = (int)(ks.row0 / ks.stride + j0);
        in_bounds(j0 < ks.count && ks.row0 + ks.stride * (ks.count - 1) < pl.k_rows);
        if (!mbar_wait(bar_k_empty(sk), ((uint32_t)(n / C::NK) & 1u) ^ 1u, abort_flag)) return false;
        mbar_arrive_expect_tx(bar_k_full(sk), C::TILE_BYTES);
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_4d(sK(sk) + b * C::BOX_BYTES, &tm_k, bar_k_full(sk), 64 * b, ky, kz, bh);
        if (!mbar_wait(bar_v_empty(sv), ((uint32_t)(n / C::NV) & 1u) ^ 1u, abort_flag)) return false;
        mbar_arrive_expect_tx(bar_v_full(sv), C::TILE_BYTES);
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_4d(sV(sv) + b * C::BOX_BYTES, &tm_v, bar_v_full(sv), 64 * b, ky, kz, bh);
        ++issued;
        return true;
      });
      // Drain: every TMA load issued lands before the CTA's shared memory goes away.
      mbar_wait_drain(bar_qo_full, 0);
      for (int u = issued > C::NK ? issued - C::NK : 0; u < issued; ++u)
        mbar_wait_drain(bar_k_full(u % C::NK), (uint32_t)(u / C::NK) & 1u);
      for (int u = issued > C::NV ? issued - C::NV : 0; u < issued; ++u)
        mbar_wait_drain(bar_v_full(u % C::NV), (uint32_t)(u / C::NV) & 1u);
    }
  } else if (warp == BQ_WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (T > 0) {
      const uint32_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);  // SBO 1 KB, sm_100 version, 128B swizzle
      auto lo_kmaj = [](uint32_t a) { return ((a & 0x3FFFFu) >> 4) | (1u << 16); };
      auto lo_mnmaj = [](uint32_t a) { return ((a & 0x3FFFFu) >> 4) | ((uint32_t)(C::BOX_BYTES >> 4) << 16); };
      auto desc = [&](uint32_t lo) { return ((uint64_t)hi << 32) | lo; };
      auto koff = [](int kk) { return (uint32_t)(((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4); };
      auto mnoff = [](int kk) { return (uint32_t)(kk * (2048 >> 4)); };
      const uint32_t tDP = tmem + C::COL_DP, tDQ = tmem + C::COL_DQ;
      auto tSb = [&](int n) { return tmem + ((n & 1) ? C::COL_S1 : C::COL_S0); };
      const uint32_t lq = lo_kmaj(sQ), ldo = lo_kmaj(sDO);
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
      };
      auto issue_s = [&](int n) {
        const uint32_t lk = lo_kmaj(sK(n % C::NK));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tSb(n), desc(lq + koff(kk)), desc(lk + koff(kk)), C::IDESC_SS, kk > 0);
        tc_commit(bar_s_full(n & 1));
      };
      auto issue_dp = [&](int n) {  // V(n) is last read here
        const int sv = n % C::NV;
        const uint32_t lv = lo_kmaj(sV(sv));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tDP, desc(ldo + koff(kk)), desc(lv + koff(kk)), C::IDESC_SS, kk > 0);
        tc_commit(bar_dp_full);
        tc_commit(bar_v_empty(sv));
      };
      bool ok = wait_all(bar_qo_full, 0) && wait_all(bar_k_full(0), 0);
      if (ok) {
        tc_fence_after_sync();
        if (elect_one()) issue_s(0);
        __syncwarp();
        ok = wait_all(bar_v_full(0), 0);
      }
      if (ok) {
        tc_fence_after_sync();
        if (elect_one()) issue_dp(0);
        __syncwarp();
      }
      for (int n = 0; n < T && ok; ++n) {
        const int sk = n % C::NK;
        if (n + 1 < T) {
          // S(n+1) goes to the other S buffer, last read by dQ(n-1) (issued before).
          const int sk1 = (n + 1) % C::NK;
          if (!(ok = wait_all(bar_k_full(sk1), (uint32_t)((n + 1) / C::NK) & 1u))) break;
          tc_fence_after_sync();
          if (elect_one()) issue_s(n + 1);
          __syncwarp();
        }
        if (!(ok = wait_all(bar_ds_ready, (uint32_t)n & 1u))) break;
        tc_fence_after_sync();
        if (elect_one()) {
          const uint32_t lk_mn = lo_mnmaj(sK(sk));
          // dS pairs: keys 0-63 in columns [0, 32) of the S buffer, keys 64-127 in [64, 96).
#pragma unroll
          for (int kk = 0; kk < BWD_TILE / 16; ++kk)
            mma_bf16_ts(tDQ, tSb(n) + kk * 8 + (kk >= 4 ? 32 : 0), desc(lk_mn + mnoff(kk)), C::IDESC_DQ,
                        (n > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar_k_empty(sk));  // K(n) is last read by dQ(n)
          if (n + 1 == T) tc_commit(bar_acc_done);
        }
        __syncwarp();
        if (n + 1 < T) {
          // dP(n+1): the math warps have read dP(n) (ds_ready above)
          if (!(ok = wait_all(bar_v_full((n + 1) % C::NV), (uint32_t)((n + 1) / C::NV) & 1u))) break;
          tc_fence_after_sync();
          if (elect_one()) issue_dp(n + 1);
          __syncwarp();
        }
      }
      if (elect_one()) {
        tc_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ math warpgroups
    regs_increase<BQ_REGS_MATH>();
    const int g = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int c0 = 64 * g;  // this thread's key columns of S / dP
    const int64_t li = qt.i0 + row;
    const int64_t qrow = qt.seg.row0 + qt.seg.stride * li;
    const bool qvalid = li < qt.seg.count && in_bounds(qrow < pl.q_rows);
    const int64_t tq = pl.q_tok0 + pl.q_tok_stride * qrow;
    float nl2row = -INFINITY, ndsrow = 0.f;  // rows past the segment end (or that saw no key): P = 0
    if (qvalid) {
      const float l = pl.lse[(int64_t)bh * pl.q_rows + qrow];
      if (l != -INFINITY) nl2row = -l * 1.4426950408889634f;
      ndsrow = -pl.delta[(int64_t)bh * pl.q_rows + qrow] * pl.scale;
    }
    int n = 0;
    bool ok = true;
    walk_k_tiles(pl, qt.p, tq_max, [&](const Seg& ks, int64_t j0) {
      const uint32_t pn = (uint32_t)n & 1u;
      const uint32_t tS = tmem + ((n & 1) ? C::COL_S1 : C::COL_S0) + lane_off + c0;
      // visible key columns of this row: j < hi (tile end, and causally tk0 + tks j <= tq)
      const int64_t tks = pl.k_tok_stride * ks.stride;
      const int64_t tk0 = pl.k_tok0 + pl.k_tok_stride * (ks.row0 + ks.stride * j0);
      int hi = (int)min((int64_t)BWD_TILE, ks.count - j0);
      if (pl.causal) hi = tq < tk0 ? 0 : min(hi, ceil_div_clamped(tq - tk0 + 1, tks, BWD_TILE));
      const int hl = hi - c0;  // relative to this thread's first column
      const bool masked = !__all_sync(0xffffffffu, hl >= 64);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full(n & 1), (uint32_t)(n >> 1) & 1u, abort_flag))))
        return false;
      tc_fence_after_sync();
      float p[64];
      bwd_exp_row64<false>(tS, nullptr, nl2row, pl.scale_log2, masked, 0, hl, p);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_full, pn, abort_flag)))) return false;
      tc_fence_after_sync();
      uint32_t dsk[32];
      bwd_ds_row64<false>(tmem + C::COL_DP + lane_off + c0, p, nullptr, ndsrow, pl.scale, dsk);
      RA_TMEM_ST32(tS, dsk);
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(bar_ds_ready);
      ++n;
      return true;
    });

    // ---- epilogue: dQ of this thread's query row, columns g d/2 .. g d/2 + d/2 - 1
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_done, 0, abort_flag));
    if (ok) {
      if (T > 0) tc_fence_after_sync();
      const int64_t off = ((int64_t)bh * pl.q_rows + qrow) * D + g * (D / 2);
      bwd_store_acc_row<D / 2>(tmem + C::COL_DQ + lane_off + g * (D / 2), T > 0, qvalid, pl.dq, off,
                               pl.accumulate != 0);
    }
  }

  // ---- teardown: TMEM is released only after every tcgen05 operation has finished.
  tc_fence_before_sync();
  __syncthreads();
  if (warp == BQ_WARP_MMA) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, BQ_TMEM_COLS);
  }
}

}  // namespace ra
