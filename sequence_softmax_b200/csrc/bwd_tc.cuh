// bwd_tc.cuh -- bf16 ring-attention backward, dK and dV, on the 5th-generation tensor cores
// (sm_100a).
//
// Key-stationary: one CTA owns a tile of 128 keys of one virtual ring position and walks
// every 128-row query tile that can see it, in ring order (positions c, c + 1, ... as the
// KV chunk travels; see bwd.cuh). Its dK and dV stay in tensor memory for the whole walk
// and are written once at the end, which is the "sum at the chunk's owner" of the ring
// backward. dQ is computed by the query-stationary kernel of bwd_dq_tc.cuh, so no CTA adds
// into memory another CTA writes: dQ, dK and dV are each produced by exactly one CTA and
// the gradients are bitwise reproducible. (Adding each tile's dQ into a shared fp32
// accumulator instead would cost 64 KB of global reductions per tile pair; measured on B200,
// the L2 absorbs about 6 TB/s of fp32 reductions, ~21 B per clock per SM, which made that
// traffic alone as long as the tile's five GEMMs.)
//
// Per query tile i (Q_i, dO_i, lse_i, D_i staged by TMA / the producer warp):
//   S^T  = K Q_i^T             (M = keys, N = queries, K = d; both operands K-major)
//   dP^T = V dO_i^T            (same form)
//   P^T  = exp2(S^T scale log2e - lse_i log2e), masked; bf16 into the S columns of TMEM
//   dV  += P^T dO_i            (A = P^T from TMEM, B = dO_i MN-major)
//   dS^T = P^T (dP^T - D_i) scale, bf16 into the dP columns of TMEM
//   dK  += dS^T Q_i            (A = dS^T from TMEM, B = Q_i MN-major)
// Four 128 x 128 x d GEMMs and one exponential per score; P and dS never leave the SM.
//
// Warp roles (384 threads, 3 warpgroups; setmaxnreg moves registers to the math warps):
//   warps 0-3, 4-7  math: thread t of warpgroup g owns key row t (TMEM lane t) and query
//                   columns 64g .. 64g + 63 of S^T / dP^T, and dK / dV columns
//                   g d/2 .. g d/2 + d/2 - 1 in the epilogue
//   warp 8          producer: K and V once, then Q_i (3 stages) and dO_i (2 stages) by TMA,
//                   and -lse_i log2e, -D_i scale (read a tile ahead) into a 2-slot ring
//   warp 9          MMA issuer (the whole warp loops, one elected lane issues); order per
//                   tile: dP(i), dV(i), S(i+1), dK(i), so that P(i+1) is computed while
//                   dK(i) runs. P and dS are released in two halves of 32 queries per
//                   thread: the k-steps of dV (dK) over the first halves run while the
//                   second halves are computed (1.4% on the 128K-token causal backward).
//
// Tensor memory (512 columns at d = 128): S^T/P^T [0,128) | dP^T/dS^T [128,256) | dV | dK.
// MMAs issued by one thread execute in order, so S(i+1) overwrites P(i) only after dV(i)
// has read it, and dP(i+1) overwrites dS(i) only after dK(i) has read it.
//
// Query rows beyond a segment's end get -lse log2e = -inf and D = 0, so their P and dS are
// exactly 0 and they add nothing to dK, dV; key rows beyond the end get P = dS = 0 and are
// not written. A query row whose forward lse is -inf saw no key and gets P = 0 as well.
#pragma once

#include "bwd.cuh"

namespace ra {

constexpr int BW_THREADS = 384;
constexpr int BW_WARP_PRODUCER = 8;
constexpr int BW_WARP_MMA = 9;
constexpr int BW_REGS_MATH = 224;   // 2 x 224 + 56 = 504 = 168 * 384 / 128 (216 / 72 spills)
constexpr int BW_REGS_OTHER = 56;
constexpr int BW_TMEM_COLS = 512;

template <int D>
struct BwCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int BOX_BYTES = BWD_TILE * 64 * 2;       // one TMA box: 128 rows x 64 bf16
  static constexpr int NBOX = D / 64;
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;       // a K, V, Q or dO tile
  // Q feeds S(i+1), which is issued before dK(i) frees Q(i): three Q stages give its load two
  // tiles of lead. dO is last read by dV, earlier in the tile: two stages suffice.
  static constexpr int NQ = (D == 128) ? 3 : 4;
  static constexpr int NDO = (D == 128) ? 2 : 4;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TILE_BYTES;
  static constexpr int Q_OFF = 2 * TILE_BYTES;
  static constexpr int DO_OFF = Q_OFF + NQ * TILE_BYTES;
  static constexpr int LD_OFF = DO_OFF + NDO * TILE_BYTES;  // slot s: -lse log2e [128], -D scale [128]
  static constexpr int BAR_OFF = LD_OFF + 2 * 2 * BWD_TILE * 4;
  static constexpr int NBAR = 1 + 2 * NQ + 2 * NDO + 4 + 8;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static constexpr int COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t IDESC_SS = idesc_bf16_f32_ab(128, 128, false, false);
  static constexpr uint32_t IDESC_KMN = idesc_bf16_f32_ab(128, D, false, true);  // dV, dK
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(COL_DK + D <= BW_TMEM_COLS, "tensor memory columns");
};

template <int D>
__global__ void __launch_bounds__(BW_THREADS, 1)
attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const BwdPlan pl) {
  using C = BwCfg<D>;
  // 128-byte-swizzled tiles need 1 KB alignment: asked of the declaration, checked here.
  extern __shared__ __align__(1024) uint8_t bw_smem[];
  uint8_t* smem = bw_smem;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) record_error(DEVERR_BOUNDS);
    return;
  }
  const uint32_t sK = sbase + C::K_OFF, sV = sbase + C::V_OFF;
  auto sQ = [&](int st) { return sbase + C::Q_OFF + (uint32_t)st * C::TILE_BYTES; };
  auto sDO = [&](int st) { return sbase + C::DO_OFF + (uint32_t)st * C::TILE_BYTES; };
  const uint32_t bar0 = sbase + C::BAR_OFF;
  const uint32_t bar_kv_full = bar0;
  auto bar_q_full = [&](int st) { return bar0 + 8u * (1 + st); };
  auto bar_q_empty = [&](int st) { return bar0 + 8u * (1 + C::NQ + st); };
  auto bar_do_full = [&](int st) { return bar0 + 8u * (1 + 2 * C::NQ + st); };
  auto bar_do_empty = [&](int st) { return bar0 + 8u * (1 + 2 * C::NQ + C::NDO + st); };
  auto bar_ld_full = [&](int sl) { return bar0 + 8u * (1 + 2 * C::NQ + 2 * C::NDO + sl); };
  auto bar_ld_empty = [&](int sl) { return bar0 + 8u * (3 + 2 * C::NQ + 2 * C::NDO + sl); };
  const uint32_t bar_s_full = bar0 + 8u * (5 + 2 * C::NQ + 2 * C::NDO), bar_dp_full = bar_s_full + 8u,
                 bar_p_ready = bar_s_full + 16u, bar_ds_ready = bar_s_full + 24u, bar_acc_done = bar_s_full + 32u,
                 bar_drain = bar_s_full + 40u, bar_p_half = bar_s_full + 48u, bar_ds_half = bar_s_full + 56u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Head-major: CTAs running together share one head's Q / dO stream through L2.
  const int units_per_head = (int)(gridDim.x / pl.BH);
  const int bh = blockIdx.x / units_per_head;
  const KTile kt = decode_ktile(pl, blockIdx.x % units_per_head);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int st = 0; st < C::NQ; ++st) {
      mbar_init(bar_q_full(st), 1);
      mbar_init(bar_q_empty(st), 1);
    }
    for (int st = 0; st < C::NDO; ++st) {
      mbar_init(bar_do_full(st), 1);
      mbar_init(bar_do_empty(st), 1);
    }
    for (int sl = 0; sl < 2; ++sl) {
      mbar_init(bar_ld_full(sl), 32);    // the producer's 32 lanes
      mbar_init(bar_ld_empty(sl), 256);  // every math thread, done with the slot
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_ready, 256);
    mbar_init(bar_ds_ready, 256);
    mbar_init(bar_p_half, 256);
    mbar_init(bar_ds_half, 256);
    mbar_init(bar_acc_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == BW_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), BW_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == BW_WARP_PRODUCER && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  int T = 0;  // query tiles this CTA visits (the same walk in every role)
  walk_q_tiles(pl, kt, [&](const Seg&, int64_t) { ++T; return true; });

  if (warp >= 8) regs_decrease<BW_REGS_OTHER>();
  if (warp == BW_WARP_PRODUCER) {
    // ------------------------------------------------------------------ producer
    if (T > 0) {
      if (lane == 0) {
        in_bounds(kt.j0 < kt.seg.count && kt.seg.row0 + kt.seg.stride * (kt.seg.count - 1) < pl.k_rows &&
                  bh < pl.BH);
        mbar_arrive_expect_tx(bar_kv_full, 2 * C::TILE_BYTES);
        const int ky = (int)(kt.seg.row0 % kt.seg.stride);
        const int kz = (int)(kt.seg.row0 / kt.seg.stride + kt.j0);
        for (int b = 0; b < C::NBOX; ++b) {
          tma_load_4d(sK + b * C::BOX_BYTES, &tm_k, bar_kv_full, 64 * b, ky, kz, bh);
          tma_load_4d(sV + b * C::BOX_BYTES, &tm_v, bar_kv_full, 64 * b, ky, kz, bh);
        }
      }
      // lse / D of a tile are read from global memory one tile ahead into registers and
      // stored into their slot when the next tile is issued, so their latency is hidden.
      // The loads are unconditional (rows past the segment end read a valid row and are
      // overridden at store time), so nothing waits for them before the store.
      float ld_l[BWD_TILE / 32], ld_d[BWD_TILE / 32];
      uint32_t ld_valid = 0;
      auto load_ld = [&](const Seg& qs, int64_t i0) {
        ld_valid = 0;
#pragma unroll
        for (int m = 0; m < BWD_TILE / 32; ++m) {
          const int64_t li = i0 + lane + 32 * m;
          const bool v = li < qs.count;
          ld_valid |= (v ? 1u : 0u) << m;
          const int64_t idx = (int64_t)bh * pl.q_rows + qs.row0 + qs.stride * (v ? li : 0);
          const bool ok = in_bounds(qs.row0 + qs.stride * (v ? li : 0) < pl.q_rows);
          ld_l[m] = ok ? pl.lse[idx] : -INFINITY;
          ld_d[m] = ok ? pl.delta[idx] : 0.f;
        }
      };
      auto store_ld = [&](int u) {  // tile u's values into slot u & 1
        const int sl = u & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_ld_empty(sl), ((uint32_t)(u >> 1) & 1u) ^ 1u, abort_flag)))
          return false;
        float* l2s = reinterpret_cast<float*>(smem + C::LD_OFF + sl * 2 * BWD_TILE * 4);
#pragma unroll
        for (int m = 0; m < BWD_TILE / 32; ++m) {
          // rows past the segment end, or that saw no key in the forward: P = 0 and dS = 0
          const bool v = (ld_valid >> m) & 1u;
          l2s[lane + 32 * m] = (v && ld_l[m] != -INFINITY) ? -ld_l[m] * 1.4426950408889634f : -INFINITY;
          l2s[BWD_TILE + lane + 32 * m] = v ? -ld_d[m] * pl.scale : 0.f;
        }
        mbar_arrive(bar_ld_full(sl));
        return true;
      };
      int issued = 0;
      walk_q_tiles(pl, kt, [&](const Seg& qs, int64_t i0) {
        const int i = issued;
        if (i > 0 && !store_ld(i - 1)) return false;
        const int sq = i % C::NQ, sd = i % C::NDO;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_q_empty(sq), ((uint32_t)(i / C::NQ) & 1u) ^ 1u, abort_flag)))
          return false;
        const int qy = (int)(qs.row0 % qs.stride);
        const int qz = (int)(qs.row0 / qs.stride + i0);
        if (lane == 0) {
          in_bounds(i0 < qs.count && qs.row0 + qs.stride * (qs.count - 1) < pl.q_rows);
          mbar_arrive_expect_tx(bar_q_full(sq), C::TILE_BYTES);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_4d(sQ(sq) + b * C::BOX_BYTES, &tm_q, bar_q_full(sq), 64 * b, qy, qz, bh);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar_do_empty(sd), ((uint32_t)(i / C::NDO) & 1u) ^ 1u, abort_flag)))
          return false;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_do_full(sd), C::TILE_BYTES);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_4d(sDO(sd) + b * C::BOX_BYTES, &tm_do, bar_do_full(sd), 64 * b, qy, qz, bh);
        }
        load_ld(qs, i0);
        ++issued;
        return true;
      });
      if (issued == T) store_ld(T - 1);
      // Drain: every TMA load issued lands before the CTA's shared memory goes away.
      if (lane == 0) {
        mbar_wait_drain(bar_kv_full, 0);
        for (int u = issued > C::NQ ? issued - C::NQ : 0; u < issued; ++u)
          mbar_wait_drain(bar_q_full(u % C::NQ), (uint32_t)(u / C::NQ) & 1u);
        for (int u = issued > C::NDO ? issued - C::NDO : 0; u < issued; ++u)
          mbar_wait_drain(bar_do_full(u % C::NDO), (uint32_t)(u / C::NDO) & 1u);
      }
      __syncwarp();
    }
  } else if (warp == BW_WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (T > 0) {
      const uint32_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);  // SBO 1 KB, sm_100 version, 128B swizzle
      auto lo_kmaj = [](uint32_t a) { return ((a & 0x3FFFFu) >> 4) | (1u << 16); };                     // LBO 16 B
      auto lo_mnmaj = [](uint32_t a) { return ((a & 0x3FFFFu) >> 4) | ((uint32_t)(C::BOX_BYTES >> 4) << 16); };
      auto desc = [&](uint32_t lo) { return ((uint64_t)hi << 32) | lo; };
      // K-major k-step kk (16 elements): 32 B inside a 128 B row, the next box every 4 steps.
      auto koff = [](int kk) { return (uint32_t)(((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4); };
      // MN-major k-step: 16 rows of 128 B.
      auto mnoff = [](int kk) { return (uint32_t)(kk * (2048 >> 4)); };
      const uint32_t tS = tmem + C::COL_S, tDP = tmem + C::COL_DP, tDV = tmem + C::COL_DV, tDK = tmem + C::COL_DK;
      const uint32_t lk = lo_kmaj(sK), lv = lo_kmaj(sV);
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
      };
      auto issue_s = [&](int st) {
        const uint32_t lq = lo_kmaj(sQ(st));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tS, desc(lk + koff(kk)), desc(lq + koff(kk)), C::IDESC_SS, kk > 0);
        tc_commit(bar_s_full);
      };
      bool ok = wait_all(bar_kv_full, 0) && wait_all(bar_q_full(0), 0);
      if (ok) {
        tc_fence_after_sync();
        if (elect_one()) issue_s(0);
        __syncwarp();
      }
      for (int i = 0; i < T && ok; ++i) {
        const int sq = i % C::NQ, sd = i % C::NDO;
        const uint32_t pi = (uint32_t)i & 1u;
        const uint32_t ldo = lo_kmaj(sDO(sd)), lq_mn = lo_mnmaj(sQ(sq)), ldo_mn = lo_mnmaj(sDO(sd));
        if (!(ok = wait_all(bar_do_full(sd), (uint32_t)(i / C::NDO) & 1u))) break;
        tc_fence_after_sync();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tDP, desc(lv + koff(kk)), desc(ldo + koff(kk)), C::IDESC_SS, kk > 0);
          tc_commit(bar_dp_full);
        }
        __syncwarp();
        // P^T pairs: queries 0-63 in columns [0, 32), queries 64-127 in [64, 96); each half
        // of a warpgroup's columns (k-steps 0,1 | 2,3 and 4,5 | 6,7) is released on its own.
        if (!(ok = wait_all(bar_p_half, pi))) break;
        tc_fence_after_sync();
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int kk = (h & 1) + (h >> 1) * 4;
            mma_bf16_ts(tDV, tS + kk * 8 + (kk >= 4 ? 32 : 0), desc(ldo_mn + mnoff(kk)), C::IDESC_KMN,
                        (i > 0 || h > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
        if (!(ok = wait_all(bar_p_ready, pi))) break;
        tc_fence_after_sync();
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int kk = 2 + (h & 1) + (h >> 1) * 4;
            mma_bf16_ts(tDV, tS + kk * 8 + (kk >= 4 ? 32 : 0), desc(ldo_mn + mnoff(kk)), C::IDESC_KMN, 1u);
          }
          tc_commit(bar_do_empty(sd));  // dO(i) is last read by dV(i)
        }
        __syncwarp();
        if (i + 1 < T) {
          // S(i+1) overwrites the S columns only after dV(i) (issued above) has read P(i).
          const int sq1 = (i + 1) % C::NQ;
          if (!(ok = wait_all(bar_q_full(sq1), (uint32_t)((i + 1) / C::NQ) & 1u))) break;
          tc_fence_after_sync();
          if (elect_one()) issue_s(sq1);
          __syncwarp();
        }
        if (!(ok = wait_all(bar_ds_half, pi))) break;
        tc_fence_after_sync();
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int kk = (h & 1) + (h >> 1) * 4;
            mma_bf16_ts(tDK, tDP + kk * 8 + (kk >= 4 ? 32 : 0), desc(lq_mn + mnoff(kk)), C::IDESC_KMN,
                        (i > 0 || h > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
        if (!(ok = wait_all(bar_ds_ready, pi))) break;
        tc_fence_after_sync();
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int kk = 2 + (h & 1) + (h >> 1) * 4;
            mma_bf16_ts(tDK, tDP + kk * 8 + (kk >= 4 ? 32 : 0), desc(lq_mn + mnoff(kk)), C::IDESC_KMN, 1u);
          }
          tc_commit(bar_q_empty(sq));  // Q(i) is last read by dK(i)
          if (i == T - 1) tc_commit(bar_acc_done);
        }
        __syncwarp();
      }
      if (elect_one()) {
        tc_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ math warpgroups
    regs_increase<BW_REGS_MATH>();
    const int g = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int c0 = 64 * g;  // this thread's query columns of S^T / dP^T
    const uint32_t tS = tmem + C::COL_S + lane_off, tDP = tmem + C::COL_DP + lane_off;
    const int64_t jl = kt.j0 + row;
    const bool kvalid = jl < kt.seg.count;
    const int64_t tk = pl.k_tok0 + pl.k_tok_stride * (kt.seg.row0 + kt.seg.stride * jl);
    int i = 0;
    bool ok = true;
    walk_q_tiles(pl, kt, [&](const Seg& qs, int64_t i0) {
      const int sl = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u, pi = (uint32_t)i & 1u;
      // Causal: query column c (token tq0 + tqs c) sees this key iff c >= lo.
      const int64_t tqs = pl.q_tok_stride * qs.stride;
      const int64_t tq0 = pl.q_tok0 + pl.q_tok_stride * (qs.row0 + qs.stride * i0);
      int lo = 0;
      if (!kvalid) lo = BWD_TILE;
      else if (pl.causal && tk > tq0) lo = ceil_div_clamped(tk - tq0, tqs, BWD_TILE);
      // columns c0 .. c0 + 63 of this thread: those below `lo` are masked
      const bool masked = !__all_sync(0xffffffffu, lo <= c0);
      const float* l2s = reinterpret_cast<const float*>(smem + C::LD_OFF + sl * 2 * BWD_TILE * 4) + c0;
      const float* dls = l2s + BWD_TILE;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_ld_full(sl), ph, abort_flag)))) return false;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full, pi, abort_flag)))) return false;
      tc_fence_after_sync();
      float p[64];
      // Two halves of 32 queries, each released once stored: P pairs of columns c0 .. c0 + 31
      // land in the S cells c0 .. c0 + 15, already read, those of c0 + 32 .. c0 + 63 in
      // c0 + 16 .. c0 + 31.
      {
        uint32_t pk[16];
        bwd_exp_part32<true, 0>(tS + c0, l2s, 0.f, pl.scale_log2, masked, lo - c0, 64, p);
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(p[2 * j], p[2 * j + 1]);
        RA_TMEM_ST16(tS + c0, pk);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar_p_half);
        bwd_exp_part32<true, 32>(tS + c0, l2s, 0.f, pl.scale_log2, masked, lo - c0, 64, p);
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(p[32 + 2 * j], p[33 + 2 * j]);
        RA_TMEM_ST16(tS + c0 + 16, pk);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar_p_ready);
      }

      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_full, pi, abort_flag)))) return false;
      tc_fence_after_sync();
      {
        uint32_t dsk[16];
        bwd_ds_part32<true, 0>(tDP + c0, p, dls, 0.f, pl.scale, dsk);
        RA_TMEM_ST16(tDP + c0, dsk);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar_ds_half);
        bwd_ds_part32<true, 32>(tDP + c0, p, dls, 0.f, pl.scale, dsk);
        RA_TMEM_ST16(tDP + c0 + 16, dsk);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar_ds_ready);
      }
      mbar_arrive(bar_ld_empty(sl));  // done with this tile's -lse log2e and -D scale
      ++i;
      return true;
    });

    // ---- epilogue: dV and dK of this thread's key row, columns g d/2 .. g d/2 + d/2 - 1
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_done, 0, abort_flag));
    if (ok) {
      if (T > 0) tc_fence_after_sync();
      const int64_t krow = kt.seg.row0 + kt.seg.stride * jl;
      const int64_t off = ((int64_t)bh * pl.k_rows + krow) * D + g * (D / 2);
      const bool row_ok = kvalid && in_bounds(krow < pl.k_rows);
      bwd_store_acc_row<D / 2>(tmem + C::COL_DV + lane_off + g * (D / 2), T > 0, row_ok, pl.dv, off,
                               pl.accumulate != 0);
      bwd_store_acc_row<D / 2>(tmem + C::COL_DK + lane_off + g * (D / 2), T > 0, row_ok, pl.dk, off,
                               pl.accumulate != 0);
    }
  }

  // ---- teardown: TMEM is released only after every tcgen05 operation has finished.
  tc_fence_before_sync();
  __syncthreads();
  if (warp == BW_WARP_MMA) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, BW_TMEM_COLS);
  }
}

}  // namespace ra
