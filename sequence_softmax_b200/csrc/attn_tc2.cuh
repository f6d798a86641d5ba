// attn_tc2.cuh -- the bf16, d = 128 ring-attention forward on CTA pairs (sm_100a).
//
// The same online-softmax walk as attn_tc.cuh ([BLOG] ring_attention_forward,
// blockwise_attention, ring_attention_causal_step; [CARD] online softmax), with the tensor
// core work of two SMs fused: a cluster of two CTAs (an even "leader" and its peer) owns a
// query block of 512 rows, and every GEMM is one pair MMA (tcgen05.mma.cta_group::2,
// M = 256) whose rows 0-127 live in the leader and 128-255 in the peer. Each CTA stages only
// half of every K/V tile (K: 64 of the 128 keys; V: 64 of the 128 head-dimension columns) and
// the two SMs' tensor cores share the halves, so per SM the K/V traffic from L2, the TMA
// writes into shared memory and the B-operand reads of shared memory are half those of the
// single-CTA kernel, for the same arithmetic.
//
// Per CTA (384 threads, as in attn_tc.cuh):
//   warps 0-7  softmax of the CTA's two 128-row query tiles (pair tiles t = 0, 1), one thread
//              per row, on the CTA's own tensor memory
//   warp  8    TMA producer: the CTA's own Q rows and its half of every K/V tile
//   warp  9    leader: MMA issuer for the pair; both: tensor-memory allocation
//   warp 10    peer: relays the arrival of its own TMA data to the leader's barriers
//
// Synchronisation across the pair:
//   * The peer's TMA loads complete on its own barriers; its relay warp waits on them and
//     arrives on the leader's (so each CTA can drain its own loads before it exits).
//   * The leader's MMA warp waits on its barriers at cluster scope and issues the pair MMAs;
//     its commits arrive on the barriers of both CTAs (S ready, O final, K/V stage free).
//   * Both CTAs' softmax warps arrive on the leader's P barriers, one arrival per warp.
//   * A cluster barrier after the barrier set-up and one before the tensor memory is freed.
// Tensor-memory layout, MMA order and conditional rescale are those of attn_tc.cuh.
#pragma once

#include "attn_tc.cuh"

namespace ra {

constexpr int TC2_BLOCK_ROWS = 4 * TC_BM;  // query rows per CTA pair
constexpr int TC2_WARP_RELAY = 10;

struct Tc2Cfg {
  static constexpr int D = 128;
  static constexpr int QBOX_BYTES = TC_BM * 64 * 2;    // 128 rows x 64 columns of bf16
  static constexpr int Q_TILE_BYTES = 2 * QBOX_BYTES;   // one 128 x 128 query tile
  static constexpr int KBOX_BYTES = (TC_BN / 2) * 64 * 2;  // 64 keys x 64 columns
  static constexpr int STAGE_BYTES = 16384;             // a K half (2 boxes) or a V half (1 box)
  static constexpr int NSTAGE = 8;                      // K/V stages (4 tiles in flight)
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * Q_TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSTAGE * STAGE_BYTES;
  // q_full[2] kv_full[NSTAGE] kv_empty[NSTAGE] s_full[2] p_half[2] p_full[2] o_done[2] drain
  // q_own[2] kv_own[NSTAGE]
  static constexpr int NBAR = 2 + 2 * NSTAGE + 2 + 2 + 2 + 2 + 1 + 2 + NSTAGE;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 384;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(2 * TC_BM, TC_BN, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(2 * TC_BM, D, true);
};

__global__ void __launch_bounds__(TC_THREADS, 1)
attn_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k64,
                    const __grid_constant__ CUtensorMap tm_v, const Plan pl) {
  using C = Tc2Cfg;
  constexpr int D = C::D;
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
  auto bar_p_half = [&](int t) { return bar0 + 8u * (4 + 2 * C::NSTAGE + t); };
  auto bar_p_full = [&](int t) { return bar0 + 8u * (6 + 2 * C::NSTAGE + t); };
  auto bar_o_done = [&](int t) { return bar0 + 8u * (8 + 2 * C::NSTAGE + t); };
  const uint32_t bar_drain = bar0 + 8u * (10 + 2 * C::NSTAGE);
  auto bar_q_own = [&](int t) { return bar0 + 8u * (11 + 2 * C::NSTAGE + t); };
  auto bar_kv_own = [&](int s) { return bar0 + 8u * (13 + 2 * C::NSTAGE + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t cr = cluster_ctarank();  // 0: leader, 1: peer
  const bool leader = cr == 0;
  // Head-major order of pairs (see attn_tc.cuh): the pairs running together share one head's
  // K/V stream through L2.
  const int pair = blockIdx.x >> 1;
  const int units_per_head = (int)((gridDim.x >> 1) / pl.BH);
  const int bh = pair / units_per_head;
  const int unit = pair % units_per_head;
  const QBlock qb = decode_unit(pl, unit, TC2_BLOCK_ROWS);
  const int64_t q_last = min(qb.i0 + TC2_BLOCK_ROWS, qb.seg.count) - 1;
  const int64_t tq_max = q_token(pl, qb.seg, q_last);
  const int nks = num_segments(pl.layout);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_q_full(t), 2);   // the leader's expect_tx arrival + the peer's relay
      mbar_init(bar_q_own(t), 1);    // the peer's own expect_tx arrival
      mbar_init(bar_s_full(t), 1);
      mbar_init(bar_p_half(t), 8);   // one arrival per softmax warp of the tile, both CTAs
      mbar_init(bar_p_full(t), 8);
      mbar_init(bar_o_done(t), 1);
    }
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar_kv_full(s), 2);
      mbar_init(bar_kv_own(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == TC_WARP_MMA) {
    tmem_alloc_pair(smem_u32(tmem_slot), TC_TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == TC_WARP_PRODUCER && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k64);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival or pair commit
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // KV tiles this pair visits (identical walk in every role of both CTAs).
  int T = 0;
  for (int s = 0; s < pl.P; ++s) {
    int c = qb.p - s;
    if (c < 0) c += pl.P;
    for (int sk = 0; sk < nks; ++sk) {
      const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
      T += (int)((visible_prefix(pl, ks, tq_max) + TC_BN - 1) / TC_BN);
    }
  }

  if (warp >= 8) regs_decrease<TC_REGS_OTHER>();
  if (warp == TC_WARP_PRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int qy = (int)(qb.seg.row0 % qb.seg.stride);
      const int64_t qz0 = qb.seg.row0 / qb.seg.stride + qb.i0;
      in_bounds(qb.i0 < qb.seg.count && qb.seg.row0 + qb.seg.stride * (qb.seg.count - 1) < pl.q_rows &&
                bh < pl.BH);
      // leader: its loads complete on the barriers the MMA waits on; peer: on its own, relayed
      auto q_bar = [&](int t) { return leader ? bar_q_full(t) : bar_q_own(t); };
      auto kv_bar = [&](int s) { return leader ? bar_kv_full(s) : bar_kv_own(s); };
      for (int t = 0; t < 2; ++t) {
        mbar_arrive_expect_tx(q_bar(t), C::Q_TILE_BYTES);
        for (int b = 0; b < 2; ++b)
          tma_load_4d(sQ + t * C::Q_TILE_BYTES + b * C::QBOX_BYTES, &tm_q, q_bar(t), 64 * b, qy,
                      (int)(qz0 + t * 2 * TC_BM + cr * TC_BM), bh);
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
              mbar_arrive_expect_tx(kv_bar(st), C::STAGE_BYTES);
              const uint32_t dst = sKV + st * C::STAGE_BYTES;
              if (kv == 0) {
                // K: this CTA's 64 keys of the tile, all 128 columns (two 64-column boxes)
                for (int b = 0; b < 2; ++b)
                  tma_load_4d(dst + b * C::KBOX_BYTES, &tm_k64, kv_bar(st), 64 * b, ky,
                              (int)(kz0 + (int64_t)jt * TC_BN + cr * (TC_BN / 2)), bh);
              } else {
                // V: all 128 keys of the tile, this CTA's 64 head-dimension columns
                tma_load_4d(dst, &tm_v, kv_bar(st), 64 * (int)cr, ky, (int)(kz0 + (int64_t)jt * TC_BN), bh);
              }
            }
          }
        }
      }
      // Drain: every load this CTA issued lands before its shared memory goes away.
      const uint32_t first = use > (uint32_t)C::NSTAGE ? use - C::NSTAGE : 0u;
      for (uint32_t u = first; u < use; ++u) mbar_wait_drain(kv_bar(u % C::NSTAGE), (u / C::NSTAGE) & 1u);
      mbar_wait_drain(q_bar(0), 0);
      mbar_wait_drain(q_bar(1), 0);
    }
  } else if (warp == TC2_WARP_RELAY && !leader) {
    // ------------------------------------------------------------------ peer relay
    if (lane == 0) {
      bool ok = true;
      for (int t = 0; t < 2 && ok; ++t) {
        ok = mbar_wait(bar_q_own(t), 0, abort_flag);
        if (ok) mbar_arrive_remote(mapa_shared(bar_q_full(t), 0));
      }
      for (uint32_t u = 0; u < 2u * (uint32_t)T && ok; ++u) {
        const int st = u % C::NSTAGE;
        ok = mbar_wait(bar_kv_own(st), (u / C::NSTAGE) & 1u, abort_flag);
        if (ok) mbar_arrive_remote(mapa_shared(bar_kv_full(st), 0));
      }
    }
  } else if (warp == TC_WARP_MMA && leader) {
    // ------------------------------------------------------------------ pair MMA issuer
    if (T > 0) {
      const uint32_t tS[2] = {tmem + C::COL_S0, tmem + C::COL_S1};
      const uint32_t tO[2] = {tmem + C::COL_O0, tmem + C::COL_O1};
      const uint32_t hi_sw128 = (1024u >> 4) | (1u << 14) | (2u << 29);  // SBO 1 KB, sm_100 version, 128B swizzle
      const uint32_t lo_q[2] = {((sQ & 0x3FFFFu) >> 4) | (1u << 16),
                                (((sQ + C::Q_TILE_BYTES) & 0x3FFFFu) >> 4) | (1u << 16)};
      const uint32_t lo_k = ((sKV & 0x3FFFFu) >> 4) | (1u << 16);  // K-major, LBO 16 B
      const uint32_t lo_v = ((sKV & 0x3FFFFu) >> 4) | ((uint32_t)(C::STAGE_BYTES >> 4) << 16);  // MN-major
      auto desc = [&](uint32_t lo) { return ((uint64_t)hi_sw128 << 32) | lo; };
      constexpr uint16_t BOTH = 0x3;
      auto issue_s = [&](int t, int st) {
        const uint32_t kb = lo_k + (uint32_t)st * (C::STAGE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = ((kk >> 2) * C::QBOX_BYTES + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * C::KBOX_BYTES + (kk & 3) * 32) >> 4;
          mma_pair_bf16_ss(tS[t], desc(lo_q[t] + qoff), desc(kb + koff), C::IDESC_S, kk > 0);
        }
      };
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity, abort_flag));
      };
      auto issue_pv_half = [&](int t, int st, bool acc, int h) {
        const uint32_t vb = lo_v + (uint32_t)st * (C::STAGE_BYTES >> 4);
#pragma unroll
        for (int k4 = 0; k4 < TC_BN / 32; ++k4) {
          const int kk = h * (TC_BN / 32) + k4;
          mma_pair_bf16_ts(tO[t], tS[t] + kk * 8, desc(vb + kk * (2048 >> 4)), C::IDESC_PV,
                           (acc || kk > 0) ? 1u : 0u);
        }
      };
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
      if (ok) ok = wait_all(bar_kv_full(0), 0);
      if (ok) {
        tc_fence_after_sync();
        if (elect_one()) {
          issue_s(0, 0);
          tc_commit_pair(bar_s_full(0), BOTH);
          issue_s(1, 0);
          tc_commit_pair(bar_s_full(1), BOTH);
          tc_commit_pair(bar_kv_empty(0), BOTH);
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
          tc_commit_pair(bar_s_full(0), BOTH);
        }
        __syncwarp();
        if (!(ok = pv_tile(1, sv, n - 1 > 0, pp))) break;
        if (elect_one()) {
          tc_commit_pair(bar_kv_empty(sv), BOTH);
          issue_s(1, sk);
          tc_commit_pair(bar_s_full(1), BOTH);
          tc_commit_pair(bar_kv_empty(sk), BOTH);
        }
        __syncwarp();
      }
      if (ok) {
        const uint32_t uv = 2u * (T - 1) + 1u;
        const int sv = uv % C::NSTAGE;
        const uint32_t pv = (uv / C::NSTAGE) & 1u, pp = (uint32_t)(T - 1) & 1u;
        ok = wait_all(bar_kv_full(sv), pv) && pv_tile(0, sv, T - 1 > 0, pp);
        if (ok) {
          if (elect_one()) tc_commit_pair(bar_o_done(0), BOTH);
          __syncwarp();
          ok = pv_tile(1, sv, T - 1 > 0, pp);
        }
        if (ok) {
          if (elect_one()) {
            tc_commit_pair(bar_o_done(1), BOTH);
            tc_commit_pair(bar_kv_empty(sv), BOTH);
          }
          __syncwarp();
        }
      }
      // Drain: every pair MMA is done before either CTA frees its tensor memory.
      if (elect_one()) {
        tc_commit_pair(bar_drain, 0x1);
        mbar_wait_drain(bar_drain, 0);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    regs_increase<TC_REGS_SOFTMAX>();
    const int t = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + (t == 0 ? C::COL_S0 : C::COL_S1) + lane_off;
    const uint32_t tO = tmem + (t == 0 ? C::COL_O0 : C::COL_O1) + lane_off;
    // this CTA's rows of pair tile t: 256 t + 128 cr .. + 127 of the pair's block
    const int64_t tile_row0 = qb.i0 + (int64_t)t * 2 * TC_BM + (int64_t)cr * TC_BM;
    const int64_t li = tile_row0 + row;
    const bool row_valid = li < qb.seg.count;
    const int64_t tq = q_token(pl, qb.seg, li);
    const int64_t tq_tile_min = q_token(pl, qb.seg, tile_row0);
    // The P barriers live in the leader: one arrival per warp at the barrier's address in CTA
    // 0 of the pair (the CTA's own copy for the leader).
    auto arrive_p = [&](uint32_t bar) {
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(bar, 0));
    };
    const float sl2 = pl.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    int n = 0;
    bool ok = true;
    for (int s = 0; s < pl.P && ok; ++s) {
      int c = qb.p - s;
      if (c < 0) c += pl.P;
      for (int sk = 0; sk < nks && ok; ++sk) {
        int ntiles, nfull;
        {
          const Seg ks = segment_of(pl.layout, pl.P, pl.k_seg_len, c, sk);
          ntiles = (int)((visible_prefix(pl, ks, tq_max) + TC_BN - 1) / TC_BN);
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
          {
            const float mx = row_max(sr) * sl2;
            float corr = 1.f;
            bool rescale = false;
            if (m == -INFINITY) {
              m = mx;
            } else if (mx > m + RESCALE_LOG2) {
              corr = ex2_approx(m - mx);
              m = mx;
              l *= corr;
              rescale = true;
            }
            if (__any_sync(0xffffffffu, rescale) && n > 0) rescale_o<D>(tO, corr);
          }
          const float shift = m == -INFINITY ? 0.f : m;
          exp_half(sr, 0, sl2x2, f2_pack(-shift, -shift), pk, sum2a, sum2b);
          RA_TMEM_ST32(tS, pk);
          arrive_p(bar_p_half(t));
          exp_half(sr, 1, sl2x2, f2_pack(-shift, -shift), pk, sum2a, sum2b);
          RA_TMEM_ST32(tS + 32, pk);
          float sa0, sa1, sb0, sb1;
          f2_unpack(sum2a, sa0, sa1);
          f2_unpack(sum2b, sb0, sb1);
          l += (sa0 + sb0) + (sa1 + sb1);
          arrive_p(bar_p_full(t));
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
      if (row_ok && pl.lse != nullptr)
        pl.lse[orow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  // ---- teardown: every pair MMA has finished (the leader drained them) and every
  // cross-CTA arrival has landed before either CTA frees its tensor memory and exits.
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();
  if (warp == TC_WARP_MMA) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem, TC_TMEM_COLS);
  }
}

}  // namespace ra
