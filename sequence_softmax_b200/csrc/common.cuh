// common.cuh -- shared device helpers of libra.so: the problem plan (token layout and
// ring visiting order), the device error word, bounded mbarrier waits, and thin inline-PTX
// wrappers for TMA, mbarriers and the tcgen05 tensor-core / tensor-memory instructions of
// sm_100a. Written for B200 only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ra.h"

namespace ra {

// ------------------------------------------------------------------------------------
// Device error word. One per device (a static variable of the library image). Kernels
// set bits with atomicOr; ra_get_device_error() reads and clears it.
// ------------------------------------------------------------------------------------
enum : unsigned { DEVERR_TIMEOUT = 1u, DEVERR_BOUNDS = 2u };
__device__ unsigned g_error_word = 0;

__device__ __forceinline__ void record_error(unsigned bits) { atomicOr(&g_error_word, bits); }

// Checked builds (compiled with -DRA_DEBUG_BOUNDS, as libra_checked.so): the kernels test
// every global row index and every TMA start row they compute against the buffer it
// addresses. A failed test records DEVERR_BOUNDS in the error word (RA_ERR_DEVICE_BOUNDS on
// the host) and the access is skipped; TMA loads, whose out-of-range parts read as zeros,
// are still issued so that no wait is left without its data. The default build compiles
// the tests away.
#ifdef RA_DEBUG_BOUNDS
__device__ __forceinline__ bool in_bounds(bool ok) {
  if (!ok) record_error(DEVERR_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(bool) { return true; }
#endif

// Time limit of every spin on an mbarrier (nanoseconds of %globaltimer). A correct kernel
// waits microseconds; the limit turns a lost arrival into an error instead of a hang.
#ifndef RA_WAIT_LIMIT_NS
#define RA_WAIT_LIMIT_NS 2000000000ull
#endif

// ------------------------------------------------------------------------------------
// Problem plan: where each virtual ring position's tokens live and in which order the
// KV chunks are visited.
//
// Both Q and K/V sides are lists of "segments": a run of `count` rows at memory rows
// row0 + stride * i (i = 0..count-1) of the per-head buffer. The global token of memory
// row r is tok0 + tok_stride * r (identity for ring_forward, where tensors are in
// natural token order; explicit for ra_partial).
//   contiguous: position p = one segment, row0 = p * len, stride 1
//   striped:    position p = one segment, row0 = p, stride P
//   zig-zag:    position p = two segments, chunks p and 2P-1-p of length len, stride 1
// Ring order: position p visits position (p - s) mod P at step s = 0..P-1.
// ------------------------------------------------------------------------------------
struct Plan {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int BH;            // batch * heads
  int d;             // head dimension
  int P;             // virtual ring positions (1 for ra_partial)
  int layout;        // ra_layout
  int causal;
  int out_f32;       // 1: O written as fp32 (partial states); 0: O in the input dtype
  int fold;          // 1: o / lse hold a running state that the result is merged into
  int kbound;        // 1: lse holds each row's max key norm of its head (keybound.cuh)
  const float* kmax_head;  // or, when not null: the max key norm of each head [BH]
  int64_t q_rows;    // rows per head in the Q / O buffers
  int64_t k_rows;    // rows per head in the K / V buffers
  int64_t q_seg_len; // rows per Q segment
  int64_t k_seg_len; // rows per K segment
  int64_t q_tok0, q_tok_stride, k_tok0, k_tok_stride;
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e): scores are exponentiated with exp2
};

struct Seg {
  int64_t row0, stride, count;
};

__host__ __device__ __forceinline__ int num_segments(int layout) {
  return layout == RA_LAYOUT_ZIGZAG ? 2 : 1;
}

__host__ __device__ __forceinline__ Seg segment_of(int layout, int P, int64_t seg_len, int p, int si) {
  Seg s;
  s.count = seg_len;
  if (layout == RA_LAYOUT_STRIPED) {
    s.row0 = p;
    s.stride = P;
  } else if (layout == RA_LAYOUT_ZIGZAG) {
    s.row0 = (si == 0 ? (int64_t)p : (int64_t)(2 * P - 1 - p)) * seg_len;
    s.stride = 1;
  } else {
    s.row0 = (int64_t)p * seg_len;
    s.stride = 1;
  }
  return s;
}

// Number of keys of segment `ks` (from its start) that can be visible to a query whose
// token is <= tq_max, i.e. the keys whose token <= tq_max.
__host__ __device__ __forceinline__ int64_t visible_prefix(const Plan& pl, const Seg& ks, int64_t tq_max) {
  if (!pl.causal) return ks.count;
  const int64_t t0 = pl.k_tok0 + pl.k_tok_stride * ks.row0;
  const int64_t ts = pl.k_tok_stride * ks.stride;
  if (tq_max < t0) return 0;
  int64_t n = (tq_max - t0) / ts + 1;
  return n < ks.count ? n : ks.count;
}

// ------------------------------------------------------------------------------------
// PTX wrappers (sm_100a).
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase of parity `parity` of barrier `bar` has completed. Gives up (and
// returns false) when the CTA's abort flag is set, or when RA_WAIT_LIMIT_NS passes, in
// which case it records a timeout in the device error word and sets the abort flag so the
// CTA's other waits give up at once.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = RA_WAIT_LIMIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        record_error(DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait used only while draining at exit: ignores the abort flag (the awaited
// operation -- a TMA load or an MMA already issued -- completes on its own).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > RA_WAIT_LIMIT_NS) {
      record_error(DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 4-D tiled TMA load of one box into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tensor memory (TMEM) ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by this thread is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], A read from tensor memory (bf16 pairs per column).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D, shape M x N,
// A K-major, B K-major or MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4)                              // D format: f32
         | (1u << 7)                            // A format: bf16
         | (1u << 10)                           // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)       // B major-ness
         | ((uint32_t)(N >> 3) << 17)           // N / 8
         | ((uint32_t)(M >> 4) << 24);          // M / 16
}

// As above with the A operand's major-ness too (bit 15: A MN-major, read from shared memory).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
  return idesc_bf16_f32(M, N, b_mn_major) | ((a_mn_major ? 1u : 0u) << 15);
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy reads
// (tensor-core operand fetches) of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand. Start address, leading
// and stride byte offsets are stored divided by 16; bit 46 is the sm_100 descriptor
// version; bits 61-63 = 2 select the 128B swizzle.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// 32 lanes x 32 columns of 32-bit TMEM cells -> 32 registers per thread (thread t of the
// warp reads lane (warp % 4) * 32 + t).
#define RA_TMEM_LD32(taddr, r)                                                                            \
  asm volatile(                                                                                           \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"   \
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                         \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),  \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),         \
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),       \
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),       \
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                                            \
      : "r"(taddr)                                                                                        \
      : "memory")

#define RA_TMEM_ST32(taddr, r)                                                                            \
  asm volatile(                                                                                           \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"\
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),               \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),  \
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),      \
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),     \
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                  \
      : "memory")

#define RA_TMEM_ST16(taddr, r)                                                                            \
  asm volatile(                                                                                           \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"\
      "%16};" ::"r"(taddr),                                                                               \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),  \
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])                   \
      : "memory")

// Registers written by tcgen05.ld are valid only after tcgen05.wait::ld. The empty asm with
// "+r" operands ties later uses of the registers to a point after the wait.
#define RA_REG_FENCE32(r)                                                                                 \
  asm volatile(""                                                                                         \
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),     \
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), \
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),           \
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),           \
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]))

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// One lane of a converged warp (the lowest active one) returns true.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}

// Register reallocation between warpgroups (all four warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction for two lanes of work).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// max of three floats in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Merging a running partial state (lse_state) with a new one (lse_new): L and the two
// weights, with exactly the operations merge_kernel performs for the parts [state, new]
// (max, shift, sum of expf, logf, expf), so that a folded row equals ra_merge's bit for bit
// when the output element is fmaf(w_new, o_new, fmaf(w_state, o_state, 0)).
struct FoldWeights {
  float L, w_state, w_new;
};
__device__ __forceinline__ FoldWeights fold_weights(float lse_state, float lse_new) {
  float mx = -INFINITY;
  mx = fmaxf(mx, lse_state);
  mx = fmaxf(mx, lse_new);
  const float sh = (mx == -INFINITY) ? 0.f : mx;
  float tot = 0.f;
  tot += expf(lse_state - sh);
  tot += expf(lse_new - sh);
  const bool empty = !(tot > 0.f);
  FoldWeights f;
  f.L = empty ? -INFINITY : sh + logf(tot);
  f.w_state = empty ? 0.f : expf(lse_state - f.L);
  f.w_new = empty ? 0.f : expf(lse_new - f.L);
  return f;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace ra
