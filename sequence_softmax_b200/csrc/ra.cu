// ra.cu -- libra.so: the C ABI of include/ra.h (argument checks, TMA tensor maps, launch
// configuration) and the kernels it launches, compiled as one translation unit for sm_100a.
#include <math.h>
#include <mutex>
#include <stdio.h>

#include <nvtx3/nvToolsExt.h>  // header-only; a profiler that is attached sees one range per call

#include "common.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "keybound.cuh"
#include "merge.cuh"
#include "bwd.cuh"
#include "bwd_tc.cuh"
#include "bwd_dq_tc.cuh"

namespace ra {

// Failure-detection self-test: one thread waits on a barrier that nothing signals, through
// the same bounded wait the attention kernel uses, and gives up after limit_ns.
__global__ void selftest_wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
}

namespace {

// An NVTX range over one entry point (named after it) for timeline tools; without a tool
// attached the push and pop are no-ops.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ---- cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D view of a [BH, rows, d] bf16 buffer as (d, S, rows / S, BH): a box of 64 columns x
// 1 x 128 rows x 1 selects 128 rows spaced S apart (S = P for the striped layout, else 1).
bool make_tile_map(CUtensorMap* map, const void* base, int BH, int64_t rows, int d, int S) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)S, (cuuint64_t)(rows / S), (cuuint64_t)BH};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)S * d * 2, (cuuint64_t)rows * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)TC_BN, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Whether the byte ranges [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void* a, int64_t na, const void* b, int64_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return a && b && na > 0 && nb > 0 && pa < pb + (uintptr_t)nb && pb < pa + (uintptr_t)na;
}

template <int D>
ra_status launch_tc(const Plan& pl, int S, cudaStream_t stream) {
  using C = TcCfg<D>;
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, pl.q, pl.BH, pl.q_rows, D, S) || !make_tile_map(&mk, pl.k, pl.BH, pl.k_rows, D, S) ||
      !make_tile_map(&mv, pl.v, pl.BH, pl.k_rows, D, S))
    return RA_ERR_CUDA;
  // The dynamic shared-memory opt-in is a per-device function attribute: set it once per device.
  static bool attr_done[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> g(mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
    if (dev < 0 || dev >= 64) return RA_ERR_UNSUPPORTED;
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(attn_fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
          cudaSuccess)
        return RA_ERR_CUDA;
      attr_done[dev] = true;
    }
  }
  const int64_t nb = (pl.q_seg_len + 2 * TC_BM - 1) / (2 * TC_BM);
  const int64_t units = nb * (int64_t)pl.P * num_segments(pl.layout);
  const int64_t grid = units * pl.BH;
  if (grid <= 0) return RA_OK;
  if (grid > 0x7FFFFFFFll) return RA_ERR_UNSUPPORTED;
  attn_fwd_tc_kernel<D><<<(unsigned)grid, TC_THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, pl);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// Chunks per head of the key-norm passes: about KB_TARGET_BLOCKS blocks in all, at least 16
// per head where the keys allow, and a one-dimensional grid below 2^31 blocks.
int key_chunks(int64_t BH, int64_t rows) {
  int64_t C = (KB_TARGET_BLOCKS + BH - 1) / BH;
  if (C < 16) C = 16;
  if (C > KB_MAX_CHUNKS) C = KB_MAX_CHUNKS;
  if (C * BH > 0x7FFFFFFFll) C = 0x7FFFFFFFll / BH;
  if (C > rows) C = rows;
  return (int)C;
}

// The two passes of keybound.cuh: every lse slot of a head gets the head's largest key norm,
// with O rows as scratch in between. bf16 only (the tensor-core forward reads the bound).
template <int D>
ra_status launch_key_bound(const Plan& pl, cudaStream_t stream) {
  const int C = key_chunks(pl.BH, pl.k_rows);
  if (pl.k_rows != pl.q_rows || C < 1) return RA_ERR_UNSUPPORTED;
  const int64_t o_row_bytes = (int64_t)D * 2;
  key_norm_chunk_kernel<D><<<(unsigned)((int64_t)C * pl.BH), KB_THREADS, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(pl.k), pl.k_rows, C, pl.o, o_row_bytes);
  int64_t G = (pl.q_rows + 4 * KB_THREADS - 1) / (4 * KB_THREADS);  // blocks per head in pass 2
  if (G > 1024) G = 1024;
  if (G * pl.BH > 0x7FFFFFFFll) G = 0x7FFFFFFFll / pl.BH;
  key_norm_spread_kernel<<<(unsigned)(G * pl.BH), KB_THREADS, 0, stream>>>(pl.o, o_row_bytes, pl.q_rows, C, (int)G,
                                                                            pl.lse);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status launch_attention(const Plan& pl, ra_dtype dt, int S, cudaStream_t stream) {
  if (dt == RA_BF16) {
    if (pl.d == 128) return launch_tc<128>(pl, S, stream);
    if (pl.d == 64) return launch_tc<64>(pl, S, stream);
    return RA_ERR_UNSUPPORTED;
  }
  const int64_t rows_per_pos = pl.q_seg_len * num_segments(pl.layout);
  const int64_t gx = (rows_per_pos + SIMT_WARPS - 1) / SIMT_WARPS;
  if (gx <= 0) return RA_OK;
  if (gx > 0x7FFFFFFFll || pl.P > 65535 || pl.BH > 65535) return RA_ERR_UNSUPPORTED;
  dim3 grid((unsigned)gx, (unsigned)pl.P, (unsigned)pl.BH);
  attn_fwd_simt_f32_kernel<<<grid, SIMT_WARPS * 32, 0, stream>>>(pl, rows_per_pos);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// Sets the dynamic shared-memory opt-in of `fn` once per device.
template <class K>
ra_status set_smem_attr_once(K* fn, int bytes, bool (&done)[64]) {
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return RA_ERR_UNSUPPORTED;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return RA_ERR_CUDA;
    done[dev] = true;
  }
  return RA_OK;
}

// Both tensor-core gradient kernels of one plan: key-stationary dK/dV, then query-stationary dQ.
template <int D>
ra_status launch_bwd_tc(const BwdPlan& pl, int S, cudaStream_t stream) {
  CUtensorMap mq, mk, mv, mdo;
  if (!make_tile_map(&mq, pl.q, pl.BH, pl.q_rows, D, S) || !make_tile_map(&mk, pl.k, pl.BH, pl.k_rows, D, S) ||
      !make_tile_map(&mv, pl.v, pl.BH, pl.k_rows, D, S) || !make_tile_map(&mdo, pl.d_o, pl.BH, pl.q_rows, D, S))
    return RA_ERR_CUDA;
  static bool done_kv[64] = {}, done_q[64] = {};
  ra_status st = set_smem_attr_once(attn_bwd_dkdv_tc_kernel<D>, BwCfg<D>::SMEM_BYTES, done_kv);
  if (st != RA_OK) return st;
  st = set_smem_attr_once(attn_bwd_dq_tc_kernel<D>, BqCfg<D>::SMEM_BYTES, done_q);
  if (st != RA_OK) return st;
  const int64_t segs = (int64_t)pl.P * num_segments(pl.layout);
  const int64_t grid_kv = (pl.k_seg_len + BWD_TILE - 1) / BWD_TILE * segs * pl.BH;
  const int64_t grid_q = (pl.q_seg_len + BWD_TILE - 1) / BWD_TILE * segs * pl.BH;
  if (grid_kv > 0x7FFFFFFFll || grid_q > 0x7FFFFFFFll) return RA_ERR_UNSUPPORTED;
  if (grid_kv > 0)
    attn_bwd_dkdv_tc_kernel<D><<<(unsigned)grid_kv, BW_THREADS, BwCfg<D>::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, pl);
  if (grid_q > 0)
    attn_bwd_dq_tc_kernel<D><<<(unsigned)grid_q, BQ_THREADS, BqCfg<D>::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, pl);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// The gradient kernels of one plan: the two tensor-core kernels for bf16, the two fp32
// kernels otherwise. S = row spacing of the striped view (P) or 1.
ra_status launch_backward(const BwdPlan& pl, ra_dtype dt, int S, cudaStream_t stream) {
  if (dt == RA_BF16) {
    if (pl.d == 128) return launch_bwd_tc<128>(pl, S, stream);
    if (pl.d == 64) return launch_bwd_tc<64>(pl, S, stream);
    return RA_ERR_UNSUPPORTED;
  }
  const int64_t krows = pl.k_seg_len * num_segments(pl.layout);
  const int64_t qrows = pl.q_seg_len * num_segments(pl.layout);
  const int64_t gk = (krows + SIMT_WARPS - 1) / SIMT_WARPS, gq = (qrows + SIMT_WARPS - 1) / SIMT_WARPS;
  if (gk > 0x7FFFFFFFll || gq > 0x7FFFFFFFll || pl.P > 65535 || pl.BH > 65535) return RA_ERR_UNSUPPORTED;
  if (gk > 0) bwd_dkdv_simt_f32_kernel<<<dim3((unsigned)gk, pl.P, pl.BH), SIMT_WARPS * 32, 0, stream>>>(pl, krows);
  if (gq > 0) bwd_dq_simt_f32_kernel<<<dim3((unsigned)gq, pl.P, pl.BH), SIMT_WARPS * 32, 0, stream>>>(pl, qrows);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

// Read and clear the error word in one atomic step: a bit that a kernel on another stream
// records between a separate read and clear would otherwise be lost.
__device__ unsigned g_error_snapshot = 0;
__global__ void take_error_word_kernel() { g_error_snapshot = atomicExch(&g_error_word, 0u); }

ra_status launch_delta(const void* o, const void* d_o, ra_dtype dt, int64_t rows, int d, float* delta,
                       cudaStream_t stream) {
  if (rows == 0) return RA_OK;
  int64_t blocks = (rows + DELTA_THREADS / 8 - 1) / (DELTA_THREADS / 8);
  if (blocks > (1ll << 20)) blocks = 1ll << 20;
  if (dt == RA_BF16)
    bwd_delta_kernel<true><<<(unsigned)blocks, DELTA_THREADS, 0, stream>>>(o, d_o, rows, d, delta);
  else
    bwd_delta_kernel<false><<<(unsigned)blocks, DELTA_THREADS, 0, stream>>>(o, d_o, rows, d, delta);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status check_dtype_d(ra_dtype dt, int d) {
  if (dt != RA_F32 && dt != RA_BF16) return RA_ERR_INVALID_ARG;
  if (d <= 0) return RA_ERR_INVALID_ARG;
  if (dt == RA_BF16 && d != 64 && d != 128) return RA_ERR_UNSUPPORTED;
  if (dt == RA_F32 && d > SIMT_DMAX) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

// ra_partial and ra_partial_fold: one Q block against one KV chunk, the result written as a
// new partial state (fold == 0) or merged into the caller's (fold == 1).
ra_status partial_impl(const void* q, const void* k, const void* v, ra_dtype dt, int B, int H, int64_t Lq,
                       int64_t Lk, int d, float scale, int causal, int64_t q_tok0, int64_t q_tok_stride,
                       int64_t k_tok0, int64_t k_tok_stride, float* o_partial, float* lse, int fold,
                       const float* k_norm_max, cudaStream_t stream) {
  if (B < 0 || H < 0 || Lq < 0 || Lk < 0) return RA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (q_tok_stride < 1 || k_tok_stride < 1) return RA_ERR_INVALID_ARG;
  ra_status st = check_dtype_d(dt, d);
  if (st != RA_OK) return st;
  if ((int64_t)B * H > 0x7FFFFFFF) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Lq == 0) return RA_OK;
  if (!q || !o_partial || !lse || !aligned16(q) || !aligned16(o_partial) || !aligned16(lse)) return RA_ERR_INVALID_ARG;
  if (Lk == 0) {
    if (fold) return RA_OK;  // nothing to fold in: the state stays as it is
    const int64_t rows = (int64_t)B * H * Lq;
    fill_empty_kernel<<<592, 256, 0, stream>>>(o_partial, lse, rows, d);
    return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
  }
  if (!k || !v || !aligned16(k) || !aligned16(v)) return RA_ERR_INVALID_ARG;
  if (k_norm_max && (reinterpret_cast<uintptr_t>(k_norm_max) & 3u)) return RA_ERR_INVALID_ARG;
  Plan pl{};
  pl.q = q; pl.k = k; pl.v = v; pl.o = o_partial; pl.lse = lse;
  pl.BH = B * H; pl.d = d; pl.P = 1; pl.layout = RA_LAYOUT_CONTIGUOUS; pl.causal = causal; pl.out_f32 = 1;
  pl.fold = fold;
  pl.kmax_head = dt == RA_BF16 ? k_norm_max : nullptr;  // the fp32 kernel always takes the row max
  pl.q_rows = Lq; pl.k_rows = Lk; pl.q_seg_len = Lq; pl.k_seg_len = Lk;
  pl.q_tok0 = q_tok0; pl.q_tok_stride = q_tok_stride; pl.k_tok0 = k_tok0; pl.k_tok_stride = k_tok_stride;
  pl.scale = scale;
  pl.scale_log2 = scale * 1.4426950408889634f;
  return launch_attention(pl, dt, 1, stream);
}

}  // namespace
}  // namespace ra

using namespace ra;

extern "C" {

int ra_abi_version(void) { return RA_ABI_VERSION; }

const char* ra_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID_ARG: return "RA_ERR_INVALID_ARG: invalid size, pointer, alignment or enum";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED: valid but not implemented (dtype / head dim / size)";
    case RA_ERR_CUDA: return "RA_ERR_CUDA: a CUDA runtime or driver call failed";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
    case RA_ERR_DEVICE_BOUNDS: return "RA_ERR_DEVICE_BOUNDS: a checked device index was out of range";
  }
  return "RA_UNKNOWN_STATUS";
}

ra_status ra_get_device_error(cudaStream_t stream) {
  // One host thread at a time: the snapshot variable is shared by all callers of a device.
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return RA_ERR_CUDA;
  take_error_word_kernel<<<1, 1, 0, stream>>>();
  if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpyFromSymbolAsync(&word, g_error_snapshot, sizeof(word), 0, cudaMemcpyDeviceToHost, stream) !=
      cudaSuccess)
    return RA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return RA_ERR_CUDA;
  if (word & DEVERR_TIMEOUT) return RA_ERR_TIMEOUT;
  if (word & DEVERR_BOUNDS) return RA_ERR_DEVICE_BOUNDS;
  return RA_OK;
}

ra_status ra_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream) {
  NvtxRange nvtx_range("ra_selftest_wait_timeout");
  if (limit_ns < 1000000 || limit_ns > 2000000000) return RA_ERR_INVALID_ARG;
  selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_ns);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status ra_partial(const void* q, const void* k, const void* v, ra_dtype dt, int B, int H, int64_t Lq,
                     int64_t Lk, int d, float scale, int causal, int64_t q_tok0, int64_t q_tok_stride,
                     int64_t k_tok0, int64_t k_tok_stride, float* o_partial, float* lse, cudaStream_t stream) {
  NvtxRange nvtx_range("ra_partial");
  return partial_impl(q, k, v, dt, B, H, Lq, Lk, d, scale, causal, q_tok0, q_tok_stride, k_tok0, k_tok_stride,
                      o_partial, lse, 0, nullptr, stream);
}

ra_status ra_partial_fold(const void* q, const void* k, const void* v, ra_dtype dt, int B, int H, int64_t Lq,
                          int64_t Lk, int d, float scale, int causal, int64_t q_tok0, int64_t q_tok_stride,
                          int64_t k_tok0, int64_t k_tok_stride, float* o_state, float* lse_state,
                          const float* k_norm_max, cudaStream_t stream) {
  NvtxRange nvtx_range("ra_partial_fold");
  return partial_impl(q, k, v, dt, B, H, Lq, Lk, d, scale, causal, q_tok0, q_tok_stride, k_tok0, k_tok_stride,
                      o_state, lse_state, 1, k_norm_max, stream);
}

ra_status ra_key_norm_max(const void* k, ra_dtype dt, int B, int H, int64_t Lk, int d, float* k_norm_max,
                          cudaStream_t stream) {
  NvtxRange nvtx_range("ra_key_norm_max");
  if (B < 0 || H < 0 || Lk < 0) return RA_ERR_INVALID_ARG;
  ra_status st = check_dtype_d(dt, d);
  if (st != RA_OK) return st;
  if (dt != RA_BF16) return RA_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH > 0x7FFFFFFF) return RA_ERR_UNSUPPORTED;
  if (BH == 0) return RA_OK;
  if (!k_norm_max || (reinterpret_cast<uintptr_t>(k_norm_max) & 3u)) return RA_ERR_INVALID_ARG;
  if (Lk > 0 && (!k || !aligned16(k))) return RA_ERR_INVALID_ARG;
  if (overlaps(k_norm_max, BH * 4, k, BH * Lk * d * 2)) return RA_ERR_INVALID_ARG;  // the memset would clobber keys
  if (cudaMemsetAsync(k_norm_max, 0, (size_t)BH * sizeof(float), stream) != cudaSuccess) return RA_ERR_CUDA;
  if (Lk == 0) return RA_OK;
  const int C = key_chunks(BH, Lk);
  const unsigned grid = (unsigned)((int64_t)C * BH);
  if (d == 128)
    key_norm_max_kernel<128><<<grid, KB_THREADS, 0, stream>>>(static_cast<const __nv_bfloat16*>(k), Lk, C, k_norm_max);
  else
    key_norm_max_kernel<64><<<grid, KB_THREADS, 0, stream>>>(static_cast<const __nv_bfloat16*>(k), Lk, C, k_norm_max);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status ra_merge(const float* o_parts, const float* lse_parts, int n, int64_t rows, int d, void* o_out,
                   ra_dtype out_dt, float* lse_out, cudaStream_t stream) {
  NvtxRange nvtx_range("ra_merge");
  if (n < 1 || rows < 0 || d < 1 || (d & 3) != 0) return RA_ERR_INVALID_ARG;
  if (out_dt != RA_F32 && out_dt != RA_BF16) return RA_ERR_INVALID_ARG;
  if (n > MERGE_MAX_PARTS) return RA_ERR_UNSUPPORTED;
  if (rows == 0) return RA_OK;
  if (!o_parts || !lse_parts || !o_out || !aligned16(o_parts) || !aligned16(o_out)) return RA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse_parts) & 3u) || (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)))
    return RA_ERR_INVALID_ARG;
  // One group of MERGE_LANES_PER_ROW lanes per row; the kernel is grid-stride beyond the cap.
  int64_t blocks = (rows * MERGE_LANES_PER_ROW + MERGE_THREADS - 1) / MERGE_THREADS;
  if (blocks > (1ll << 22)) blocks = 1ll << 22;
  const unsigned g = (unsigned)blocks;
  const bool bf = out_dt == RA_BF16;
#define RA_MERGE_LAUNCH(CPL)                                                                             \
  (bf ? merge_kernel<true, CPL><<<g, MERGE_THREADS, 0, stream>>>(o_parts, lse_parts, n, rows, d, o_out, lse_out) \
      : merge_kernel<false, CPL><<<g, MERGE_THREADS, 0, stream>>>(o_parts, lse_parts, n, rows, d, o_out, lse_out))
  switch (d) {
    case 32: RA_MERGE_LAUNCH(1); break;
    case 64: RA_MERGE_LAUNCH(2); break;
    case 128: RA_MERGE_LAUNCH(4); break;
    case 256: RA_MERGE_LAUNCH(8); break;
    default: RA_MERGE_LAUNCH(0); break;
  }
#undef RA_MERGE_LAUNCH
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status ra_ring_forward(const void* q, const void* k, const void* v, ra_dtype dt, int B, int H, int64_t N, int d,
                          float scale, int n_chunks, int causal, ra_layout layout, void* o, float* lse,
                          cudaStream_t stream) {
  NvtxRange nvtx_range("ra_ring_forward");
  if (B < 0 || H < 0 || N < 0 || n_chunks < 1) return RA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (layout != RA_LAYOUT_CONTIGUOUS && layout != RA_LAYOUT_STRIPED && layout != RA_LAYOUT_ZIGZAG)
    return RA_ERR_INVALID_ARG;
  const int64_t parts = layout == RA_LAYOUT_ZIGZAG ? 2 * (int64_t)n_chunks : n_chunks;
  if (N % parts != 0) return RA_ERR_INVALID_ARG;
  ra_status st = check_dtype_d(dt, d);
  if (st != RA_OK) return st;
  if ((int64_t)B * H > 0x7FFFFFFF) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return RA_OK;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return RA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return RA_ERR_INVALID_ARG;
  {
    // o and lse are written (and serve as scratch before the attention kernel runs): neither
    // may share memory with an input or with the other.
    const int64_t nt = (int64_t)B * H * N * d * (dt == RA_F32 ? 4 : 2), nl = (int64_t)B * H * N * 4;
    for (const void* in : {q, k, v})
      if (overlaps(o, nt, in, nt) || overlaps(lse, nl, in, nt)) return RA_ERR_INVALID_ARG;
    if (overlaps(lse, nl, o, nt)) return RA_ERR_INVALID_ARG;
  }
  Plan pl{};
  pl.q = q; pl.k = k; pl.v = v; pl.o = o; pl.lse = lse;
  pl.BH = B * H; pl.d = d; pl.P = n_chunks; pl.layout = layout; pl.causal = causal; pl.out_f32 = (dt == RA_F32);
  pl.q_rows = N; pl.k_rows = N;
  pl.q_seg_len = pl.k_seg_len = N / parts;
  pl.q_tok0 = 0; pl.q_tok_stride = 1; pl.k_tok0 = 0; pl.k_tok_stride = 1;
  pl.scale = scale;
  pl.scale_log2 = scale * 1.4426950408889634f;
  const int S = layout == RA_LAYOUT_STRIPED ? n_chunks : 1;
  if (dt == RA_BF16 && lse) {
    // Key-norm bound for the row-max skip: lse and O are scratch until the forward writes them.
    st = d == 128 ? launch_key_bound<128>(pl, stream) : launch_key_bound<64>(pl, stream);
    if (st != RA_OK) return st;
    pl.kbound = 1;
  }
  return launch_attention(pl, dt, S, stream);
}

ra_status ra_backward_delta(const void* o, const void* d_o, ra_dtype dt, int64_t rows, int d, float* delta,
                            cudaStream_t stream) {
  NvtxRange nvtx_range("ra_backward_delta");
  if (rows < 0) return RA_ERR_INVALID_ARG;
  ra_status st = check_dtype_d(dt, d);
  if (st != RA_OK) return st;
  if (rows == 0) return RA_OK;
  if (!o || !d_o || !delta || !aligned16(o) || !aligned16(d_o) || (reinterpret_cast<uintptr_t>(delta) & 3u))
    return RA_ERR_INVALID_ARG;
  return launch_delta(o, d_o, dt, rows, d, delta, stream);
}

ra_status ra_partial_backward(const void* q, const void* k, const void* v, const void* d_o, const float* lse,
                              const float* delta, ra_dtype dt, int B, int H, int64_t Lq, int64_t Lk, int d,
                              float scale, int causal, int64_t q_tok0, int64_t q_tok_stride, int64_t k_tok0,
                              int64_t k_tok_stride, float* dq_acc, float* dk_acc, float* dv_acc,
                              cudaStream_t stream) {
  NvtxRange nvtx_range("ra_partial_backward");
  if (B < 0 || H < 0 || Lq < 0 || Lk < 0) return RA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (q_tok_stride < 1 || k_tok_stride < 1) return RA_ERR_INVALID_ARG;
  ra_status st = check_dtype_d(dt, d);
  if (st != RA_OK) return st;
  if ((int64_t)B * H > 0x7FFFFFFF) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Lq == 0 || Lk == 0) return RA_OK;
  if (!q || !k || !v || !d_o || !lse || !delta || !dq_acc || !dk_acc || !dv_acc) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) || !aligned16(dq_acc) ||
      !aligned16(dk_acc) || !aligned16(dv_acc) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(delta) & 3u))
    return RA_ERR_INVALID_ARG;
  BwdPlan pl{};
  pl.q = q; pl.k = k; pl.v = v; pl.d_o = d_o; pl.lse = lse; pl.delta = delta;
  pl.dq = dq_acc; pl.dk = dk_acc; pl.dv = dv_acc;
  pl.BH = B * H; pl.d = d; pl.P = 1; pl.layout = RA_LAYOUT_CONTIGUOUS; pl.causal = causal;
  pl.accumulate = 1;
  pl.q_rows = Lq; pl.k_rows = Lk; pl.q_seg_len = Lq; pl.k_seg_len = Lk;
  pl.q_tok0 = q_tok0; pl.q_tok_stride = q_tok_stride; pl.k_tok0 = k_tok0; pl.k_tok_stride = k_tok_stride;
  pl.scale = scale;
  pl.scale_log2 = scale * 1.4426950408889634f;
  return launch_backward(pl, dt, 1, stream);
}

int64_t ra_ring_backward_workspace_bytes(ra_dtype dt, int B, int H, int64_t N, int d) {
  (void)dt;
  if (B < 0 || H < 0 || N < 0 || d < 1) return -1;
  return (int64_t)B * H * N * 4;  // D, one fp32 per query row
}

ra_status ra_ring_backward(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                           const float* lse, ra_dtype dt, int B, int H, int64_t N, int d, float scale,
                           int n_chunks, int causal, ra_layout layout, void* dq, void* dk, void* dv,
                           void* workspace, int64_t workspace_bytes, cudaStream_t stream) {
  NvtxRange nvtx_range("ra_ring_backward");
  if (B < 0 || H < 0 || N < 0 || n_chunks < 1) return RA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return RA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID_ARG;
  if (layout != RA_LAYOUT_CONTIGUOUS && layout != RA_LAYOUT_STRIPED && layout != RA_LAYOUT_ZIGZAG)
    return RA_ERR_INVALID_ARG;
  const int64_t parts = layout == RA_LAYOUT_ZIGZAG ? 2 * (int64_t)n_chunks : n_chunks;
  if (N % parts != 0) return RA_ERR_INVALID_ARG;
  ra_status st = check_dtype_d(dt, d);
  if (st != RA_OK) return st;
  if ((int64_t)B * H > 0x7FFFFFFF) return RA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) return RA_OK;
  if (workspace_bytes < ra_ring_backward_workspace_bytes(dt, B, H, N, d)) return RA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !d_o || !lse || !dq || !dk || !dv || !workspace) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return RA_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)B * H * N;
  float* delta = static_cast<float*>(workspace);
  st = launch_delta(o, d_o, dt, rows, d, delta, stream);
  if (st != RA_OK) return st;
  BwdPlan pl{};
  pl.q = q; pl.k = k; pl.v = v; pl.d_o = d_o; pl.lse = lse; pl.delta = delta;
  pl.dq = dq; pl.dk = dk; pl.dv = dv;
  pl.BH = B * H; pl.d = d; pl.P = n_chunks; pl.layout = layout; pl.causal = causal;
  pl.accumulate = 0;
  pl.q_rows = N; pl.k_rows = N;
  pl.q_seg_len = pl.k_seg_len = N / parts;
  pl.q_tok0 = 0; pl.q_tok_stride = 1; pl.k_tok0 = 0; pl.k_tok_stride = 1;
  pl.scale = scale;
  pl.scale_log2 = scale * 1.4426950408889634f;
  return launch_backward(pl, dt, layout == RA_LAYOUT_STRIPED ? n_chunks : 1, stream);
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// ra_ring_backward_noalloc: the workspace of ra_ring_backward in a static device array, so
// that callers who cannot allocate device memory still get the backward pass.
// ------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[RA_NOALLOC_SCRATCH_BYTES];

namespace {

// cuCtxGetCurrent through the runtime's driver entry point (no -lcuda).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of this device's copy of g_noalloc_scratch (host code only sees a
// host-side stand-in for the name). Looked up with the device current, once per device and
// CUDA context: the address belongs to the context the library's module is loaded in, so a
// new context on the device (after cudaDeviceReset, or another context made current) gets
// a fresh lookup instead of a stale address.
ra_status noalloc_scratch(void** out) {
  static void* addr[64] = {};
  static CUcontext owner[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return RA_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  // No context current yet (nothing has touched this device): the lookup binds the
  // runtime's context, which is then recorded as the owner.
  if (ctx == nullptr || addr[dev] == nullptr || owner[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return RA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return RA_ERR_CUDA;
    addr[dev] = p;
    owner[dev] = ctx;
  }
  *out = addr[dev];
  return RA_OK;
}

}  // namespace

extern "C" ra_status ra_ring_backward_noalloc(const void* q, const void* k, const void* v, const void* o,
                                              const void* d_o, const float* lse, ra_dtype dt, int B, int H,
                                              int64_t N, int d, float scale, int n_chunks, int causal,
                                              ra_layout layout, void* dq, void* dk, void* dv,
                                              cudaStream_t stream) {
  NvtxRange nvtx_range("ra_ring_backward_noalloc");
  const int64_t need = ra_ring_backward_workspace_bytes(dt, B, H, N, d);
  if (need < 0) return RA_ERR_INVALID_ARG;
  if (need > RA_NOALLOC_SCRATCH_BYTES) return RA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  const ra_status st = noalloc_scratch(&ws);
  if (st != RA_OK) return st;
  return ra_ring_backward(q, k, v, o, d_o, lse, dt, B, H, N, d, scale, n_chunks, causal, layout, dq, dk, dv, ws,
                          RA_NOALLOC_SCRATCH_BYTES, stream);
}
