/*
 * ra.h -- C ABI of libra.so: ring attention (forward, merge and backward) on one NVIDIA B200.
 *
 * Ring attention computes exact softmax attention while a query block stays fixed and
 * key/value chunks arrive one at a time; each chunk's partial result is folded into a
 * running online-softmax state (running max m, running sum l, running output o), so the
 * final output equals full attention. On one GPU the ring becomes an ordered loop over
 * KV chunks inside one kernel.
 *
 * Sources (web pages, cited by title and section):
 *   [BLOG]     "Ring Attention 논문 분석" (youngju.dev), listings blockwise_attention,
 *              ring_attention_forward, ring_attention_causal_step.
 *   [GLOSSARY] "Ring Attention" glossary (ultralytics.com), section "How Ring Attention works".
 *   [LECTURE]  gpumode lecture 013 notes (brianyu43.github.io): log-sum-exp associativity,
 *              causal load imbalance and striped placement.
 *   [CARD]     "Context Parallelism" card (llm-engineer.pages.dev): online softmax (m, l, o),
 *              causal imbalance and zig-zag placement.
 *
 * Conventions shared by every entry point
 *   - Pointers are device pointers owned by the caller, contiguous, 16-byte aligned.
 *     Tensors are row-major [B, H, rows, d] with d innermost (the head dimension).
 *     ra_partial's k, v and ra_partial_backward's k, v, dk_acc, dv_acc may address another
 *     GPU's memory mapped into this process (CUDA IPC with peer access): the kernels read
 *     it with plain per-CTA TMA loads (each CTA fetches its own tiles) and writes it with
 *     plain stores.
 *   - Calls are asynchronous on `stream`. The return value reports argument and launch
 *     errors only; nothing has been launched when it is not RA_OK. Errors found on the
 *     device (a bounded wait that ran out) are reported by ra_get_device_error().
 *   - The library allocates no device memory. Its only device state is static variables of
 *     the library image, per device: the 32-bit error word (and the copy that
 *     ra_get_device_error reads it through) and the scratch array of
 *     ra_ring_backward_noalloc.
 *   - scale is the softmax scale, normally d^-1/2 ([BLOG] blockwise_attention; [GLOSSARY]).
 *   - Causal masking keeps key token j for query token i iff j <= i: the diagonal is kept
 *     ([BLOG] ring_attention_causal_step masks triu(diagonal=1)).
 *   - lse values are natural-log log-sum-exp of the scaled scores, fp32. A query row that
 *     sees no key has lse = -inf and output 0.
 *   - Supported: dt = RA_BF16 with d in {64, 128} (tcgen05 tensor-core kernel), or
 *     dt = RA_F32 with 1 <= d <= 128 (fp32 CUDA-core kernel). Anything else returns
 *     RA_ERR_UNSUPPORTED.
 */
#ifndef RA_H
#define RA_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RA_OK = 0,
    RA_ERR_INVALID_ARG = 1,   /* a size, pointer, alignment or enum value is invalid */
    RA_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels implement (dtype, d) */
    RA_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed (launch, tensor map) */
    RA_ERR_TIMEOUT = 4,       /* device: a bounded wait inside a kernel ran out */
    RA_ERR_DEVICE_BOUNDS = 5  /* device: a checked index was out of range (checked builds) */
} ra_status;

typedef enum { RA_F32 = 0, RA_BF16 = 1 } ra_dtype;

/* Token -> virtual ring position maps ([LECTURE] striped placement; [CARD] zig-zag). */
typedef enum {
    RA_LAYOUT_CONTIGUOUS = 0, /* position p holds tokens [p N/P, (p+1) N/P) */
    RA_LAYOUT_STRIPED = 1,    /* position p holds tokens t with t mod P == p */
    RA_LAYOUT_ZIGZAG = 2      /* N cut into 2P chunks; position p holds chunks p and 2P-1-p */
} ra_layout;

/*
 * ra_partial -- one query block against one KV chunk ([BLOG] ring_attention_causal_step),
 * returned as a normalised partial state: O_partial = sum_j exp(s_ij - m_i) v_j / l_i and
 * lse_i = m_i + log l_i, with s = q k^T * scale.
 *
 *   q          [B, H, Lq, d]  dtype dt
 *   k, v       [B, H, Lk, d]  dtype dt
 *   causal     0 or 1. Query row i has global token q_tok0 + q_tok_stride * i, key row j has
 *              k_tok0 + k_tok_stride * j (stride 1 for a contiguous chunk, P for a striped
 *              position); key j is visible to query i iff its token <= the query's token.
 *              Token arguments are ignored when causal == 0. Strides must be >= 1.
 *   o_partial  [B, H, Lq, d] fp32, written (rows with no visible key: 0)
 *   lse        [B, H, Lq]    fp32, written (rows with no visible key: -inf)
 *
 * Lq == 0 is a no-op. Lk == 0 writes the empty state for every row.
 */
ra_status ra_partial(const void* q, const void* k, const void* v, ra_dtype dt,
                     int B, int H, int64_t Lq, int64_t Lk, int d, float scale, int causal,
                     int64_t q_tok0, int64_t q_tok_stride, int64_t k_tok0, int64_t k_tok_stride,
                     float* o_partial, float* lse, cudaStream_t stream);

/*
 * ra_partial_fold -- ra_partial whose result is merged, in the same kernel, into a running
 * partial state held by the caller: the per-step update of the ring ([BLOG]
 * ring_attention_forward: the state (m, l, o) is carried from step to step and every new KV
 * chunk is folded into it; [LECTURE] log-sum-exp passage for the merge in (O, lse) form).
 *
 *   q, k, v, dt, B, H, Lq, Lk, d, scale, causal, q_tok0 ... k_tok_stride: as ra_partial
 *   o_state    [B, H, Lq, d]  fp32, read and written: the normalised state O
 *   lse_state  [B, H, Lq]     fp32, read and written: the state's lse (-inf: nothing seen yet)
 *   k_norm_max [B, H]         fp32 or NULL: the largest norm of each head's keys of this
 *                             chunk, or any larger value (ra_key_norm_max writes it)
 *
 * With k_norm_max NULL, afterwards (o_state, lse_state) equal, bit for bit, what ra_partial
 * into a scratch state followed by ra_merge (n = 2, parts [state, new], fp32 output) would
 * leave, without the scratch state, the merge launch or the copies back. With k_norm_max
 * (bf16 only; ignored for fp32), a warp skips a tile's row max as ra_ring_forward does, which
 * changes only the rounding; |V| must then stay below 2^72. A value below a key's true norm
 * breaks that guarantee: exponentials may then overflow. Start a ring with o_state = 0 and
 * lse_state = -inf. Lq == 0 and Lk == 0 leave the state as it is. The state must not overlap
 * q, k or v.
 */
ra_status ra_partial_fold(const void* q, const void* k, const void* v, ra_dtype dt,
                          int B, int H, int64_t Lq, int64_t Lk, int d, float scale, int causal,
                          int64_t q_tok0, int64_t q_tok_stride, int64_t k_tok0, int64_t k_tok_stride,
                          float* o_state, float* lse_state, const float* k_norm_max, cudaStream_t stream);

/*
 * ra_key_norm_max -- the largest L2 norm of each head's keys, the key half of the bound
 * |q| max|k| scale log2(e) on a row's scaled scores (Cauchy-Schwarz) that lets the forward
 * keep its running max on a tile: see ra_ring_forward and ra_partial_fold.
 *   k           [B, H, Lk, d]  bf16 (d in {64, 128}); read
 *   k_norm_max  [B, H]         fp32, written: max over j of |k_j|, rounded as fp32 sums of
 *                              squares and a square root (+inf if a key holds inf or NaN;
 *                              0 when Lk == 0)
 * RA_ERR_UNSUPPORTED for fp32 keys; RA_ERR_INVALID_ARG if k_norm_max overlaps k. The array
 * is first set to zero on `stream` (a memset, no allocation). The pages have no counterpart:
 * it only feeds the skip.
 */
ra_status ra_key_norm_max(const void* k, ra_dtype dt, int B, int H, int64_t Lk, int d, float* k_norm_max,
                          cudaStream_t stream);

/*
 * ra_merge -- lse-weighted combination of n partial states, from the associativity
 * lse(x) = lse([lse(x1), lse(x2)]) ([LECTURE] log-sum-exp passage):
 *   L = max_i lse_i + log sum_i exp(lse_i - max_i lse_i),   O = sum_i exp(lse_i - L) O_i.
 * Parts with lse = -inf have weight 0; a row whose parts are all -inf gets O = 0, L = -inf.
 *
 *   o_parts    [n, rows, d]  fp32 (for attention outputs rows = B*H*Lq)
 *   lse_parts  [n, rows]     fp32
 *   o_out      [rows, d]     dtype out_dt (RA_F32 or RA_BF16), written
 *   lse_out    [rows]        fp32, written; may be NULL
 *
 * Needs n >= 1, d >= 1 and d % 4 == 0 (16-byte vector access). rows == 0 is a no-op.
 */
ra_status ra_merge(const float* o_parts, const float* lse_parts, int n, int64_t rows, int d,
                   void* o_out, ra_dtype out_dt, float* lse_out, cudaStream_t stream);

/*
 * ra_ring_forward -- full exact attention by the ring ([BLOG] ring_attention_forward;
 * [GLOSSARY] "How Ring Attention works"): the sequence is split over n_chunks virtual
 * positions by `layout`; position p keeps its query tokens and at step s = 0..P-1 folds the
 * KV tokens of position (p - s) mod P into its running (m, l, o) state. With causal != 0,
 * KV tiles wholly in the future of a query tile are skipped and the rest are masked
 * elementwise. Q, K, V, O and lse are in natural token order for every layout: the layout
 * changes the work partition and the visiting order, not the result.
 *
 *   q, k, v    [B, H, N, d]  dtype dt
 *   o          [B, H, N, d]  dtype dt, written
 *   lse        [B, H, N]     fp32, written; may be NULL
 *
 * Needs N % n_chunks == 0 (N % (2 n_chunks) == 0 for zig-zag) and n_chunks >= 1.
 * N == 0, B == 0 or H == 0 is a no-op. o and lse must not overlap q, k, v or each other
 * (RA_ERR_INVALID_ARG).
 *
 * Row-max skip (bf16 with lse given): two short kernels first write each
 * head's largest key norm into every lse slot of the head, using the first rows of o as
 * scratch; the attention kernel reads its rows' slots before it writes them. A warp then
 * skips a tile's row max when |q| max|k| scale log2(e) of each of its rows is within 24
 * log2 units of the running max: no exponential can exceed 2^24, and the result is exact up
 * to rounding as with the max. Until the call completes on `stream`, o and lse hold these
 * intermediate values. Keep |V| below 2^72 (fp32 O stays finite with exponentials <= 2^24).
 */
ra_status ra_ring_forward(const void* q, const void* k, const void* v, ra_dtype dt,
                          int B, int H, int64_t N, int d, float scale, int n_chunks, int causal,
                          ra_layout layout, void* o, float* lse, cudaStream_t stream);

/*
 * Backward pass ([BLOG] ring_attention_backward, with the causal mask the listing leaves
 * out). With P = exp(S - lse) (S = q k^T * scale, lse from the forward) and upstream
 * gradient dO of the output O:
 *   dV = P^T dO,   dP = dO V^T,   D_i = sum_e dO_ie O_ie,
 *   dS = P * (dP - D) * scale,   dQ = dS K,   dK = dS^T Q.
 * In the ring, each position keeps Q, dO, O, lse and its dQ; the KV chunk travels with its
 * dK, dV contributions, which are summed at the chunk's owner. The listing returns them
 * with a reduce whose root differs per rank; that sum is the reading implemented here.
 */

/*
 * ra_backward_delta -- the row term D_i = sum_e dO_ie O_ie (fp32 accumulation).
 *   o, d_o     [rows, d]  dtype dt (O of the forward and its upstream gradient)
 *   delta      [rows]     fp32, written
 * Same dtype / d support as the forward. rows == 0 is a no-op.
 */
ra_status ra_backward_delta(const void* o, const void* d_o, ra_dtype dt, int64_t rows, int d,
                            float* delta, cudaStream_t stream);

/*
 * ra_partial_backward -- one query block against one KV chunk: adds this pair's
 * contributions to three fp32 accumulators (the caller zeroes them first):
 *   dq_acc += dS K      [B, H, Lq, d] fp32
 *   dk_acc += dS^T Q    [B, H, Lk, d] fp32
 *   dv_acc += P^T dO    [B, H, Lk, d] fp32
 *   q, d_o     [B, H, Lq, d]  dtype dt
 *   k, v       [B, H, Lk, d]  dtype dt
 *   lse        [B, H, Lq]     fp32, the FINAL log-sum-exp of each query row (over all keys,
 *                             e.g. from ra_ring_forward or ra_merge), so that P is the true
 *                             softmax probability
 *   delta      [B, H, Lq]     fp32, from ra_backward_delta on the final O
 *   causal and the token arguments as in ra_partial.
 * Every row of dq_acc, dk_acc and dv_acc is read, added to and written by the one CTA that
 * owns it (a key-stationary kernel for dK/dV, a query-stationary one for dQ), so results are
 * bitwise reproducible. Lq == 0 or Lk == 0 is a no-op.
 */
ra_status ra_partial_backward(const void* q, const void* k, const void* v, const void* d_o,
                              const float* lse, const float* delta, ra_dtype dt,
                              int B, int H, int64_t Lq, int64_t Lk, int d, float scale, int causal,
                              int64_t q_tok0, int64_t q_tok_stride, int64_t k_tok0, int64_t k_tok_stride,
                              float* dq_acc, float* dk_acc, float* dv_acc, cudaStream_t stream);

/*
 * ra_ring_backward_workspace_bytes -- bytes of the caller-owned workspace ra_ring_backward
 * needs: B*H*N*4 (the row term D, fp32), for either dtype. Returns -1 for negative sizes.
 */
int64_t ra_ring_backward_workspace_bytes(ra_dtype dt, int B, int H, int64_t N, int d);

/*
 * ra_ring_backward -- gradients of ra_ring_forward's output, by the ring: KV chunk c meets
 * the query positions c, c+1, ... (mod P) in turn and each key tile's dK, dV accumulate on
 * chip; each query tile's dQ accumulates on chip over the KV tiles it sees in the forward's
 * order. Three launches on `stream`: D, the dK/dV kernel, the dQ kernel. Deterministic.
 *   q, k, v, o, d_o  [B, H, N, d]  dtype dt, natural token order
 *   lse              [B, H, N]     fp32 (from ra_ring_forward)
 *   dq, dk, dv       [B, H, N, d]  dtype dt, written
 *   workspace        device memory of at least ra_ring_backward_workspace_bytes() bytes,
 *                    16-byte aligned, owned by the caller; its contents are scratch
 * Shape rules as ra_ring_forward. RA_ERR_INVALID_ARG if workspace_bytes is too small.
 */
ra_status ra_ring_backward(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                           const float* lse, ra_dtype dt, int B, int H, int64_t N, int d, float scale,
                           int n_chunks, int causal, ra_layout layout, void* dq, void* dk, void* dv,
                           void* workspace, int64_t workspace_bytes, cudaStream_t stream);

/*
 * ra_ring_backward_noalloc -- ra_ring_backward for callers that must not allocate device
 * memory themselves. Examples: a plugin or custom operator inside another runtime that hands
 * it device pointers but owns every byte of the GPU through its own pool allocator (a raw
 * cudaMalloc there takes memory the pool counts as free), or a latency-critical loop where
 * cudaMalloc/cudaFree, which may synchronise the whole device, cannot run. The paper has no
 * counterpart: this is an interface convenience, not part of the method.
 *
 * The scratch (the row term D, 4 bytes per query row) lives in one static device array of
 * RA_NOALLOC_SCRATCH_BYTES bytes inside the library. Every GPU that loads the library holds
 * it until the process exits. Problems whose ra_ring_backward_workspace_bytes() exceeds it
 * (B*H*N > 16777216 rows) return RA_ERR_UNSUPPORTED without launching anything.
 *
 * The first call on a device (in a given CUDA context) looks up the array's device address,
 * with that device current, and keeps it; make that first call before any stream capture.
 * A later call from another context on the same device (after cudaDeviceReset, or with a
 * different context made current through the driver API) looks the address up again. All
 * calls on a device share the one array: two calls whose work overlaps on the GPU
 * (different streams, or different host threads without ordering) race on it and corrupt
 * each other's gradients, so order them on one stream or synchronise between them. Nothing
 * needs clearing: every call overwrites each scratch entry it reads (the row term of each of
 * its B*H*N query rows) before reading it, so what an earlier call left there never matters.
 * Arguments, layouts and outputs are those of ra_ring_backward.
 */
#define RA_NOALLOC_SCRATCH_BYTES (64ll * 1024 * 1024)
ra_status ra_ring_backward_noalloc(const void* q, const void* k, const void* v, const void* o,
                                   const void* d_o, const float* lse, ra_dtype dt, int B, int H,
                                   int64_t N, int d, float scale, int n_chunks, int causal,
                                   ra_layout layout, void* dq, void* dk, void* dv,
                                   cudaStream_t stream);

/* Static, human-readable name of a status code (never NULL). */
const char* ra_status_string(ra_status status);

/*
 * ra_get_device_error -- synchronises `stream`, then reads and clears this device's error
 * word in one atomic exchange on the device (an error recorded meanwhile by a kernel on
 * another stream is reported by this call or the next, never lost). Returns RA_OK if no
 * kernel recorded an error since the last call, RA_ERR_TIMEOUT or RA_ERR_DEVICE_BOUNDS if
 * one did, RA_ERR_CUDA if the synchronisation or the exchange failed. Calls from several
 * host threads are serialised.
 */
ra_status ra_get_device_error(cudaStream_t stream);

/*
 * ra_selftest_wait_timeout -- exercises the library's failure detection without faulting
 * the GPU: launches one block whose thread waits on a shared-memory barrier that nothing
 * signals, through the same bounded wait every kernel here uses. After limit_ns of device
 * time (1 ms to 2 s) the wait gives up, records RA_ERR_TIMEOUT in the device error word and
 * the kernel returns; the context stays usable. Read the outcome with
 * ra_get_device_error(). Returns RA_ERR_INVALID_ARG for a limit outside the range.
 */
ra_status ra_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream);

/* ABI version of this header (incremented on any signature change); ra_abi_version()
 * returns the version the library was built with, so a caller can compare the two. */
#define RA_ABI_VERSION 4
int ra_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RA_H */
