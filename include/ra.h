/*
 * ra.h -- C ABI of libra.so: the forward hot path of ring attention on one NVIDIA B200.
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
 *   - Calls are asynchronous on `stream`. The return value reports argument and launch
 *     errors only; nothing has been launched when it is not RA_OK. Errors found on the
 *     device (a bounded wait that ran out) are reported by ra_get_device_error().
 *   - The library allocates no device memory. Its only device state is one 32-bit error
 *     word per device, a static variable of the library image.
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
 * N == 0, B == 0 or H == 0 is a no-op.
 */
ra_status ra_ring_forward(const void* q, const void* k, const void* v, ra_dtype dt,
                          int B, int H, int64_t N, int d, float scale, int n_chunks, int causal,
                          ra_layout layout, void* o, float* lse, cudaStream_t stream);

/* Static, human-readable name of a status code (never NULL). */
const char* ra_status_string(ra_status status);

/*
 * ra_get_device_error -- synchronises `stream`, then reads and clears this device's error
 * word. Returns RA_OK if no kernel recorded an error since the last call, RA_ERR_TIMEOUT
 * or RA_ERR_DEVICE_BOUNDS if one did, RA_ERR_CUDA if the synchronisation itself failed.
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

/* ABI version of this header (incremented on any signature change). */
int ra_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RA_H */
