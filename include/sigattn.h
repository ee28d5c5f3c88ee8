/*
 * sigattn.h -- C ABI of the B200 (sm_100a) sigmoid-attention library.
 *
 * The library computes bidirectional sigmoid attention over ragged, padded
 * batches ("Better Models, Faster Training: Sigmoid Attention for single-cell
 * Foundation Models", sec. 2A):
 *
 *     O = sigma(Q K^T / sqrt(d) + b) V,   sigma(x) = 1/(1+e^-x),   b = -ln(n_b)
 *
 * and its gradient with respect to Q, K and V (sec. 2B: sigma' = sigma(1-sigma);
 * sec. 2C: one kernel for dQ and one for dK/dV, activations recomputed, no
 * atomics). n_b is the valid length of sequence b; tokens at positions >= n_b
 * are padding and are ignored on both the query and the key side (sec. 2C,
 * native padding support): P_ij = 0 unless i < n_b and j < n_b.
 *
 * Conventions shared by every call
 *  - Tensors Q, K, V, dO, O, dQ, dK, dV are bf16, contiguous [B][H][Lmax][d]
 *    (d fastest), in device memory, 16-byte aligned. d must be 64 or 128.
 *  - lengths is int32 [B] in device memory; each n_b must lie in [0, Lmax].
 *    A value outside that range is treated as 0 (all outputs of sequence b
 *    are zero) and raises SIGATTN_ERR_INVALID_ARG in the workspace's sticky
 *    error word (read it with sigattn_read_error).
 *  - Outputs are fully written: rows i >= n_b of O, dQ, dK and dV are exact
 *    zeros. Values in padded rows of the inputs never change an output, but
 *    must be finite: a padded value v enters a valid result only as 0 * v
 *    inside the tensor-core sums (the discarded results of padded rows
 *    themselves may use it).
 *  - The scale is 1/sqrt(d) and the bias -ln(n_b) is computed in-kernel; the
 *    bias has no gradient. There is no causal mask.
 *  - Arithmetic: bf16 operands, fp32 accumulation, P (and dS) rounded to bf16
 *    before the second matrix product, outputs rounded to nearest bf16. sigma
 *    takes one hardware exp2 per score: with u = e^-|x|, sigma(x) = u r(u)
 *    for x < 0 and r(u) for x >= 0, where r is a polynomial for 1/(1+u) of
 *    relative error <= 8e-4 (about 1e-7 for the tail weights near 1/n that
 *    the bias -ln n makes typical); see sigattn_eval_sigmoid.
 *  - workspace: caller-owned device memory of at least
 *    sigattn_workspace_size(B, H, Lmax, d) bytes, 16-byte aligned. Each call
 *    writes its work list there; calls that may run concurrently (different
 *    streams) need different workspaces. Word 0 is a sticky error status, so
 *    zero the workspace once after allocating it (cudaMemset); the library
 *    keeps it consistent afterwards.
 *  - stream: a cudaStream_t (NULL = legacy default stream). Calls only
 *    enqueue work: they neither allocate nor synchronise, so a sequence of
 *    calls can be captured into a CUDA graph and replayed (make one call on
 *    the device outside the capture first: it sets up per-device kernel
 *    attributes).
 *  - Return value: a sigattn_status. Argument errors are reported before
 *    anything is enqueued. A kernel-side timeout (a bounded wait that gave up)
 *    is recorded in the workspace and surfaces through sigattn_read_error.
 *  - Outputs must not overlap the inputs or each other: the kernels read
 *    input tiles while other tiles of the outputs are being written.
 *  - Ownership: the library keeps no pointer after a call returns.
 */
#ifndef SIGATTN_H_
#define SIGATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SIGATTN_API __attribute__((visibility("default")))
#else
#define SIGATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SIGATTN_OK = 0,
  SIGATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad length */
  SIGATTN_ERR_UNSUPPORTED = 2, /* d not in {64, 128}, or a size beyond the limits */
  SIGATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  SIGATTN_ERR_TIMEOUT = 4      /* a kernel's bounded wait expired (sticky, in the workspace) */
} sigattn_status;

/* Work-list kinds (used by the plan helpers). */
enum { SIGATTN_KIND_FWD = 0, SIGATTN_KIND_DQ = 1, SIGATTN_KIND_DKDV = 2 };

/* Limits: 1 <= B <= SIGATTN_MAX_BATCH, 1 <= H, 1 <= Lmax <= SIGATTN_MAX_LEN. */
#define SIGATTN_MAX_BATCH 4096
#define SIGATTN_MAX_LEN (1 << 20)

/* Library version, e.g. 100 for 0.1.0. */
SIGATTN_API int sigattn_version(void);

/* Human-readable name of a status code (static string). */
SIGATTN_API const char* sigattn_status_str(int status);

/* Rows of one work item for a kind: 256 (forward), 128 (dQ), 128 (dK/dV).
 * Returns -1 for an unknown kind. */
SIGATTN_API int sigattn_block_rows(int kind);

/* Bytes of workspace needed for any of the three calls with these sizes
 * (a 256-byte header plus one 16-byte entry per possible work item).
 * Returns 0 if the sizes are out of range. */
SIGATTN_API size_t sigattn_workspace_size(int B, int H, int Lmax, int d);

/* Forward pass (sec. 2A): o = sigma(q k^T / sqrt(d) - ln n) v.
 * q, k, v: inputs; o: output. All [B][H][Lmax][d] bf16 on the device. */
SIGATTN_API int sigattn_fwd(const void* q, const void* k, const void* v, void* o, const int32_t* lengths, int B, int H,
                int Lmax, int d, void* workspace, size_t workspace_bytes, void* stream);

/* Backward pass, query side (sec. 2B/2C): dq = (1/sqrt(d)) * dS k with
 * dS = (dout v^T) * P * (1 - P). dout is the gradient of the loss w.r.t. o. */
SIGATTN_API int sigattn_bwd_dq(const void* q, const void* k, const void* v, const void* dout, void* dq,
                   const int32_t* lengths, int B, int H, int Lmax, int d, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Backward pass, key/value side (sec. 2B/2C): dk = (1/sqrt(d)) * dS^T q and
 * dv = P^T dout. */
SIGATTN_API int sigattn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                     const int32_t* lengths, int B, int H, int Lmax, int d, void* workspace,
                     size_t workspace_bytes, void* stream);

/* The whole backward pass in one call: dq as sigattn_bwd_dq, dk and dv as
 * sigattn_bwd_dkdv, with identical results (the same kernels, each with one
 * owner per output block and a fixed summation order). The two gradients
 * depend only on q, k, v and dout (sec. 2B/2C: no row statistics of the
 * forward pass are needed), so one plan launch builds both work lists and
 * the dK/dV kernel takes each SM as soon as the dQ kernel's CTA on it has
 * finished, instead of after the last of them: the end of the dQ kernel,
 * where fewer work items than SMs remain, overlaps the start of the dK/dV
 * kernel. The call's last kernel completes only after both have, so later
 * work in the stream sees all three outputs.
 *  - workspace: at least sigattn_bwd_workspace_size(B, H, Lmax, d) bytes
 *    (two work lists); 16-byte aligned and zeroed once, as for every call.
 *    Errors of both kernels go to its sticky error word.
 *  - dq, dk, dv must not overlap each other or the inputs.
 * Returns 0 from sigattn_bwd_workspace_size if the sizes are out of range. */
SIGATTN_API size_t sigattn_bwd_workspace_size(int B, int H, int Lmax, int d);
SIGATTN_API int sigattn_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                            void* dv, const int32_t* lengths, int B, int H, int Lmax, int d, void* workspace,
                            size_t workspace_bytes, void* stream);
/* The same for the packed layout (arguments as sigattn_bwd_dq_varlen; the
 * workspace is sigattn_bwd_workspace_size(B, H, max_seqlen, d) bytes). */
SIGATTN_API int sigattn_bwd_varlen(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
                                   void* dv, const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total,
                                   int d, void* workspace, size_t workspace_bytes, void* stream);

/* Key ranges: the padded-layout calls restricted to the keys at positions
 * [key_begin, key_begin + key_count) of every sequence, for attention whose
 * keys are split over several calls or GPUs (sequence sharding). Because each
 * weight sigma(q.k/sqrt(d) - ln n) stands on its own, with no normalisation
 * over the keys (sec. 2A), O = sigma(S + b) V is the plain sum over key ranges
 * of each range's contribution, and so is dQ = scale dS K (sec. 2B/2C); dK and
 * dV of a key depend on that key and on all queries only. The bias still uses
 * each sequence's full length n_b.
 *  - q, dout: [B][H][Lmax][d] bf16, all query rows. k, v: [B][H][key_count][d]
 *    bf16 holding keys key_begin .. key_begin + key_count - 1 of every
 *    sequence; a key at position key_begin + j is valid if it is < n_b.
 *  - 0 <= key_begin, 1 <= key_count, key_begin + key_count <= Lmax; the
 *    workspace is sigattn_workspace_size(B, H, Lmax, d) as usual.
 *  - sigattn_fwd_partial writes o_partial [B][H][Lmax][d] fp32 (16-byte
 *    aligned): for valid rows i the sum over the range's valid keys j of
 *    P_ij V_j, not rounded; rows i >= n_b, and every row of a sequence with no
 *    valid key in the range, are 0. Summing the partials of ranges that tile
 *    [0, Lmax) gives O in fp32.
 *  - sigattn_bwd_dq_partial writes dq_partial [B][H][Lmax][d] fp32 likewise:
 *    the range's share of dQ, scale included.
 *  - sigattn_bwd_dkdv_range writes dk, dv [B][H][key_count][d] bf16: the rows
 *    of dK and dV for the range's keys (zero for keys >= n_b). With
 *    key_begin a multiple of 128 they are the same bits as the matching rows
 *    of sigattn_bwd_dkdv.
 *  - Everything else as for sigattn_fwd / sigattn_bwd_dq / sigattn_bwd_dkdv. */
SIGATTN_API int sigattn_fwd_partial(const void* q, const void* k, const void* v, float* o_partial,
                                    const int32_t* lengths, int B, int H, int Lmax, int d, int key_begin,
                                    int key_count, void* workspace, size_t workspace_bytes, void* stream);
SIGATTN_API int sigattn_bwd_dq_partial(const void* q, const void* k, const void* v, const void* dout,
                                       float* dq_partial, const int32_t* lengths, int B, int H, int Lmax, int d,
                                       int key_begin, int key_count, void* workspace, size_t workspace_bytes,
                                       void* stream);
SIGATTN_API int sigattn_bwd_dkdv_range(const void* q, const void* k, const void* v, const void* dout, void* dk,
                                       void* dv, const int32_t* lengths, int B, int H, int Lmax, int d, int key_begin,
                                       int key_count, void* workspace, size_t workspace_bytes, void* stream);

/* The softmax counterpart of sigattn_fwd, for comparisons on equal terms
 * (Better Models, Faster Training, sec. 4A compares the sigmoid kernel with
 * softmax attention's FlashAttention-2 on padded batches): the same plan,
 * scheduler, data movement and MMAs, with the sigmoid replaced by a softmax
 * over each sequence's valid keys,
 *     O_i = sum_{j<n} exp(S_ij) V_j / sum_{j<n} exp(S_ij),  S = Q K^T / sqrt(d),
 * computed online (running row maximum, lazily rescaled O and row sums).
 * Forward only, d = 64 only (SIGATTN_ERR_UNSUPPORTED otherwise), padded
 * layout; arguments, outputs (rows >= n_b zero) and workspace as sigattn_fwd.
 * No log-sum-exp is returned. */
SIGATTN_API int sigattn_softmax_fwd(const void* q, const void* k, const void* v, void* o, const int32_t* lengths,
                                    int B, int H, int Lmax, int d, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Round `count` fp32 values to bf16 (nearest even), x -> y, both device
 * pointers, 16-byte aligned; count a multiple of 8. The last step after the
 * fp32 partial sums of key ranges were added (e.g. by an all-reduce). */
SIGATTN_API int sigattn_cast_bf16(const float* x, void* y, long long count, void* stream);

/* Packed ("varlen") layout: the same three operations on sequences stored
 * back to back instead of padded to Lmax, so padding costs neither FLOPs nor
 * HBM bytes. Sequence b's tokens are rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 * of every tensor; n_b = cu_seqlens[b+1] - cu_seqlens[b].
 *  - Tensors are bf16, contiguous [total][H][d] (d fastest, then heads, then
 *    tokens), in device memory, 16-byte aligned; d is 64 or 128.
 *  - cu_seqlens is int32 [B+1] in device memory, nondecreasing, with
 *    0 <= cu_seqlens[b] and cu_seqlens[B] <= total. max_seqlen >= every n_b
 *    plays the part of Lmax (work-list size, limits). A sequence whose bounds
 *    break these rules gets no work: its rows are left untouched and
 *    SIGATTN_ERR_INVALID_ARG is raised in the workspace's sticky error word.
 *  - Only rows that belong to a sequence are written; rows outside every
 *    [cu_seqlens[b], cu_seqlens[b+1]) are never touched. Results equal those of
 *    the padded calls on the same sequences. The last row block of a sequence
 *    reads up to 255 rows past its end (the next sequence, or rows after
 *    cu_seqlens[B]); those enter a result of the sequence only as 0 * value
 *    and must be finite, as padded rows must be in the padded layout.
 *  - 1 <= total <= INT32_MAX - 4096; workspace: sigattn_workspace_size(B, H,
 *    max_seqlen, d) bytes. Everything else as for the padded calls. */
SIGATTN_API int sigattn_fwd_varlen(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                                   int B, int H, int max_seqlen, int total, int d, void* workspace,
                                   size_t workspace_bytes, void* stream);
SIGATTN_API int sigattn_bwd_dq_varlen(const void* q, const void* k, const void* v, const void* dout, void* dq,
                                      const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total, int d,
                                      void* workspace, size_t workspace_bytes, void* stream);
SIGATTN_API int sigattn_bwd_dkdv_varlen(const void* q, const void* k, const void* v, const void* dout, void* dk,
                                        void* dv, const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total,
                                        int d, void* workspace, size_t workspace_bytes, void* stream);

/* Run only the ragged tile scheduler for `kind` on the device: afterwards the
 * workspace holds, at byte offset 8, the item count (int32), and at byte
 * offset 256, `count` entries of four int32 (bh = b*H + h, block index, the
 * valid length n_b, 0), ordered longest sequence first (ties in batch order),
 * heads ascending, blocks ascending. Only blocks whose first row is < n_b appear (sec. 2C: fully
 * padded blocks are skipped). */
SIGATTN_API int sigattn_plan(const int32_t* lengths, int B, int H, int Lmax, int d, int kind, void* workspace,
                 size_t workspace_bytes, void* stream);

/* Host-side statement of the same schedule (no GPU needed): writes up to
 * `cap` (bh, block) pairs to `items_out` (2*cap int32) and the full count to
 * `*count`. lengths_host is host memory. */
SIGATTN_API int sigattn_plan_host(const int32_t* lengths_host, int B, int H, int Lmax, int kind, int32_t* items_out, int cap,
                      int* count);

/* Size of the fixed device scratch array used by sigattn_fwd_noalloc. */
#define SIGATTN_NOALLOC_SCRATCH_BYTES (1 << 20)

/* sigattn_fwd for callers that cannot allocate device memory (code that runs
 * where cudaMalloc is unavailable or forbidden, e.g. inside a host framework
 * that owns the whole device pool, or a plugin that may only touch the
 * buffers it is handed). The paper has no counterpart: it is a deployment
 * convenience of this library.
 *  - Same computation, inputs and outputs as sigattn_fwd; instead of a
 *    caller workspace it uses a SIGATTN_NOALLOC_SCRATCH_BYTES array that is
 *    part of the library's device image, held on every GPU that loads the
 *    library until the process exits. It calls no cudaMalloc/cudaFree.
 *  - Size limit: sigattn_workspace_size(B, H, Lmax, d) must not exceed
 *    SIGATTN_NOALLOC_SCRATCH_BYTES, i.e. B*H*ceil(Lmax/128) <= 65520 work
 *    items; larger problems return SIGATTN_ERR_UNSUPPORTED (message in
 *    sigattn_last_error) before anything is enqueued.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *  - Every call, on every stream, shares the one array: calls that overlap
 *    on the GPU race. Each call clears the array's status words first.
 *  - status_out: optional device int32 (4-byte aligned); if not NULL, it
 *    receives (in stream order) this call's device-side status: 0,
 *    SIGATTN_ERR_INVALID_ARG for an out-of-range length, or
 *    SIGATTN_ERR_TIMEOUT.
 *  - Argument errors (the checks of sigattn_fwd, a misaligned status_out, a
 *    size beyond the array) are returned before anything is enqueued and
 *    leave the array untouched. */
SIGATTN_API int sigattn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, const int32_t* lengths,
                                    int B, int H, int Lmax, int d, int32_t* status_out, void* stream);

/* Text of the last CUDA failure behind a SIGATTN_ERR_CUDA returned to the
 * calling thread (static, thread-local; "no error" if none yet). */
SIGATTN_API const char* sigattn_last_error(void);

/* Diagnostic for the failure path: enqueue a one-warp kernel whose bounded
 * wait on an mbarrier that nothing arrives on must give up after limit_us
 * microseconds (1 .. 10^7). The kernel records SIGATTN_ERR_TIMEOUT with site
 * 901 in the workspace header, exactly as a compute kernel's expired wait
 * does, and returns normally (the context stays usable). Needs only the
 * 256-byte header of a workspace. */
SIGATTN_API int sigattn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int limit_us, void* stream);

/* Diagnostic: the attention weight of raw scores exactly as the compute
 * kernels evaluate it, P = sigma(s / sqrt(d) - ln n) (sec. 2A: the sigmoid of
 * the scaled score plus the bias b = -ln n), and its derivative
 * P (1 - P) (sec. 2B) as the backward kernels use it. scores, p and slope are
 * device float arrays of `count` elements (4-byte aligned); d is 64 or 128,
 * 1 <= n <= SIGATTN_MAX_LEN. The kernels form x = s / sqrt(d) - ln n and
 * take sigma from one hardware exp2 of -|x| log2(e) and a polynomial for
 * 1/(1 + e^-|x|); this entry point lets a test measure that form's error
 * against the exact function on any set of scores. Stream-ordered, no sync. */
SIGATTN_API int sigattn_eval_sigmoid(const float* scores, float* p, float* slope, int count, int d, int n,
                                     void* stream);

/* Synchronise `stream`, read the workspace's sticky error word, clear it and
 * return it (SIGATTN_OK if no kernel reported a problem). If `site` is not
 * NULL it receives a code naming the failing check or wait (0 if none). */
SIGATTN_API int sigattn_read_error(void* workspace, int* site, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SIGATTN_H_ */
