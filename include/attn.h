/*
 * attn.h: C ABI of the exact scaled-dot-product attention library for one
 * NVIDIA B200 (sm_100a).
 *
 * Operation: hysenlabs.com, "FlashAttention: exakte Attention-Kernel fuer CUDA
 * und ROCm", section "Die Schnittstellen von flash_attn_func bis KV-Cache".
 * Every entry point computes
 *
 *     O = softmax(Q @ K^T * softmax_scale) @ V
 *
 * `causal` masks key j for query i when j > i. In attn_fwd/attn_bwd queries
 * and keys have the same length N. attn_fwd_masked/attn_bwd_masked take
 * Nq != Nk and a sliding window. There the causal mask is aligned to the
 * bottom-right corner (same page, section "Von 2.0 bis 2.7", release 2.1),
 * and the window of release 2.3 (`window_size` in the interface section)
 * applies. K and V may have fewer heads than Q when Hq is divisible by Hkv
 * (MQA/GQA, same interface section). Query head h reads KV head
 * h / (Hq / Hkv).
 *
 * The method is exact, not an approximation (tokenwerk.de "FlashAttention",
 * section "Was FlashAttention veraendert"). Results differ from a float64
 * evaluation of the formula only by floating-point rounding. The N x N score
 * matrix is never written to memory: tiles of Q, K and V are staged on chip,
 * and a running row max and row sum normalise the output as it accumulates
 * (unite.ai "Was ist FlashAttention?", five-stage map, stages 1-4).
 *
 * Conventions shared by all calls
 *  - Tensors are contiguous, row-major [B, H, N, d] bfloat16 (d fastest).
 *    lse and the workspace are float32.
 *  - Every tensor pointer is a DEVICE pointer owned by the caller. It must
 *    be 16-byte aligned and must not alias another argument. The library
 *    allocates no memory and keeps no pointer after a call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t, may be 0), like a
 *    kernel launch. They return after the launches are queued. The kernels
 *    are launched with programmatic stream serialization: one may start its
 *    set-up while the work before it on the stream finishes, but it touches
 *    no global memory until that work has completed, so the stream order a
 *    caller sees is that of ordinary launches.
 *  - Supported: d in {64, 128}; N >= 1 (any length; ragged tail tiles are
 *    masked); B, Hq, Hkv >= 1; Hq % Hkv == 0; scale finite and > 0.
 *    B == 0 or N == 0 is an empty problem: nothing is launched and ATTN_OK
 *    is returned.
 *  - Errors are return codes, never aborts. An argument error launches
 *    nothing. The message of the last error on the calling thread is in
 *    attn_get_last_error().
 *  - There is no CPU fallback. Without a usable sm_100 device the calls
 *    return ATTN_ERR_CUDA.
 *  - Kernel waits are bounded. A kernel that stalls for two seconds on a
 *    pipeline barrier records a timeout in a device status word and exits.
 *    attn_check_status() reports it (ATTN_ERR_TIMEOUT), as it reports
 *    invalid packed-batch offsets found on the GPU (ATTN_ERR_ARG).
 */
#ifndef EXACT_ATTENTION_B200_ATTN_H_
#define EXACT_ATTENTION_B200_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_ARG = 1,          /* invalid argument (null/misaligned pointer, bad shape)   */
  ATTN_ERR_UNSUPPORTED = 2,  /* valid but not built (head dim other than 64 or 128)     */
  ATTN_ERR_CUDA = 3,         /* CUDA runtime/driver error, or no sm_100 device          */
  ATTN_ERR_TIMEOUT = 4       /* a kernel gave up on a pipeline wait (see check_status)   */
} attn_status;

/* Opaque stream handle; pass a cudaStream_t (or 0 for the legacy default stream). */
typedef void* attn_stream_t;

/*
 * attn_fwd: forward pass.
 *   q    [B, Hq,  N, d] bf16, read
 *   k, v [B, Hkv, N, d] bf16, read
 *   o    [B, Hq,  N, d] bf16, written: softmax(q k^T * scale [causal]) v
 *   lse  [B, Hq,  N]    f32,  written: natural-log logsumexp of the scaled,
 *        masked logits of each query row, ln sum_j exp(scale * q_i . k_j).
 *        (The pages do not define lse. This is the plainest definition
 *        that the backward pass needs.)
 *   scale: softmax_scale (for example 1/sqrt(d)); causal: 0 or 1.
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                     attn_stream_t stream);

/*
 * attn_bwd: recompute-based backward pass of attn_fwd.
 *   q, k, v, o, lse: as passed to / returned by attn_fwd (read)
 *   dO  [B, Hq,  N, d] bf16, read: gradient of the loss with respect to o
 *   dq  [B, Hq,  N, d] bf16, written
 *   dk, dv [B, Hkv, N, d] bf16, written. Under GQA each KV head's gradient
 *        is the sum over the Hq/Hkv query heads that read it.
 *   workspace: caller-owned device scratch of at least
 *        attn_bwd_workspace_size(B, Hq, N, d) bytes, 16-byte aligned. Its
 *        contents on entry are ignored, and it is overwritten. It must not be
 *        shared by backward calls that can overlap on the GPU.
 * The pages do not write out the backward math. It is the exact gradient of
 * the forward definition: dV = P^T dO, dS = P * (dP - rowsum(dO * O)) with
 * dP = dO V^T, dQ = scale * dS K, dK = scale * dS^T Q. The P used is
 * recomputed from q, k and lse, so no N x N matrix is stored. The result is
 * deterministic, the same bits on every run: each gradient tile is computed
 * by one CTA alone (the only atomics hand out work items, which does not
 * change what any item computes).
 */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dO, void* dq, void* dk, void* dv,
                     void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N,
                     int d, float scale, int causal, attn_stream_t stream);

/*
 * Bytes of workspace attn_bwd needs for this shape (0 for an empty problem).
 * The pages have no counterpart: it exists because this library never
 * allocates, so the caller sizes and owns the backward's scratch (two fp32
 * rows per query, padded to a multiple of 128 per head, and 64 bytes of work
 * counters). d is accepted for symmetry with the other calls and does not
 * change the size.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int N, int d);

/*
 * attn_bwd_noalloc: attn_bwd for callers that cannot allocate device memory.
 * Some callers cannot call cudaMalloc, or any allocator, at the point where
 * they run the backward pass. Examples: plugins whose execute step must not
 * allocate, code running inside an allocator or memory-pool callback, and
 * processes that place all device memory at start-up under a fixed budget.
 * Such callers cannot supply attn_bwd's workspace. This entry point takes the
 * same tensors as attn_bwd (inputs and outputs are still caller-owned) and
 * keeps its scratch in a fixed array of 8 MiB + 64 bytes that the library places in device
 * memory. Every GPU that loads the library holds that array until the process
 * exits. The pages describe no such entry point. It has no counterpart there.
 *   - Limit: attn_bwd_workspace_size(B, Hq, N, d) must not exceed 8 MiB + 64
 *     bytes (8388672 bytes), i.e. B * Hq * (N rounded up to a multiple of 128)
 *     <= 1048576. Larger shapes return ATTN_ERR_ARG with a message, and
 *     nothing is launched.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine. The first
 *     call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and caches it. Make
 *     that first call on a device before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Each call rewrites every scratch entry it reads before reading it, so
 *     nothing has to be cleared. Calls whose kernels overlap on the GPU (for
 *     example on two streams without ordering between them) race on the
 *     array and may return wrong gradients. Order such calls on one stream or
 *     with events.
 * Results are the same as attn_bwd's for the same inputs.
 */
attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dO, void* dq, void* dk, void* dv,
                             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                             attn_stream_t stream);

/*
 * attn_fwd_masked: attn_fwd with Nq queries, Nk keys and a sliding window.
 *   q, o [B, Hq, Nq, d] bf16; k, v [B, Hkv, Nk, d] bf16; lse [B, Hq, Nq] f32.
 *   With off = Nk - Nq, query row i sees key j (0 <= j < Nk) iff
 *       i + off - window_left <= j <= i + off + window_right,
 *   and, with causal = 1, also j <= i + off (so causal caps window_right at
 *   0). A negative window side is unbounded. window_left = window_right = -1
 *   and Nq == Nk is exactly attn_fwd.
 *   A query row that sees no key (Nq > Nk with causal, or a window that
 *   falls outside the keys) gets o = 0 and lse = -inf. Nk == 0 with Nq > 0
 *   is such a case for every row. Nq == 0 or B == 0 writes nothing.
 *   softcap: 0 turns it off. With softcap = c > 0 each scaled logit
 *   z = scale * q_i . k_j becomes c * tanh(z / c) before the mask and the
 *   softmax (release 2.6 on the same page, "softcapping as used in Gemma-2
 *   and Grok"; the pages give no formula, this is the form those models
 *   use), and lse is over the capped logits. Must be finite and >= 0.
 * Errors as in attn_fwd.
 */
attn_status attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                            int causal, int window_left, int window_right, float softcap,
                            attn_stream_t stream);

/*
 * attn_bwd_masked: backward of attn_fwd_masked, with the same Nq, Nk,
 * causal and window arguments.
 *   dO, dq [B, Hq, Nq, d]; dk, dv [B, Hkv, Nk, d]; lse as attn_fwd_masked
 *   wrote it. The workspace needs attn_bwd_workspace_size(B, Hq, Nq, d)
 *   bytes. A query row that sees no key gets dq = 0. A key that no query
 *   sees gets dk = dv = 0. With Nk == 0 only dq (zeros) is written; with
 *   Nq == 0 only dk and dv (zeros).
 * Errors as in attn_bwd.
 */
attn_status attn_bwd_masked(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                            int Nq, int Nk, int d, float scale, int causal, int window_left,
                            int window_right, float softcap, attn_stream_t stream);

/*
 * attn_fwd_varlen / attn_bwd_varlen: a packed ("varlen", release 2.0 on the
 * same page) batch of B sequences of different lengths, stored token by
 * token with no padding:
 *   q, o, dO, dq [total_q, Hq, d] bf16; k, v, dk, dv [total_k, Hkv, d] bf16;
 *   lse [Hq, total_q] f32.
 *   cu_seqlens_q, cu_seqlens_k: DEVICE int32 arrays of B + 1 offsets,
 *   non-decreasing, starting at 0 and ending at total_q / total_k. Sequence b
 *   is rows cu_seqlens_q[b] .. cu_seqlens_q[b+1] of q and cu_seqlens_k[b] ..
 *   cu_seqlens_k[b+1] of k and v, and attends only within itself, with its
 *   own Nq_b and Nk_b: causal, window and softcap as in attn_fwd_masked, per
 *   sequence (bottom-right alignment with off_b = Nk_b - Nq_b).
 *   max_seqlen_q/k: the longest sequence (sizes the grid). Every Nq_b must be
 *   <= max_seqlen_q and every Nk_b <= max_seqlen_k.
 *   Backward workspace: attn_bwd_workspace_size(B, Hq, max_seqlen_q, d) bytes.
 * The offsets are read on the GPU, so the host cannot check them. Offsets
 * that break the rules above are clipped into range (no access leaves the
 * tensors) and the next attn_check_status() returns ATTN_ERR_ARG; results
 * of the affected sequences are then undefined. Rows that belong to no
 * sequence (past cu_seqlens_q[B]) are not written. Sequences with Nk_b = 0
 * get o = 0, lse = -inf and dq = 0; keys no query sees get dk = dv = 0.
 * Errors otherwise as in attn_fwd / attn_bwd.
 */
attn_status attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int Hq,
                            int Hkv, int total_q, int total_k, int max_seqlen_q,
                            int max_seqlen_k, int d, float scale, int causal, int window_left,
                            int window_right, float softcap, attn_stream_t stream);

attn_status attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, void* workspace,
                            size_t workspace_bytes, int B, int Hq, int Hkv, int total_q,
                            int total_k, int max_seqlen_q, int max_seqlen_k, int d, float scale,
                            int causal, int window_left, int window_right, float softcap,
                            attn_stream_t stream);

/*
 * attn_check_status: own design; the pages have no counterpart. The kernels
 * never trap: a pipeline wait that gives up, or packed offsets that had to be
 * clipped, is recorded in a device status word instead, and this call turns
 * that word into a status code and a message.
 * Synchronises `stream`, then reads and clears the device status word.
 * Returns ATTN_ERR_TIMEOUT if a kernel gave up on a wait since the last
 * check, ATTN_ERR_ARG if a varlen call met invalid cu_seqlens offsets,
 * ATTN_ERR_CUDA on a CUDA error, and ATTN_OK otherwise.
 */
attn_status attn_check_status(attn_stream_t stream);

/*
 * Failure-detection self-test (not an attention operation, so the pages have
 * no counterpart). It launches one kernel on `stream` that waits on a pipeline
 * barrier nothing ever signals, with the same bounded wait the attention
 * kernels use. That wait gives up after two seconds and records a timeout.
 * The next attn_check_status(stream) returns ATTN_ERR_TIMEOUT and clears the
 * word. The GPU context stays usable. Returns ATTN_OK when the launch was
 * queued, or ATTN_ERR_CUDA.
 */
attn_status attn_selftest_wait_timeout(attn_stream_t stream);

/*
 * Message of the last error on the calling thread ("" if none). The library
 * owns the string. It stays valid until the next call on the same thread.
 * tokenwerk.de "FlashAttention", section "Fehler und Leistungsversprechen
 * richtig einordnen": when a kernel is missing, the version, the GPU and the
 * input shape are checked first and the exact message is recorded. Every
 * non-OK status therefore comes with a message that names the argument, the
 * shape or the CUDA call that failed (for example "head dim 96 not supported
 * (built: 64, 128)" or "this library is built for sm_100a (B200); device 0 is
 * sm_90").
 */
const char* attn_get_last_error(void);

/*
 * Opt-in per-kernel timing (tracing). While enabled, each kernel launch is
 * bracketed by two CUDA events recorded on its stream. The events come from
 * a pool that the library creates on first use. attn_profile_read() waits for
 * the recorded events and returns, for kernel index `kernel` (0 fwd_kernel,
 * 1 bwd_pre_kernel, 2 bwd_dkdv_kernel, 3 bwd_dq_kernel), its name, the number
 * of launches timed and their summed duration in milliseconds since the last
 * reset. An out-of-range index returns ATTN_ERR_ARG. Off by default. When it
 * is off, calls record nothing.
 */
void attn_profile_enable(int on);
void attn_profile_reset(void);
attn_status attn_profile_read(int kernel, const char** name, int* launches, double* total_ms);

/* ABI version of this header: major * 100 + minor (1.02: masked, softcap and varlen calls). */
int attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_B200_ATTN_H_ */
