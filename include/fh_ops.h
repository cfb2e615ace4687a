/*
 * fh_ops.h - operator-level entry points of the FlashHead DiT library, for unit
 * parity tests of single kernels. Same conventions as fh.h (return codes,
 * fh_last_error, caller-owned 16-byte-aligned device pointers, asynchronous on
 * `stream`). They allocate nothing.
 */
#ifndef FH_OPS_H_
#define FH_OPS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* out[M, N] (float32) = A[M, K] * W[N, K]^T + bias[N]: the dense contraction every
 * Linear of the DiT uses (gizai:flashhead, Types > FlashHead: `patch`, `head` and the
 * blocks' projections are Linear layers). dtype FH_BF16: A, W bfloat16, tensor-core
 * (tcgen05) path, requires N % 128 == 0, K % 64 == 0; FH_F32: A, W float32, CUDA-core
 * path, requires N % 128 == 0, K % 32 == 0. Errors: FH_ERR_ARG, FH_ERR_SHAPE,
 * FH_ERR_CUDA. */
int fh_op_linear(const void* A, const void* W, const float* bias, float* out, int M, int N, int K, int dtype,
                 void* stream);

/* Non-causal self-attention over L tokens per (stream, head), as inside a block
 * (gizai:flashhead, opening paragraph; readings R4-R6): q, k, v [batch, heads, L,
 * 128] in dtype, except that with FH_BF16 v is float16 (as the QKV projection stores it:
 * the kernel multiplies v by float16 softmax weights); ssq float32 [batch*L, 2*heads] with the per-head partial sums of
 * squares of q (first heads columns) and k (last heads columns), whose sum over
 * heads divided by heads*128, plus eps, gives each token's RMS factor r^-2; scores
 * are r_i r_j (q_i . k_j) / sqrt(128). out [batch*L, heads*128] in dtype. */
int fh_op_attention(const void* q, const void* k, const void* v, const float* ssq, void* out, int batch,
                    int heads, int L, float eps, int dtype, void* stream);

/* Per-frame audio cross-attention, as inside a block (gizai:flashhead, opening paragraph:
 * each slice's audio becomes 5 latent frames of 32 audio tokens; readings R4-R6): token n
 * of latent frame f = n / hw of stream b attends to the audio_tokens (= 32, else
 * FH_ERR_SHAPE) keys of that frame only,
 *   out_n = sum_a softmax_a(r_n r_a (q_n . k_a) / sqrt(128)) v_a   per head.
 * q [batch*frames*hw, heads*128] (token-major, frame-major within a stream) in dtype;
 * ssq_q float32 [batch*frames*hw, heads] per-head partial sums of squares of the query
 * row, whose sum over heads divided by heads*128, plus eps, gives r_n^-2; kv
 * [batch*frames*32, 2*heads*128] in dtype: row (b*frames + f)*32 + a holds key a of that
 * frame in its first heads*128 columns and its value in the rest; ssq_k float32
 * [batch*frames*32, heads] the keys' partial sums. out like q. dtype FH_BF16: the
 * tensor-core kernel (TMA over 3D [frame][hw][D] views: hw need not be a multiple of
 * 128, rows past a frame are neither read nor written); FH_F32: CUDA cores. */
int fh_op_cross_attention(const void* q, const float* ssq_q, const void* kv, const float* ssq_k, void* out,
                          int batch, int heads, int frames, int hw, int audio_tokens, float eps, int dtype,
                          void* stream);

/* One norm and modulation per row, as before the block's projections (gizai:flashhead,
 * opening paragraph, "Wan-style"; readings R1, R2, R7, R9): x float32 [M, D] (D / 128 in
 * {1, 2, 3, 4, 6, 8, 12, 16}, else FH_ERR_SHAPE), out [M, D] in dtype.
 *   mode 0: LayerNorm(x) * (1 + a) + c    mode 2: RMSNorm(x) * (1 + a) + c
 *     (a = scale, c = shift: float32 vectors of D, the stream's own at a + (row /
 *      rows_per_batch) * bstride)
 *   mode 1: LayerNorm(x) * a + c            (a = weight, c = bias; bstride ignored)
 * LayerNorm with the biased variance, no gain of its own; eps inside the root. */
int fh_op_row_norm(const float* x, void* out, int M, int D, int mode, const float* a, const float* c, long bstride,
                   int rows_per_batch, float eps, int dtype, void* stream);

/* Failure-detection check (no counterpart on the pages; reading of the pages'
 * reject-don't-hang stance): launches one CTA whose mbarrier wait has no arriving
 * party. The kernel's bounded wait (the same one every production kernel uses, about
 * one second of %globaltimer) runs out, latches the timeout bit into the model's
 * device-visible error word and the kernel returns; nothing faults or hangs. The next
 * fh_dit_sync on `stream` reports FH_ERR_TIMEOUT once and clears the word. */
struct fh_dit;
int fh_dit_probe_wait_timeout(struct fh_dit* m, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FH_OPS_H_ */
