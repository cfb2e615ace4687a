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
 * 128] in dtype; ssq float32 [batch*L, 2*heads] with the per-head partial sums of
 * squares of q (first heads columns) and k (last heads columns), whose sum over
 * heads divided by heads*128, plus eps, gives each token's RMS factor r^-2; scores
 * are r_i r_j (q_i . k_j) / sqrt(128). out [batch*L, heads*128] in dtype. */
int fh_op_attention(const void* q, const void* k, const void* v, const float* ssq, void* out, int batch,
                    int heads, int L, float eps, int dtype, void* stream);

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
