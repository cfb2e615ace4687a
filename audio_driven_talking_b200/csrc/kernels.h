// kernels.h - host-side launchers of the library's kernels (internal interface).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace fh {

typedef __nv_bfloat16 bf16;
struct EpiParams;

// Launch with programmatic stream serialization (PDL): a kernel may begin its prologue
// while its predecessor in the stream drains. Every kernel of this library calls
// pdl_wait() before it touches global memory that an earlier kernel writes. The GEMM
// signals its dependents only after its producer has issued the last tile loads (a
// trigger at kernel entry measured slower on B200: the early dependents took SM slots).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// bf16 tensor-core GEMM (gemm_tc.cu): out = epilogue(A[M,K] * W[N,K]^T); `a`, `b`
// are TMA maps of A (box 64 x 128) and W (box 64 x bn, or 64 x bn/2 when `pair`) with
// the 128-byte swizzle. N % bn == 0, K % 64 == 0. `pair`: 256 x bn tiles computed by
// two CTAs of a cluster with cta_group::2, persistent over every CTA pair; their epilogues
// store through `c`, a TMA map of the output (EPI_RESID: of the fp32 residual; EPI_QKV: 3D
// [3*B*heads][L][128]) with box 32 x 32 (x 1) and the 128-byte (fp32) or 64-byte (bf16)
// swizzle.
cudaError_t gemm_tc_prepare();  // sets the kernels' shared-memory attributes on the current device
cudaError_t gemm_tc(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap* c, int M, int N, int K, int bn,
                    int kind, bool out_bf16, const EpiParams& ep, unsigned* err, int num_sms, cudaStream_t st,
                    bool pair = false);

// fp32 CUDA-core GEMM (misc.cu) with the same epilogues; N % 128 == 0.
cudaError_t gemm_simt(const float* A, long lda, const float* W, long ldw, int M, int N, int K, int kind,
                      const EpiParams& ep, cudaStream_t st);

// self-attention (attention.cu). q/k/v: [B, heads, L, 128]; out [B*L, heads*128];
// ssq [B*L, ssq_ld] holds per-head partial sums of squares, q heads then k heads.
cudaError_t attn_tc_prepare();
cudaError_t attn_tc(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const float* ssq,
                    int ssq_ld, int batch, int heads, int L, float eps, bf16* out, unsigned* err,
                    cudaStream_t st);
template <typename T>
cudaError_t attn_simt(const T* q, const T* k, const T* v, const float* ssq, int ssq_ld, int batch, int heads,
                      int L, float eps, T* out, cudaStream_t st);

// per-frame audio cross-attention (misc.cu).
// q [B*L, D] row-major with ssq_q [B*L, heads]; keys/values: rows (b*F + f)*A + a of
// kv (row stride ldkv), key columns at koff, value columns at voff, with key partial
// sums of squares ssq_k[row * ssq_k_ld + ssq_k_off + h]. out [B*L, D].
// bf16 per-frame cross-attention on the tensor cores (xattn.cu): `q` a 3D TMA map of the
// cross queries [B*F frames][HW][D] (box 64 x 128 x 1), `kv` a 2D map of the cross
// keys/values [B*F*A rows][ldkv] (box 64 x 32), `o` a 3D map of the output like `q` with
// box 64 x 32 x 1; all bf16 with the 128-byte swizzle. A == 32, L % F == 0.
cudaError_t xattn_tc_prepare();
cudaError_t xattn_tc(const CUtensorMap& q, const CUtensorMap& kv, const CUtensorMap& o, const float* ssq_q,
                     const float* ssq_k, int ssq_k_ld, int ssq_k_off, int koff, int voff, int batch, int heads, int L,
                     int F, int A, float eps, unsigned* err, cudaStream_t st);
cudaError_t cross_attn_prepare();  // shared-memory attribute, outside any stream capture
template <typename T>
cudaError_t cross_attn(const T* q, const float* ssq_q, const T* kv, long ldkv, int koff, int voff,
                       const float* ssq_k, int ssq_k_ld, int ssq_k_off, int batch, int heads, int L, int F, int A,
                       float eps, T* out, cudaStream_t st);

// row norms (misc.cu): out[row] = norm(x[row]) then
//   mode 0: LayerNorm, * (1 + scale[b]) + shift[b]   (scale/shift rows of stride mod_bstride)
//   mode 1: LayerNorm, * w + bb                       (learned affine)
//   mode 2: RMSNorm,   * (1 + scale[b]) + shift[b]
template <typename T>
cudaError_t norm_rows(const float* x, T* out, int M, int D, int rows_per_batch, int mode, const float* shift,
                      const float* scale, long mod_bstride, const float* w, const float* bb, float eps,
                      cudaStream_t st);

// timestep conditioning (misc.cu)
struct TVals {
  float t[8];
};
cudaError_t time_sinusoid(float* out, int batch, TVals tv, int dim, cudaStream_t st);
template <typename WT>
cudaError_t gemv(const WT* W, const float* x, const float* bias, float* y, int N, int K, int batch, int silu_in,
                 int silu_out, cudaStream_t st);
// mods[b][k][i][c] = table[k][i][c] + e0[b][i][c]; hmods[b][i][c] = htable[i][c] + e[b][c]
cudaError_t assemble_mods(const float* table, const float* e0, const float* htable, const float* e, float* mods,
                          float* hmods, int batch, int blocks, int D, cudaStream_t st);

// latents (misc.cu). Channel-first [B, C, F*H*W] <-> token-major rows.
template <typename T>
cudaError_t prep_tokens(const float* x, const float* ref, const float* motion, int pin_frames, float* lat, T* tok,
                        int batch, int C, int L, int HW, cudaStream_t st);
template <typename T>
cudaError_t euler_step(float* lat, const float* v, float dsig, int pinned_tokens, T* tok, int batch, int C, int L,
                       cudaStream_t st);
// the re-noising step: x0 = x - sig v, x = (1 - sig_next) x0 + sig_next eps (eps
// channel-first [B, C, L], this step's draw), motion tokens untouched, tok refreshed.
template <typename T>
cudaError_t renoise_step(float* lat, const float* v, const float* eps, float sig, float sig_next, int pinned_tokens,
                         T* tok, int batch, int C, int L, cudaStream_t st);
cudaError_t tokens_to_latent(const float* tok, float* out, int batch, int C, int L, cudaStream_t st);

// seeded weights (misc.cu): element (r, c) of tensor `tid` -> dst[r * ld + c]
// kind 0: z * 1/sqrt(fan) (computed as z / sqrt(fan)); 1: 1 + 0.1 z; 2: 0.1 z
template <typename T>
cudaError_t gen_tensor(T* dst, long rows, long cols, long ld, uint64_t seed, int tid, int kind, int fan,
                       bool round_bf16, cudaStream_t st);
cudaError_t rope_table(float2* tab, int F, int H, int W, int pf, int ph, int pw, float theta, cudaStream_t st);
cudaError_t fill_f32(float* p, long n, float v, cudaStream_t st);
cudaError_t wait_probe(unsigned* err, cudaStream_t st);

// audio projection (audio.cu): gather the encoder states each latent frame reads, and a
// skinny split-K product y = act(x W^T + b) with an output row map (see audio.cu)
cudaError_t audio_windows(const float* states, float* win0, float* winv, int batch, int S, int per_state, int F,
                          int s0, int window, int stride, int group, cudaStream_t st);
int audio_gemv_chunks(int K);
template <typename WT>
cudaError_t audio_linear(const WT* W, const float* x, const float* bias, float* part, float* y, int N, int K, int R,
                         int relu, int per, int ostride, int ooff, cudaStream_t st);

}  // namespace fh
