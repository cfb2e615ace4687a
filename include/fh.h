/*
 * fh.h - C ABI of the FlashHead Lite DiT hot path on NVIDIA B200 (sm_100a).
 *
 * The library computes the flow-prediction transformer of SoulX-FlashHead Lite
 * and its 4-step flow sampler, as described by
 *   - gizai:flashhead (gizstack API reference), opening paragraph: a Wan-style
 *     transformer of 30 blocks of width 1536 with 12 heads and rotary over frame,
 *     row and column predicts, in 4 steps, the flow of the noisy video latent
 *     (5 latent frames of 16 x 16 at 512 x 512), conditioned on the reference
 *     latent, the timestep and 5 latent frames of 32 audio tokens; the first
 *     latent frames are the previous slice's motion;
 *   - gizai:flashhead, Types > FlashHead: `patch`/`head` Linear layers, `headMods`
 *     (output norm shift and scale per step, [2, 1536]), `cos`/`sin` rotary
 *     tables [1280, 768], `work: Scratch`;
 *   - gizai:flashhead, Functions > load and Methods > talk: a model is bound to
 *     one GPU at load; a talk request runs slice by slice;
 *   - SoulX-FlashHead (audio-cpp model doc), request options (height/width on the
 *     VAE grid, 4 inference steps, seed) and "an unavailable implementation is
 *     rejected rather than silently substituted".
 * Block-internal details the pages leave open follow fixed readings R1-R16
 * (adaLN order, eps 1e-6, rotary pairing and frequencies, full-width Q/K
 * RMSNorm, per-frame cross-attention, Euler update, motion pinning), stated in
 * the library's design notes and identical in the test oracle.
 *
 * Conventions for every call:
 *   - Return FH_OK (0) or a negative FH_ERR_* code; fh_last_error() returns the
 *     calling thread's last message. No exception crosses the ABI.
 *   - Pointers named *device* are caller-owned CUDA device memory on the model's
 *     GPU, contiguous, 16-byte aligned (checked: FH_ERR_ARG). The library never
 *     frees them. Pointers named *host* are ordinary host memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it; outputs are valid once the stream has reached the
 *     call's end. Kernel-side failures (a bounded wait that ran out) are latched
 *     and reported by fh_dit_sync() or by the next call.
 *   - A handle is not thread-safe; use one stream per handle at a time.
 *   - There is no CPU or library fallback: a device that is not sm_100 is
 *     rejected with FH_ERR_UNSUPPORTED.
 *
 * Layouts (B = batch of independent streams, C = latent channels, F = latent
 * frames, H x W = latent grid, L = F*H*W tokens, token n = f*H*W + h*W + w,
 * D = width, A = audio tokens per latent frame):
 *   latents (noise, ref, x_noisy, v, x_out)  float32 [B, C, F, H, W]
 *   motion                                   float32 [B, C, 2, H, W]
 *   audio tokens                             [B, F, A, D] in the model dtype
 *                                            (bfloat16 for FH_BF16, float32 for FH_F32)
 *   residual stream x (block call)           float32 [B, L, D]
 */
#ifndef FH_H_
#define FH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum fh_status {
  FH_OK = 0,
  FH_ERR_ARG = -1,          /* null/unaligned pointer, bad index, bad value */
  FH_ERR_SHAPE = -2,        /* off-grid size, batch > max_batch, config mismatch */
  FH_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
  FH_ERR_OOM = -4,          /* device allocation failed (create only) */
  FH_ERR_TIMEOUT = -5,      /* a kernel's bounded wait ran out (device error latched) */
  FH_ERR_UNSUPPORTED = -6   /* device is not sm_100, or dtype/shape not supported */
};

enum fh_dtype { FH_F32 = 0, FH_BF16 = 1 };

/* Model configuration. The Lite network is {1536, 12, 128, 8960, 30, 128, 5, 16,
 * 16, 32, max_batch, FH_BF16, 1e4, {44, 42, 42}, 1e-6, device}. Constraints:
 * heads * head_dim == dim, head_dim == 128, dim % 128 == 0, ffn % 128 == 0,
 * latent_ch % 64 == 0, frames >= 2, rope_split sums to head_dim with even parts,
 * 1 <= max_batch <= 8. `device` is the CUDA ordinal the model lives on. */
typedef struct fh_config {
  int dim, heads, head_dim, ffn, blocks, latent_ch, frames, lat_h, lat_w, audio_tokens;
  int max_batch;
  int dtype;            /* FH_F32 (fp32 SIMT path) or FH_BF16 (tcgen05 path) */
  float rope_theta;
  int rope_split[3];    /* rotary dims per head for frame, row, column */
  float eps;
  int device;
} fh_config;

typedef struct fh_dit fh_dit;

/* Weight tensor ids (the seeded generator's stream ids). Block k, slot s has id
 * 64*k + s; global slot g has id 4096 + g. Shapes are nn.Linear style [out, in].
 *   block slots: 0 mod[6,D] (rows: shift/scale/gate of self-attn, shift/scale/gate
 *   of FFN)  1 wq[D,D] 2 bq 3 wk 4 bk 5 wv 6 bv 7 wo 8 bo 9 gq[D] 10 gk[D]
 *   11 ln3_w[D] 12 ln3_b[D] 13 wcq 14 bcq 15 wck 16 bck 17 wcv 18 bcv 19 wco 20 bco
 *   21 gcq[D] 22 gck[D] 23 w1[FF,D] 24 b1[FF] 25 w2[D,FF] 26 b2[D]
 *   global slots: 0 patch_w[D,2C] 1 patch_b[D] 2 head_w[C,D] 3 head_b[C]
 *   4 head_mod[2,D] 5 t_w1[D,256] 6 t_b1[D] 7 t_w2[D,D] 8 t_b2[D] 9 t_wp[6D,D] 10 t_bp[6D]
 * Values: element i (row-major) of tensor id t under seed s is one Box-Muller
 * normal z from SplitMix64 hashes of the counters (s ^ (t << 40)) + 2i and + 2i + 1
 * (53-bit uniforms u1, u2; z = sqrt(-2 ln(1 - u1)) cos(2 pi u2), float64). Linear
 * weights and biases: z / sqrt(fan_in); modulation tables: z / sqrt(D); norm gains:
 * 1 + 0.1 z; LayerNorm bias: 0.1 z. Rounded to float32, then to bfloat16 (ties to
 * even) for FH_BF16 models. */
#define FH_BLOCK_TENSOR(k, s) (64 * (k) + (s))
#define FH_GLOBAL_TENSOR(g) (4096 + (g))
/* Audio projection tensors (fh_audio_project), id 4096 + 32 + a, HID = 512, K0 = 5 * 12 * 768,
 * KV = 12 * 12 * 768: 0 proj1_w[HID,K0] 1 proj1_b[HID] 2 proj1vf_w[HID,KV] 3 proj1vf_b[HID]
 * 4 proj2_w[HID,HID] 5 proj2_b[HID] 6 proj3_w[32D,HID] 7 proj3_b[32D] 8 projnorm_w[D] (a gain)
 * 9 projnorm_b[D] (a LayerNorm bias). */
#define FH_AUDIO_TENSOR(a) (4096 + 32 + (a))

/* Create a model on cfg->device: allocates and owns the weights (generated on the
 * GPU from `seed`), the rotary table [L, 64] and internal buffers. Synchronises
 * `stream` before returning. Errors: FH_ERR_ARG (null), FH_ERR_SHAPE (config
 * constraints), FH_ERR_UNSUPPORTED (not sm_100), FH_ERR_OOM, FH_ERR_CUDA. */
int fh_dit_create(const fh_config* cfg, uint64_t seed, void* stream, fh_dit** out);

/* Free everything the model owns (the counterpart of the pages' model load, gizai:flashhead
 * Functions > load: a model holds its weights on one GPU until it is dropped). NULL is
 * accepted; the handle must not be used afterwards. Returns FH_OK. */
int fh_dit_destroy(fh_dit* m);

/* Bytes of caller-allocated workspace (device, 256-byte aligned) that every
 * compute call with this batch needs. Returns 0 for a bad batch. The workspace
 * plays the role of the pages' `work: Scratch`: the caller owns it; calls on one
 * handle must not overlap in time on the same workspace. */
size_t fh_dit_workspace_bytes(const fh_dit* m, int batch);

/* One transformer block k (gizai:flashhead, opening paragraph: one of the 30 Wan-style
 * blocks, with self-attention over the whole latent and cross-attention to the audio
 * tokens; readings R1-R8 fix the block's internal order) for timesteps t (host float32
 * [batch], in [0, 1]): x_out = block_k(x_in) with x device float32 [B, L, D] (x_in may
 * equal x_out), audio device [B, F, A, D] in the model dtype. The block's adaLN vectors
 * come from the timestep MLP of t; its cross-attention keys/values from `audio`. Errors:
 * FH_ERR_ARG (null or unaligned pointer, workspace null or not 256-byte aligned, block out
 * of range), FH_ERR_SHAPE (batch outside [1, max_batch]), FH_ERR_TIMEOUT (a kernel-side
 * error latched by an earlier call), FH_ERR_CUDA; asynchronous on `stream`. */
int fh_dit_block_forward(fh_dit* m, int block, const float* x_in, float* x_out,
                         const void* audio, const float* t, int batch, void* ws,
                         void* stream);

/* One flow prediction at noise level sigma (timestep t = sigma) (gizai:flashhead, opening
 * paragraph: the transformer predicts the flow of the noisy latent conditioned on the
 * reference latent; Types > FlashHead: `patch` over the concatenation [noisy | reference],
 * the 30 blocks, the output norm modulated by `headMods` + the timestep embedding, `head`):
 * v_out = head(blocks(patch([x_noisy | ref]))), all device float32 [B, C, F, H, W];
 * audio device [B, F, A, D]. No motion pinning (the sampler does that). Errors as
 * fh_dit_block_forward. */
int fh_dit_predict_flow(fh_dit* m, const float* x_noisy, const float* ref,
                        const void* audio, float sigma, float* v_out, int batch,
                        void* ws, void* stream);

/* The slice sampler (gizai:flashhead, opening paragraph and Methods > talk: 4 flow steps per
 * slice, the first latent frames carrying the previous slice's motion): x starts as `noise` (frames 0-1 ignored), frames 0-1 are set
 * to `motion` before each of the `nsteps` flow predictions and on the output, and
 * each step applies x += (sigmas[s+1] - sigmas[s]) * v. sigmas: host float32
 * [nsteps + 1]. noise/ref/x_out device [B, C, F, H, W], motion device
 * [B, C, 2, H, W], audio device [B, F, A, D]. The cross-attention keys/values of
 * all blocks are computed once per call (the audio is fixed over the steps). The
 * first call for a (workspace, batch, sigmas) combination records a CUDA graph of
 * the step loop; later calls replay it. */
int fh_sample_slice(fh_dit* m, const float* noise, const float* ref, const float* motion,
                    const void* audio, const float* sigmas, int nsteps, float* x_out,
                    int batch, void* ws, void* stream);

/* The slice sampler with the re-noising update that the SoulX-FlashHead audio-cpp doc
 * (Generate / Variant boundaries) names for distilled checkpoints without defining it,
 * read as: x0 = x - sigmas[s] v, then x = (1 - sigmas[s+1]) x0 + sigmas[s+1] eps[s].
 * Everything else (motion pinning, inputs, outputs, graph recording) is as in
 * fh_sample_slice; at sigmas[s+1] = 0 the step equals the Euler step exactly.
 * eps: device float32 [nsteps, B, C, F, H, W], the fresh N(0, 1) draw of each step,
 * caller-owned and read during the call (frames 0-1 are overwritten by the motion pin,
 * so their values do not matter). The recorded graph is keyed on the eps pointer too:
 * refill the same buffer between slices to replay it. Errors as fh_sample_slice;
 * FH_ERR_ARG also for a null or unaligned eps. */
int fh_sample_slice_renoise(fh_dit* m, const float* noise, const float* ref, const float* motion,
                            const void* audio, const float* sigmas, int nsteps, const float* eps,
                            float* x_out, int batch, void* ws, void* stream);

/* fh_sample_slice with HOST buffers: the inputs are copied host -> device into the
 * workspace, the slice runs, and the clean latent is copied back to x_out_host;
 * returns once x_out_host is written (the stream is synchronised). Pinned host
 * memory gives asynchronous copies; pageable memory works but is slower. */
int fh_sample_slice_host(fh_dit* m, const float* noise_host, const float* ref_host,
                         const float* motion_host, const void* audio_host,
                         const float* sigmas, int nsteps, float* x_out_host, int batch,
                         void* ws, void* stream);

/* The audio projection of one slice (gizai:flashhead, opening paragraph: the last 8 s of
 * speech through wav2vec 2.0 base, its 12 layers' states at 200 frames; 5 states around each
 * of the slice's 33 frames make 5 latent frames of 32 audio tokens; Types > FlashHead: proj1,
 * proj1vf, proj2, proj3, projNorm). states: device float32 [B, 200, 12, 768], the encoder's
 * states over the audio window (the last of them at the slice's last video frame). tokens:
 * device [B, frames, 32, dim] in the model dtype, the `audio` argument of the calls above.
 * Video frame t of the slice's 1 + 8 (frames - 1) takes the states within two of state
 * 200 - (1 + 8 (frames - 1)) + t (clamped to the window); latent frame 0 reads video frame
 * 0's 5 states through proj1, latent frame j >= 1 the 12 states spanning video frames
 * 8j-7..8j through proj1vf; both with a ReLU, then proj2 with a ReLU, proj3 to 32 tokens and
 * projNorm, a LayerNorm with weight and bias over each token. Asynchronous on `stream`; uses
 * the workspace. Errors: as fh_dit_block_forward; FH_ERR_SHAPE if the latent frames need more
 * than 200 states. */
int fh_audio_project(fh_dit* m, const float* states, void* tokens, int batch, void* ws, void* stream);

/* Copy weight tensor `tensor_id` to host memory as float32 in its logical
 * row-major shape; `bytes` must equal 4 * element count (else FH_ERR_ARG; an unknown id
 * is FH_ERR_ARG too). Synchronous. The pages have no such call: it exists so that a test
 * can give the oracle the very weights the GPU uses (Types > FlashHead names the tensors). */
int fh_dit_get_weight(const fh_dit* m, int tensor_id, void* host_dst, size_t bytes);

/* Wait for `stream`, then report a latched kernel-side error (FH_ERR_TIMEOUT) and
 * clear it. */
int fh_dit_sync(fh_dit* m, void* stream);

/* Kernel launches issued by the last compute call on this handle (a graph replay
 * counts the kernels inside the graph). */
int fh_dit_last_launch_count(const fh_dit* m);

/* Optional per-launch timing of one kernel class inside fh_sample_slice, for
 * roofline reporting: 0 off, 1 the gated-residual GEMMs (O-proj, cross-O, FFN2),
 * 2 the FFN1 GEMM, 3 the QKV GEMM, 4 self-attention, 5 cross-attention, 6 the
 * first row norm of each block, 7 the cross-Q GEMM. Changing it re-records
 * graphs. fh_dit_get_timing returns the mean device time (microseconds) and count
 * of that class's launches in the last completed fh_sample_slice call. */
int fh_dit_set_timing(fh_dit* m, int kernel_class);
int fh_dit_get_timing(fh_dit* m, double* mean_us, int* launches);

/* fh_dit_block_forward without a workspace argument, for callers that cannot allocate
 * device memory where they run a block (plugins inside a host framework that owns all
 * device memory, real-time threads that must not take the allocator's locks). The pages
 * have no counterpart: this is a
 * deployment variant, not a step of the method. The scratch is a file-scope __device__
 * array of FH_STATIC_SCRATCH_BYTES (16 MiB) inside the library, held on every GPU that
 * loads the library until the process exits; calls whose fh_dit_workspace_bytes exceeds
 * it fail with FH_ERR_SHAPE (the full 1536-wide network needs more: use
 * fh_dit_block_forward there). The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, which may load the library's module): make that first
 * call before any stream capture. Every call on a device shares the one array and it
 * keeps the last call's contents; calls that overlap in time on the GPU (different
 * streams, or different handles) race on it. Nothing in it needs to start at zero.
 * Arguments and errors otherwise as fh_dit_block_forward. Allocates nothing. */
#define FH_STATIC_SCRATCH_BYTES (16u << 20)
int fh_dit_block_forward_noalloc(fh_dit* m, int block, const float* x_in, float* x_out, const void* audio,
                                 const float* t, int batch, void* stream);

/* Thread-local text of the last error ("" if none). */
const char* fh_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* FH_H_ */
