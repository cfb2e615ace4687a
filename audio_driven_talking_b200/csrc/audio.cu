// audio.cu - the audio projection: speech-encoder states -> the latent frames' audio tokens.
//
// gizai:flashhead (gizstack API reference), opening paragraph: for each slice the last 8 s
// of speech go through wav2vec 2.0 base, whose 12 layers' states are taken at 200 frames,
// and 5 states around each of the slice's 33 frames make 5 latent frames of 32 audio tokens;
// Types > FlashHead names the layers proj1, proj1vf, proj2, proj3 (Linear) and projNorm.
// Readings (the pages give no widths): video frame t of the slice sits at state
// 200 - 33 + t and takes the states within two of it (indices clamped to [0, 199]); latent
// frame 0 is video frame 0 alone (5 states), latent frame j >= 1 is video frames 8j-7..8j,
// whose windows span 12 consecutive states; proj1 (frame 0) / proj1vf (later frames) map
// the flattened states to 512 with a ReLU, proj2 512 -> 512 with a ReLU, proj3 to 32 tokens
// of width D, and projNorm is a LayerNorm with learned affine over each token.
//
// The weights stream from HBM once per slice (about 210 MB in bf16 at D = 1536) against at
// most a few rows of activations, so every projection is a skinny, bandwidth-bound product:
// audio_gemv_kernel splits K into chunks over a grid of CTAs (one warp per output column,
// 16-byte weight loads, the rows' activation chunk staged in shared memory) and writes one
// partial sum per chunk; audio_reduce_kernel adds the chunks in a fixed order (a
// deterministic result), the bias and the activation.
#include "common.cuh"
#include "kernels.h"

namespace fh {

namespace {

constexpr int AG_KC = 1024;   // K per chunk
constexpr int AG_RG = 8;      // activation rows per CTA
constexpr int AG_WARPS = 8;   // output columns per CTA

// win0[b][w][l][c] = states[b][clamp(s0 - 2 + w)][l][c]  (w < 5)
// winv[b][j-1][g][l][c] = states[b][clamp(s0 + 8j - 7 - 2 + g)][l][c]  (g < 12)
__global__ void audio_windows_kernel(const float* __restrict__ states, float* __restrict__ win0,
                                     float* __restrict__ winv, int batch, int S, int per_state, int F, int s0,
                                     int window, int stride, int group) {
  pdl_launch_dependents();
  pdl_wait();
  const long n0 = (long)batch * window * per_state;
  const long nv = (long)batch * (F - 1) * group * per_state;
  const int half = window / 2;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n0 + nv; i += (long)gridDim.x * blockDim.x) {
    long r = i < n0 ? i : i - n0;
    const int c = (int)(r % per_state);
    r /= per_state;
    int pos;
    int b;
    if (i < n0) {
      const int w = (int)(r % window);
      b = (int)(r / window);
      pos = s0 - half + w;
    } else {
      const int g = (int)(r % group);
      r /= group;
      const int j = (int)(r % (F - 1)) + 1;
      b = (int)(r / (F - 1));
      pos = s0 + stride * j - (stride - 1) - half + g;
    }
    pos = pos < 0 ? 0 : (pos > S - 1 ? S - 1 : pos);
    const float v = states[((long)b * S + pos) * per_state + c];
    if (i < n0)
      win0[i] = v;
    else
      winv[i - n0] = v;
  }
}

// part[kc][r][n] = sum over k in chunk kc of W[n][k] * x[r][k], rows r of group blockIdx.z
template <typename WT>
__global__ void __launch_bounds__(32 * AG_WARPS) audio_gemv_kernel(const WT* __restrict__ W,
                                                                   const float* __restrict__ x,
                                                                   float* __restrict__ part, int N, int K, int R) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ __align__(16) float xs[AG_RG][AG_KC];
  const int kc = blockIdx.y;
  const int k0 = kc * AG_KC;
  const int kn = min(AG_KC, K - k0);
  const int r0 = blockIdx.z * AG_RG;
  const int nr = min(AG_RG, R - r0);
  for (int i = threadIdx.x; i < nr * kn; i += blockDim.x) {
    const int r = i / kn, k = i - r * kn;
    xs[r][k] = x[(long)(r0 + r) * K + k0 + k];
  }
  __syncthreads();
  const int n = blockIdx.x * AG_WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  float acc[AG_RG];
#pragma unroll
  for (int r = 0; r < AG_RG; ++r) acc[r] = 0.f;
  const WT* wr = W + (long)n * K + k0;
  if (sizeof(WT) == 2 && kn % 256 == 0 && (K % 8) == 0) {
#pragma unroll 2
    for (int k = lane * 8; k < kn; k += 256) {
      float w8[8];
      load8(reinterpret_cast<const bf16*>(wr) + k, w8);
#pragma unroll
      for (int r = 0; r < AG_RG; ++r) {
        if (r < nr) {
          const float4 a = *reinterpret_cast<const float4*>(&xs[r][k]);
          const float4 c = *reinterpret_cast<const float4*>(&xs[r][k + 4]);
          float s = acc[r];
          s = fmaf(w8[0], a.x, s); s = fmaf(w8[1], a.y, s); s = fmaf(w8[2], a.z, s); s = fmaf(w8[3], a.w, s);
          s = fmaf(w8[4], c.x, s); s = fmaf(w8[5], c.y, s); s = fmaf(w8[6], c.z, s); s = fmaf(w8[7], c.w, s);
          acc[r] = s;
        }
      }
    }
  } else {
    for (int k = lane; k < kn; k += 32) {
      const float wv = to_f(wr[k]);
#pragma unroll
      for (int r = 0; r < AG_RG; ++r)
        if (r < nr) acc[r] = fmaf(wv, xs[r][k], acc[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < AG_RG; ++r) {
    if (r < nr) {
      const float s = warp_sum(acc[r]);
      if (lane == 0) part[((long)kc * R + r0 + r) * N + n] = s;
    }
  }
}

// y[out_row(r)][n] = act(sum_kc part[kc][r][n] + bias[n]), out_row(r) = (r / per) * ostride + r % per + ooff
__global__ void audio_reduce_kernel(const float* __restrict__ part, const float* __restrict__ bias,
                                    float* __restrict__ y, int N, int R, int nkc, int relu, int per, int ostride,
                                    int ooff) {
  pdl_launch_dependents();
  pdl_wait();
  const long total = (long)R * N;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int r = (int)(i / N), n = (int)(i - (long)r * N);
    float s = 0.f;
    for (int kc = 0; kc < nkc; ++kc) s += part[((long)kc * R + r) * N + n];
    s += bias[n];
    if (relu) s = fmaxf(s, 0.f);
    y[((long)(r / per) * ostride + r % per + ooff) * N + n] = s;
  }
}

}  // namespace

cudaError_t audio_windows(const float* states, float* win0, float* winv, int batch, int S, int per_state, int F,
                          int s0, int window, int stride, int group, cudaStream_t st) {
  const long n = (long)batch * (window + (long)(F - 1) * group) * per_state;
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  return launch_pdl(audio_windows_kernel, dim3(grid), dim3(256), 0, st, states, win0, winv, batch, S, per_state, F,
                    s0, window, stride, group);
}

int audio_gemv_chunks(int K) { return (K + AG_KC - 1) / AG_KC; }

template <typename WT>
cudaError_t audio_linear(const WT* W, const float* x, const float* bias, float* part, float* y, int N, int K, int R,
                         int relu, int per, int ostride, int ooff, cudaStream_t st) {
  const int nkc = audio_gemv_chunks(K);
  dim3 grid((N + AG_WARPS - 1) / AG_WARPS, nkc, (R + AG_RG - 1) / AG_RG);
  cudaError_t e = launch_pdl(audio_gemv_kernel<WT>, grid, dim3(32 * AG_WARPS), 0, st, W, x, part, N, K, R);
  if (e != cudaSuccess) return e;
  const long total = (long)R * N;
  const int g2 = (int)((total + 255) / 256 < 2048 ? (total + 255) / 256 : 2048);
  return launch_pdl(audio_reduce_kernel, dim3(g2), dim3(256), 0, st, part, bias, y, N, R, nkc, relu, per, ostride,
                    ooff);
}
template cudaError_t audio_linear<bf16>(const bf16*, const float*, const float*, float*, float*, int, int, int, int,
                                        int, int, int, cudaStream_t);
template cudaError_t audio_linear<float>(const float*, const float*, const float*, float*, float*, int, int, int,
                                         int, int, int, int, cudaStream_t);

}  // namespace fh
