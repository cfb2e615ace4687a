// misc.cu - CUDA-core kernels of the DiT hot path: row norms with adaLN
// modulation, per-frame audio cross-attention, timestep conditioning, latent
// layout/Euler/motion pinning, the seeded weight generator, and the fp32 GEMM of
// the fp32 configuration.
#include <math.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "rownorm.cuh"

namespace fh {

namespace {

// ------------------------------------------------------------------ row norms
// One warp per row (rownorm.cuh): the adaLN modulate of the block and of the output norm
// (modes 0, 2) and the learned-affine LayerNorm before the audio cross-attention (mode 1).
template <typename T, int NV>
__global__ void norm_rows_kernel(const float* __restrict__ x, T* __restrict__ out, int M, int rows_per_batch,
                                 int mode, const float* __restrict__ shift, const float* __restrict__ scale,
                                 long mod_bstride, const float* __restrict__ w, const float* __restrict__ bb,
                                 float eps) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int D = NV * 128;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const long mb = (long)(row / rows_per_batch) * mod_bstride;
  norm_row<T, NV>(x + (long)row * D, out + (long)row * D, lane, mode, mode == 1 ? w : scale + mb,
                  mode == 1 ? bb : shift + mb, eps);
}

// ------------------------------------------------------ per-frame cross-attention
// A token of latent frame f attends to frame f's A = 32 audio tokens only (gizai:flashhead,
// opening paragraph: 5 latent frames of 32 audio tokens; reading R5). One CTA per (frame,
// head, stream, chunk of XA_QPB queries) stages that frame's keys/values (fp32) and key RMS
// factors in shared memory. Each warp takes XA_QPW queries at once: for the scores lane a
// owns audio key a and every float4 of k_a read from shared memory serves all XA_QPW
// queries; for the output lane l owns dims 4l..4l+3 and every float4 of v_a serves all of
// them, so shared-memory traffic per query is XA_QPW times smaller than one query at a time.
constexpr int XA_WARPS = 8;
constexpr int XA_QPW = 8;                    // queries per warp, processed together
constexpr int XA_QPB = XA_WARPS * XA_QPW;    // queries per CTA
constexpr int XA_A = 32;                     // audio tokens per latent frame
constexpr int XA_KS = 132;                   // padded row stride of staged keys (float4-aligned)
constexpr size_t XA_SMEM = (size_t)XA_A * XA_KS * 4 + (size_t)XA_A * 128 * 4 + (size_t)XA_WARPS * XA_QPW * 128 * 4 +
                           XA_A * 4;

template <typename T>
__device__ __forceinline__ float4 load4f(const T* p) {
  if constexpr (sizeof(T) == 2) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    float2 a0 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
    float2 a1 = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
    return make_float4(a0.x, a0.y, a1.x, a1.y);
  } else {
    return *reinterpret_cast<const float4*>(p);
  }
}

template <typename T>
__global__ void __launch_bounds__(XA_WARPS * 32)
    cross_attn_kernel(const T* __restrict__ q, const float* __restrict__ ssq_q, const T* __restrict__ kv, long ldkv,
                      int koff, int voff, const float* __restrict__ ssq_k, int ssq_k_ld, int ssq_k_off, int heads,
                      int L, int F, int nqc, float eps, float scale, T* __restrict__ out) {
  extern __shared__ __align__(16) float xa_smem[];
  float* ks = xa_smem;                                   // [A][XA_KS]
  float* vs = ks + XA_A * XA_KS;                         // [A][128]
  float* qs = vs + XA_A * 128;                           // [warps][QPW][128]
  float* rks = qs + XA_WARPS * XA_QPW * 128;             // [A]
  pdl_launch_dependents();
  pdl_wait();
  const int f = blockIdx.x / nqc, qc = blockIdx.x % nqc;
  const int h = blockIdx.y, b = blockIdx.z;
  const int D = heads * 128;
  const float inv_d = 1.f / (float)D;
  const long kv_row0 = ((long)b * F + f) * XA_A;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int HW = L / F;
  const int n0 = qc * XA_QPB + warp * XA_QPW;
  // this warp's query slices and RMS partial sums, all loads in flight together
  float4 qv[XA_QPW];
  float sq[XA_QPW];
#pragma unroll
  for (int i = 0; i < XA_QPW; ++i) {
    const int n = n0 + i < HW ? n0 + i : HW - 1;
    const long row = (long)b * L + (long)f * HW + n;
    sq[i] = lane < heads ? ssq_q[row * heads + lane] : 0.f;
    qv[i] = load4f(q + row * D + h * 128 + lane * 4);
  }
  for (int idx = threadIdx.x; idx < XA_A * 32; idx += blockDim.x) {
    const int a = idx >> 5, d = (idx & 31) * 4;
    const T* r = kv + (kv_row0 + a) * ldkv;
    *reinterpret_cast<float4*>(&ks[a * XA_KS + d]) = load4f(r + koff + h * 128 + d);
    *reinterpret_cast<float4*>(&vs[a * 128 + d]) = load4f(r + voff + h * 128 + d);
  }
  if (threadIdx.x < XA_A) {
    const float* p = ssq_k + (kv_row0 + threadIdx.x) * ssq_k_ld + ssq_k_off;
    float s = 0.f;
    for (int i = 0; i < heads; ++i) s += p[i];
    rks[threadIdx.x] = rsqrtf(s * inv_d + eps);
  }
  float* qw = qs + warp * XA_QPW * 128;
#pragma unroll
  for (int i = 0; i < XA_QPW; ++i) *reinterpret_cast<float4*>(&qw[i * 128 + lane * 4]) = qv[i];
  __syncthreads();
  if (n0 >= HW) return;

  // scores: lane = audio key
  float s[XA_QPW];
#pragma unroll
  for (int i = 0; i < XA_QPW; ++i) s[i] = 0.f;
  const float* kr = ks + lane * XA_KS;
#pragma unroll 4
  for (int d = 0; d < 128; d += 4) {
    const float4 k4 = *reinterpret_cast<const float4*>(kr + d);
#pragma unroll
    for (int i = 0; i < XA_QPW; ++i) {
      const float4 q4 = *reinterpret_cast<const float4*>(qw + i * 128 + d);
      s[i] = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, fmaf(q4.w, k4.w, s[i]))));
    }
  }
  const float rk = rks[lane] * scale;
#pragma unroll
  for (int i = 0; i < XA_QPW; ++i) {
    const float rq = rsqrtf(warp_sum(sq[i]) * inv_d + eps);
    const float si = s[i] * rq * rk;
    const float m = warp_max(si);
    const float p = expf(si - m);
    s[i] = p / warp_sum(p);  // normalised weight of key `lane` for query i
  }
  // output: lane = 4 dims
  float4 o[XA_QPW];
#pragma unroll
  for (int i = 0; i < XA_QPW; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int a = 0; a < XA_A; ++a) {
    const float4 vv = *reinterpret_cast<const float4*>(&vs[a * 128 + lane * 4]);
#pragma unroll
    for (int i = 0; i < XA_QPW; ++i) {
      const float pa = __shfl_sync(0xffffffffu, s[i], a);
      o[i].x = fmaf(pa, vv.x, o[i].x);
      o[i].y = fmaf(pa, vv.y, o[i].y);
      o[i].z = fmaf(pa, vv.z, o[i].z);
      o[i].w = fmaf(pa, vv.w, o[i].w);
    }
  }
#pragma unroll
  for (int i = 0; i < XA_QPW; ++i) {
    const int n = n0 + i;
    if (n >= HW) break;
    T* dst = out + ((long)b * L + (long)f * HW + n) * D + h * 128 + lane * 4;
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(o[i].x, o[i].y);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(o[i].z, o[i].w);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(dst) = u;
    } else {
      *reinterpret_cast<float4*>(dst) = o[i];
    }
  }
}

// ------------------------------------------------------------ conditioning
// 256-dim sinusoid of tau = 1000 t: [cos(tau w_k) | sin(tau w_k)], w_k = 10000^(-k/128)
// (reading R10 of the timestep embedding that yields the per-step modulations,
// gizai:flashhead Types > FlashHead, field headMods).
__global__ void time_sinusoid_kernel(float* out, int batch, TVals tv, int dim) {
  pdl_launch_dependents();
  pdl_wait();
  const int half = dim / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= batch * dim) return;
  const int b = idx / dim, k = idx % dim;
  const int kk = k < half ? k : k - half;
  const double w = pow(10000.0, -(double)kk / (double)half);
  const double ang = 1000.0 * (double)tv.t[b] * w;
  out[idx] = (float)(k < half ? cos(ang) : sin(ang));
}

// y[b, n] = act(sum_k W[n, k] * act_in(x[b, k]) + bias[n]); one warp per output.
constexpr int GV_CHUNKS = 8;  // 16-byte bf16 loads per lane held in registers (K up to 2048)
template <typename WT>
__global__ void gemv_kernel(const WT* __restrict__ W, const float* __restrict__ x, const float* __restrict__ bias,
                            float* __restrict__ y, int N, int K, int batch, int silu_in, int silu_out) {
  pdl_launch_dependents();
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const WT* wr = W + (long)(n < N ? n : 0) * K;
  // bf16 rows: the whole row's weights (8 per lane per 16-byte load) are requested at once,
  // before the dependency wait (the weights are never written by any kernel), so the loads
  // overlap the preceding kernel and the staging of x
  const bool vec = sizeof(WT) == 2 && K % 256 == 0 && K <= 256 * GV_CHUNKS;
  const int nc = K / 256;
  uint4 wq[GV_CHUNKS];
  if (vec) {
#pragma unroll
    for (int c = 0; c < GV_CHUNKS; ++c)
      if (c < nc) wq[c] = __ldg(reinterpret_cast<const uint4*>(wr + c * 256 + lane * 8));
  }
  pdl_wait();
  extern __shared__ float xs[];
  for (int i = threadIdx.x; i < batch * K; i += blockDim.x) {
    const float v = x[i];
    xs[i] = silu_in ? silu(v) : v;
  }
  __syncthreads();
  if (n >= N) return;
  float acc[8];
  for (int b = 0; b < batch; ++b) acc[b] = 0.f;
  if (vec) {
#pragma unroll
    for (int c = 0; c < GV_CHUNKS; ++c) {
      if (c >= nc) break;
      const int k0 = c * 256 + lane * 8;
      float w8[8];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&wq[c]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        w8[2 * e] = f.x;
        w8[2 * e + 1] = f.y;
      }
      for (int b = 0; b < batch; ++b) {
        const float4 x0 = *reinterpret_cast<const float4*>(xs + b * K + k0);
        const float4 x1 = *reinterpret_cast<const float4*>(xs + b * K + k0 + 4);
        float a = acc[b];
        a = fmaf(w8[0], x0.x, a); a = fmaf(w8[1], x0.y, a); a = fmaf(w8[2], x0.z, a); a = fmaf(w8[3], x0.w, a);
        a = fmaf(w8[4], x1.x, a); a = fmaf(w8[5], x1.y, a); a = fmaf(w8[6], x1.z, a); a = fmaf(w8[7], x1.w, a);
        acc[b] = a;
      }
    }
  } else {
    for (int k = lane; k < K; k += 32) {
      const float wv = to_f(wr[k]);
      for (int b = 0; b < batch; ++b) acc[b] = fmaf(wv, xs[b * K + k], acc[b]);
    }
  }
  for (int b = 0; b < batch; ++b) {
    float s = warp_sum(acc[b]);
    if (lane == 0) {
      s += bias[n];
      y[(long)b * N + n] = silu_out ? silu(s) : s;
    }
  }
}

__global__ void assemble_mods_kernel(const float* __restrict__ table, const float* __restrict__ e0,
                                     const float* __restrict__ htable, const float* __restrict__ e,
                                     float* __restrict__ mods, float* __restrict__ hmods, int batch, int blocks,
                                     int D) {
  pdl_launch_dependents();
  pdl_wait();
  const long per = (long)blocks * 6 * D;
  const long total = (long)batch * per;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total + (long)batch * 2 * D;
       i += (long)gridDim.x * blockDim.x) {
    if (i < total) {
      const long b = i / per, r = i % per;
      const long ic = r % (6L * D);  // (i, c) within the block
      mods[i] = table[r] + e0[b * 6L * D + ic];
    } else {
      const long j = i - total;
      const long b = j / (2L * D), r = j % (2L * D);
      hmods[j] = htable[r] + e[b * D + (r % D)];
    }
  }
}

// ------------------------------------------------------------------ latents
// Channel-first latents [B, C, L] -> token-major rows: lat[b*L+n][c] (float32, optional)
// and the patch-embed input tok[b*L+n] = [x | ref] in T (the noisy latent's channels
// first, reading R16). Frames below pin_frames take the motion latent (reading R14).
template <typename T>
__global__ void prep_tokens_kernel(const float* __restrict__ x, const float* __restrict__ ref,
                                   const float* __restrict__ motion, int pin_frames, float* __restrict__ lat,
                                   T* __restrict__ tok, int C, int L, int HW) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float tx[32][33];
  __shared__ float tr[32][33];
  const int b = blockIdx.z;
  const int n0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  const int pinned = pin_frames * HW;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, n = n0 + threadIdx.x;
    float xv = 0.f, rv = 0.f;
    if (n < L) {
      const long src = ((long)b * C + c) * L + n;
      xv = (motion != nullptr && n < pinned) ? motion[((long)b * C + c) * pinned + n] : x[src];
      rv = ref[src];
    }
    tx[i][threadIdx.x] = xv;
    tr[i][threadIdx.x] = rv;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i, c = c0 + threadIdx.x;
    if (n >= L) continue;
    const long row = (long)b * L + n;
    const float xv = tx[threadIdx.x][i];
    if (lat) lat[row * C + c] = xv;
    tok[row * 2 * C + c] = from_f<T>(xv);
    tok[row * 2 * C + C + c] = from_f<T>(tr[threadIdx.x][i]);
  }
}

// Euler step of the flow sampler, x <- x + (sigma' - sigma) v on unpinned tokens
// (readings R12, R14), then the next patch-embed input for those channels.
template <typename T>
__global__ void euler_kernel(float* __restrict__ lat, const float* __restrict__ v, float dsig, int pinned_tokens,
                             T* __restrict__ tok, int C, int L, long total) {
  pdl_launch_dependents();
  pdl_wait();
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long row = i / C;
    const int c = (int)(i % C);
    const int n = (int)(row % L);
    float x = lat[i];
    if (n >= pinned_tokens) {
      x = fmaf(dsig, v[i], x);
      lat[i] = x;
    }
    tok[row * 2 * C + c] = from_f<T>(x);
  }
}

// The re-noising step (reading R12 of the update the audio-cpp doc names for distilled
// checkpoints): x0 = x - sigma v, then x = (1 - sigma') x0 + sigma' eps with this step's
// fresh draw eps, channel-first [B, C, L]; the motion tokens (n < pinned_tokens) keep x.
// At sigma' = 0 it computes the Euler step's fmaf(-sigma, v, x) exactly.
template <typename T>
__global__ void renoise_kernel(float* __restrict__ lat, const float* __restrict__ v, const float* __restrict__ eps,
                               float sig, float sig_next, int pinned_tokens, T* __restrict__ tok, int C, int L,
                               long total) {
  pdl_launch_dependents();
  pdl_wait();
  const float keep = 1.f - sig_next;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long row = i / C;
    const int c = (int)(i % C);
    const int n = (int)(row % L);
    const long b = row / L;
    float x = lat[i];
    if (n >= pinned_tokens) {
      const float x0 = fmaf(-sig, v[i], x);
      x = fmaf(sig_next, eps[(b * C + c) * L + n], keep * x0);
      lat[i] = x;
    }
    tok[row * 2 * C + c] = from_f<T>(x);
  }
}

__global__ void tokens_to_latent_kernel(const float* __restrict__ tok, float* __restrict__ out, int C, int L) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float t[32][33];
  const int b = blockIdx.z;
  const int n0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i;
    t[i][threadIdx.x] = n < L ? tok[((long)b * L + n) * C + c0 + threadIdx.x] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, n = n0 + threadIdx.x;
    if (n < L) out[((long)b * C + c) * L + n] = t[threadIdx.x][i];
  }
}

// ------------------------------------------------------------ seeded weights
// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) as a hash of a counter, two 53-bit
// uniforms per element and one Box-Muller normal, all in float64 with explicitly
// rounded operations so the value is the same as a host evaluation of the formula.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double seeded_normal(uint64_t base, uint64_t i) {
  const uint64_t c1 = base + 2ull * i;
  const double u1 = (double)(splitmix64(c1) >> 11) * 0x1.0p-53;
  const double u2 = (double)(splitmix64(c1 + 1ull) >> 11) * 0x1.0p-53;
  const double r = sqrt(__dmul_rn(-2.0, log1p(-u1)));
  const double a = __dmul_rn(2.0 * 3.141592653589793, u2);
  return __dmul_rn(r, cos(a));
}

template <typename T>
__global__ void gen_tensor_kernel(T* __restrict__ dst, long rows, long cols, long ld, uint64_t base, int kind,
                                  double fan_sqrt, bool round_bf16) {
  pdl_launch_dependents();
  pdl_wait();
  const long n = rows * cols;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const double z = seeded_normal(base, (uint64_t)i);
    double w;
    if (kind == 0)
      w = __ddiv_rn(z, fan_sqrt);
    else if (kind == 1)
      w = __dadd_rn(1.0, __dmul_rn(0.1, z));
    else
      w = __dmul_rn(0.1, z);
    float f = __double2float_rn(w);
    if (round_bf16) f = __bfloat162float(__float2bfloat16_rn(f));
    dst[(i / cols) * ld + (i % cols)] = from_f<T>(f);
  }
}

// rotary (cos, sin) per token and pair: pairs [0, pf) turn with the frame index,
// [pf, pf+ph) with the row, the rest with the column; pair j of an axis with n dims
// turns theta^(-2j/n) rad per position (reading R3; table shape as the `cos`/`sin`
// fields of gizai:flashhead Types > FlashHead, one head's 64 columns).
// Rotary (cos, sin) per axis (reading R3): [F][pf] by frame index, [H][ph] by row, [W][pw] by
// column, one after the other; pair j of an axis of n = 2 * (pairs) dims at position pos turns
// pos * theta^(-2j / n) radians (float64, then rounded to float32).
__global__ void rope_table_kernel(float2* tab, int F, int H, int W, int pf, int ph, int pw, double theta) {
  pdl_launch_dependents();
  pdl_wait();
  const int L = F * H * W;
  const int np = pf + ph + pw;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= L * np) return;
  const int n = idx / np, d = idx % np;
  const int f = n / (H * W), r = (n / W) % H, c = n % W;
  int pos, j, ndim;
  if (d < pf) {
    pos = f; j = d; ndim = 2 * pf;
  } else if (d < pf + ph) {
    pos = r; j = d - pf; ndim = 2 * ph;
  } else {
    pos = c; j = d - pf - ph; ndim = 2 * pw;
  }
  const double ang = (double)pos * pow(theta, -2.0 * (double)j / (double)ndim);
  tab[idx] = make_float2((float)cos(ang), (float)sin(ang));
}

__global__ void fill_kernel(float* p, long n, float v) {
  pdl_launch_dependents();
  pdl_wait();
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) p[i] = v;
}

// ------------------------------------------------------------ fp32 GEMM
// 32 x 128 output tile per CTA; thread t owns row t%32 and the 32 columns (t/32)*32..
// so the shared epilogue sees whole 32-column chunks of one row.
template <int KIND>
__global__ void __launch_bounds__(128) gemm_simt_kernel(const float* __restrict__ A, long lda,
                                                        const float* __restrict__ W, long ldw, int M, int N, int K,
                                                        EpiParams ep) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float As[32][33];
  __shared__ float Ws[32][129];
  __shared__ float ssq_s[4][32];
  const int t = threadIdx.x;
  const int r = t & 31, q = t >> 5;
  const int m0 = blockIdx.y * 32, n0 = blockIdx.x * 128;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int i = t; i < 32 * 32; i += 128) {
      const int kk = i & 31, rr = i >> 5;
      As[kk][rr] = (m0 + rr < M && k0 + kk < K) ? A[(long)(m0 + rr) * lda + k0 + kk] : 0.f;
    }
    for (int i = t; i < 32 * 128; i += 128) {
      const int kk = i & 31, cc = i >> 5;
      Ws[kk][cc] = (k0 + kk < K) ? W[(long)(n0 + cc) * ldw + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      const float a = As[kk][r];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = fmaf(a, Ws[kk][q * 32 + j], acc[j]);
    }
    __syncthreads();
  }
  const int row = m0 + r;
  float ssq = 0.f;
  if (row < M) epi_chunk<KIND, float>(ep, row, n0 + q * 32, acc, ssq);
  ssq_s[q][r] = ssq;
  __syncthreads();
  if (q == 0 && row < M) epi_group_end<KIND>(ep, row, n0, ssq_s[0][r] + ssq_s[1][r] + ssq_s[2][r] + ssq_s[3][r]);
}

// One CTA waits on an mbarrier that nothing arrives at: the bounded wait of the
// production kernels runs out, latches its error bit and the kernel returns normally.
__global__ void wait_probe_kernel(unsigned* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, ERRBIT_TIMEOUT_GEMM);
}

inline int grid_for(long n, int block) {
  long g = (n + block - 1) / block;
  if (g > 148 * 16) g = 148 * 16;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

// ------------------------------------------------------------------ launchers
cudaError_t gemm_simt(const float* A, long lda, const float* W, long ldw, int M, int N, int K, int kind,
                      const EpiParams& ep, cudaStream_t st) {
  if (N % 128 != 0) return cudaErrorInvalidValue;
  dim3 grid(N / 128, (M + 31) / 32);
  switch (kind) {
    case EPI_STORE: { cudaError_t e_ = launch_pdl(gemm_simt_kernel<EPI_STORE>, dim3(grid), dim3(128), 0, st, A, lda, W, ldw, M, N, K, ep); if (e_ != cudaSuccess) return e_; } break;
    case EPI_GELU: { cudaError_t e_ = launch_pdl(gemm_simt_kernel<EPI_GELU>, dim3(grid), dim3(128), 0, st, A, lda, W, ldw, M, N, K, ep); if (e_ != cudaSuccess) return e_; } break;
    case EPI_RESID: { cudaError_t e_ = launch_pdl(gemm_simt_kernel<EPI_RESID>, dim3(grid), dim3(128), 0, st, A, lda, W, ldw, M, N, K, ep); if (e_ != cudaSuccess) return e_; } break;
    case EPI_NORM: { cudaError_t e_ = launch_pdl(gemm_simt_kernel<EPI_NORM>, dim3(grid), dim3(128), 0, st, A, lda, W, ldw, M, N, K, ep); if (e_ != cudaSuccess) return e_; } break;
    case EPI_QKV: { cudaError_t e_ = launch_pdl(gemm_simt_kernel<EPI_QKV>, dim3(grid), dim3(128), 0, st, A, lda, W, ldw, M, N, K, ep); if (e_ != cudaSuccess) return e_; } break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t cross_attn_prepare() {
  cudaError_t e = cudaFuncSetAttribute(cross_attn_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)XA_SMEM);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(cross_attn_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)XA_SMEM);
}

template <typename T>
cudaError_t cross_attn(const T* q, const float* ssq_q, const T* kv, long ldkv, int koff, int voff,
                       const float* ssq_k, int ssq_k_ld, int ssq_k_off, int batch, int heads, int L, int F, int A,
                       float eps, T* out, cudaStream_t st) {
  if (A != XA_A || heads > 32) return cudaErrorInvalidValue;
  const int HW = L / F;
  const int nqc = (HW + XA_QPB - 1) / XA_QPB;
  dim3 grid(F * nqc, heads, batch);
  return launch_pdl(cross_attn_kernel<T>, grid, dim3(XA_WARPS * 32), XA_SMEM, st, q, ssq_q, kv, ldkv, koff, voff,
                    ssq_k, ssq_k_ld, ssq_k_off, heads, L, F, nqc, eps, 1.f / sqrtf(128.f), out);
}

template cudaError_t cross_attn<float>(const float*, const float*, const float*, long, int, int, const float*, int,
                                       int, int, int, int, int, int, float, float*, cudaStream_t);
template cudaError_t cross_attn<bf16>(const bf16*, const float*, const bf16*, long, int, int, const float*, int,
                                      int, int, int, int, int, int, float, bf16*, cudaStream_t);

template <typename T>
cudaError_t norm_rows(const float* x, T* out, int M, int D, int rows_per_batch, int mode, const float* shift,
                      const float* scale, long mod_bstride, const float* w, const float* bb, float eps,
                      cudaStream_t st) {
  const int rows_per_cta = 4;
  dim3 grid((M + rows_per_cta - 1) / rows_per_cta);
#define FH_NORM_CASE(NVV)                                                                                     \
  case NVV:                                                                                                   \
    { cudaError_t e_ = launch_pdl(norm_rows_kernel<T, NVV>, dim3(grid), dim3(32 * rows_per_cta), 0, st, x, out, M, rows_per_batch, mode, shift, scale, \
                                                                 mod_bstride, w, bb, eps); if (e_ != cudaSuccess) return e_; }                    \
    break;
  switch (D / 128) {
    FH_NORM_CASE(1) FH_NORM_CASE(2) FH_NORM_CASE(3) FH_NORM_CASE(4) FH_NORM_CASE(6) FH_NORM_CASE(8)
    FH_NORM_CASE(12) FH_NORM_CASE(16)
    default: return cudaErrorInvalidValue;
  }
#undef FH_NORM_CASE
  return cudaGetLastError();
}
template cudaError_t norm_rows<float>(const float*, float*, int, int, int, int, const float*, const float*, long,
                                      const float*, const float*, float, cudaStream_t);
template cudaError_t norm_rows<bf16>(const float*, bf16*, int, int, int, int, const float*, const float*, long,
                                     const float*, const float*, float, cudaStream_t);

cudaError_t time_sinusoid(float* out, int batch, TVals tv, int dim, cudaStream_t st) {
  const int n = batch * dim;
  { cudaError_t e_ = launch_pdl(time_sinusoid_kernel, dim3((n + 255) / 256), dim3(256), 0, st, out, batch, tv, dim); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

template <typename WT>
cudaError_t gemv(const WT* W, const float* x, const float* bias, float* y, int N, int K, int batch, int silu_in,
                 int silu_out, cudaStream_t st) {
  if (batch > 8) return cudaErrorInvalidValue;
  const size_t smem = (size_t)batch * K * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  { cudaError_t e_ = launch_pdl(gemv_kernel<WT>, dim3((N + 7) / 8), dim3(256), smem, st, W, x, bias, y, N, K, batch, silu_in, silu_out); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}
template cudaError_t gemv<float>(const float*, const float*, const float*, float*, int, int, int, int, int,
                                 cudaStream_t);
template cudaError_t gemv<bf16>(const bf16*, const float*, const float*, float*, int, int, int, int, int,
                                cudaStream_t);

cudaError_t assemble_mods(const float* table, const float* e0, const float* htable, const float* e, float* mods,
                          float* hmods, int batch, int blocks, int D, cudaStream_t st) {
  const long n = (long)batch * blocks * 6 * D + (long)batch * 2 * D;
  { cudaError_t e_ = launch_pdl(assemble_mods_kernel, dim3(grid_for(n, 256)), dim3(256), 0, st, table, e0, htable, e, mods, hmods, batch, blocks, D); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

template <typename T>
cudaError_t prep_tokens(const float* x, const float* ref, const float* motion, int pin_frames, float* lat, T* tok,
                        int batch, int C, int L, int HW, cudaStream_t st) {
  if (C % 32 != 0) return cudaErrorInvalidValue;
  dim3 grid((L + 31) / 32, C / 32, batch);
  { cudaError_t e_ = launch_pdl(prep_tokens_kernel<T>, dim3(grid), dim3(dim3(32, 8)), 0, st, x, ref, motion, pin_frames, lat, tok, C, L, HW); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}
template cudaError_t prep_tokens<float>(const float*, const float*, const float*, int, float*, float*, int, int, int,
                                        int, cudaStream_t);
template cudaError_t prep_tokens<bf16>(const float*, const float*, const float*, int, float*, bf16*, int, int, int,
                                       int, cudaStream_t);

template <typename T>
cudaError_t euler_step(float* lat, const float* v, float dsig, int pinned_tokens, T* tok, int batch, int C, int L,
                       cudaStream_t st) {
  const long n = (long)batch * L * C;
  { cudaError_t e_ = launch_pdl(euler_kernel<T>, dim3(grid_for(n, 256)), dim3(256), 0, st, lat, v, dsig, pinned_tokens, tok, C, L, n); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}
template cudaError_t euler_step<float>(float*, const float*, float, int, float*, int, int, int, cudaStream_t);
template cudaError_t euler_step<bf16>(float*, const float*, float, int, bf16*, int, int, int, cudaStream_t);

template <typename T>
cudaError_t renoise_step(float* lat, const float* v, const float* eps, float sig, float sig_next, int pinned_tokens,
                         T* tok, int batch, int C, int L, cudaStream_t st) {
  const long n = (long)batch * L * C;
  { cudaError_t e_ = launch_pdl(renoise_kernel<T>, dim3(grid_for(n, 256)), dim3(256), 0, st, lat, v, eps, sig, sig_next, pinned_tokens, tok, C, L, n); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}
template cudaError_t renoise_step<float>(float*, const float*, const float*, float, float, int, float*, int, int, int,
                                         cudaStream_t);
template cudaError_t renoise_step<bf16>(float*, const float*, const float*, float, float, int, bf16*, int, int, int,
                                        cudaStream_t);

cudaError_t tokens_to_latent(const float* tok, float* out, int batch, int C, int L, cudaStream_t st) {
  if (C % 32 != 0) return cudaErrorInvalidValue;
  dim3 grid((L + 31) / 32, C / 32, batch);
  { cudaError_t e_ = launch_pdl(tokens_to_latent_kernel, dim3(grid), dim3(dim3(32, 8)), 0, st, tok, out, C, L); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

template <typename T>
cudaError_t gen_tensor(T* dst, long rows, long cols, long ld, uint64_t seed, int tid, int kind, int fan,
                       bool round_bf16, cudaStream_t st) {
  const uint64_t base = seed ^ ((uint64_t)tid << 40);
  const long n = rows * cols;
  { cudaError_t e_ = launch_pdl(gen_tensor_kernel<T>, dim3(grid_for(n, 256)), dim3(256), 0, st, dst, rows, cols, ld, base, kind, sqrt((double)fan),
                                                         round_bf16); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}
template cudaError_t gen_tensor<float>(float*, long, long, long, uint64_t, int, int, int, bool, cudaStream_t);
template cudaError_t gen_tensor<bf16>(bf16*, long, long, long, uint64_t, int, int, int, bool, cudaStream_t);

cudaError_t rope_table(float2* tab, int F, int H, int W, int pf, int ph, int pw, float theta, cudaStream_t st) {
  const int n = F * H * W * (pf + ph + pw);
  { cudaError_t e_ = launch_pdl(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, st, tab, F, H, W, pf, ph, pw, (double)theta); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

cudaError_t wait_probe(unsigned* err, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

cudaError_t fill_f32(float* p, long n, float v, cudaStream_t st) {
  { cudaError_t e_ = launch_pdl(fill_kernel, dim3(grid_for(n, 256)), dim3(256), 0, st, p, n, v); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

}  // namespace fh
