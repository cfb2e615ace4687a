// rownorm.cuh - one row's norm and modulation, by one warp.
//
// D = 128 * NV floats held in registers (a float4 per lane per step). Mode 0 / 2: the adaLN
// modulate h = n(x) * (1 + scale) + shift of the Wan-style block (reading R1) and of the
// output norm (headMods, gizai:flashhead Types > FlashHead, reading R9), n a LayerNorm (mode 0)
// or an RMSNorm without gain (mode 2); mode 1: the learned-affine LayerNorm before the audio
// cross-attention (reading R7, a = weight, c = bias). Biased variance, eps inside the root (R2).
#pragma once

#include "common.cuh"

namespace fh {

// xr: the row (fp32, read through L2); a, c: scale and shift (modes 0, 2) or weight and bias
// (mode 1) for this row's stream; orow: the output row.
template <typename T, int NV>
__device__ __forceinline__ void norm_row(const float* xr, T* orow, int lane, int mode, const float* a,
                                         const float* c, float eps) {
  constexpr int D = NV * 128;
  float4 v[NV], ma[NV], mc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = __ldcg(reinterpret_cast<const float4*>(xr) + lane + 32 * i);
  // the affine / modulation vectors are loaded alongside the row, before the reductions
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    ma[i] = reinterpret_cast<const float4*>(a)[lane + 32 * i];
    mc[i] = reinterpret_cast<const float4*>(c)[lane + 32 * i];
  }
  float mu = 0.f, rstd;
  if (mode != 2) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    mu = warp_sum(s) * (1.f / D);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float p = v[i].x - mu, r = v[i].y - mu, t = v[i].z - mu, u = v[i].w - mu;
      q += (p * p + r * r) + (t * t + u * u);
    }
    rstd = rsqrtf(warp_sum(q) * (1.f / D) + eps);
  } else {
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) q += (v[i].x * v[i].x + v[i].y * v[i].y) + (v[i].z * v[i].z + v[i].w * v[i].w);
    rstd = rsqrtf(warp_sum(q) * (1.f / D) + eps);
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int col = (lane + 32 * i) * 4;
    float y[4] = {(v[i].x - mu) * rstd, (v[i].y - mu) * rstd, (v[i].z - mu) * rstd, (v[i].w - mu) * rstd};
    float4 g = ma[i];
    const float4 h = mc[i];
    if (mode != 1) {
      g.x += 1.f; g.y += 1.f; g.z += 1.f; g.w += 1.f;
    }
    y[0] = y[0] * g.x + h.x;
    y[1] = y[1] * g.y + h.y;
    y[2] = y[2] * g.z + h.z;
    y[3] = y[3] * g.w + h.w;
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(y[2], y[3]);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(orow + col) = u;
    } else {
      *reinterpret_cast<float4*>(orow + col) = make_float4(y[0], y[1], y[2], y[3]);
    }
  }
}

}  // namespace fh
