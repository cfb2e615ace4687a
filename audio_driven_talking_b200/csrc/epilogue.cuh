// epilogue.cuh - fused GEMM epilogues of the DiT block.
//
// Every Linear of the block ends in one of these, applied by the thread that owns
// one output row to 32 consecutive columns at a time (columns come in groups of
// 128 = one attention head):
//   EPI_STORE  y = acc + bias                              (patch embed, head, v-part)
//   EPI_GELU   y = gelu_tanh(acc + bias)                    (FFN1)
//   EPI_RESID  x[row] += gate[stream] * (acc + bias)        (O-proj, cross-O, FFN2; gate
//                                                            null means 1: ungated, R8)
//   EPI_NORM   y = acc + bias; on "normed" columns the partial sum of y^2 over the
//              head's 128 columns goes to ssq[row, group] and y *= gain (cross-attn
//              q and k: full-width RMSNorm split per head, reading R4)
//   EPI_QKV    as EPI_NORM for the q and k sections, plus 3D rotary on adjacent
//              pairs (2d, 2d+1) of q and k, and a head-major scatter of q, k, v to
//              [3][B][heads][L][128] (reading R3). With bf16 outputs q and k are bf16
//              and v is fp16 (11-bit significand): the attention kernel multiplies it by
//              fp16 softmax weights P, and a tensor-core product takes A and B of one type.
// The RMS factor r = (sum(ssq)/D + eps)^-1/2 itself is applied later, inside the
// attention kernels, to the scores: r is one scalar per row and both the gain and
// the rotation are linear per channel, so RoPE(g * r * y) = r * RoPE(g * y).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace fh {

enum EpiKind { EPI_STORE = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_NORM = 3, EPI_QKV = 4 };

struct EpiParams {
  const float* bias;      // [N]
  void* out;              // output base (row-major [M, ldo] unless EPI_QKV)
  long ldo;
  float* resid;           // EPI_RESID: float32 residual [M, ldr]
  long ldr;
  const float* gate;      // EPI_RESID: gate[(row / rows_per_batch) * gate_bstride + col], or null
  long gate_bstride;
  int rows_per_batch;     // tokens per stream (L)
  const float* gain;      // EPI_NORM/QKV: gain[col] on normed columns
  float* ssq;             // EPI_NORM/QKV: ssq[row * ssq_ld + col / 128] on normed columns
  int ssq_ld;
  int norm_period;        // column c is normed iff (c % norm_period) < norm_count
  int norm_count;
  const float2* rope;     // EPI_QKV: (cos, sin) [rows_per_batch, 64]
  int dim;                // EPI_QKV: width D of each of the q, k, v sections
  long sec_stride;        // EPI_QKV: elements per section = B * heads * L * 128
};

__device__ __forceinline__ bool epi_normed(const EpiParams& p, int col) {
  return (col % p.norm_period) < p.norm_count;
}

// The arithmetic of the epilogue on 32 consecutive columns of one row, in registers:
//   EPI_STORE  v = acc + bias;   EPI_GELU  v = gelu_tanh(acc + bias)
//   EPI_RESID  v = gate * (acc + bias)  (the increment of the residual)
//   EPI_NORM / EPI_QKV  v = acc + bias; on normed columns ssq_acc += sum v^2 and v *= gain
// OutT is the type the result is stored in: bf16 results take the hardware tanh in GELU.
template <int KIND, typename OutT>
__device__ __forceinline__ void epi_math(const EpiParams& p, int row, int col0, float (&v)[32], float& ssq_acc) {
  const float* b = p.bias + col0;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    float4 bb = *reinterpret_cast<const float4*>(b + j);
    v[j] += bb.x; v[j + 1] += bb.y; v[j + 2] += bb.z; v[j + 3] += bb.w;
  }
  if constexpr (KIND == EPI_GELU) {
    if constexpr (std::is_same<OutT, bf16>::value) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = gelu_tanh_approx(v[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
    }
  } else if constexpr (KIND == EPI_RESID) {
    if (p.gate) {
      const float* g = p.gate + (long)(row / p.rows_per_batch) * p.gate_bstride + col0;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 gg = *reinterpret_cast<const float4*>(g + j);
        v[j] *= gg.x; v[j + 1] *= gg.y; v[j + 2] *= gg.z; v[j + 3] *= gg.w;
      }
    }
  } else if constexpr (KIND == EPI_NORM || KIND == EPI_QKV) {
    if (epi_normed(p, col0)) {
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) s = fmaf(v[j], v[j], s);
      ssq_acc += s;
      const float* g = p.gain + col0;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 gg = *reinterpret_cast<const float4*>(g + j);
        v[j] *= gg.x; v[j + 1] *= gg.y; v[j + 2] *= gg.z; v[j + 3] *= gg.w;
      }
    }
  }
}

// EPI_QKV on q and k columns: rotate adjacent pairs (2d, 2d+1) by the angles of the row's
// token position (table (cos, sin) [rows_per_batch, 64]).
__device__ __forceinline__ void epi_rope(const EpiParams& p, int row, int col0, float (&v)[32]) {
  const int l = row % p.rows_per_batch;
  const int d0 = (col0 % p.dim) & 127;
  const float2* rt = p.rope + (long)l * 64 + (d0 >> 1);
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float2 cs = rt[j >> 1];
    float x0 = v[j], x1 = v[j + 1];
    v[j] = x0 * cs.x - x1 * cs.y;
    v[j + 1] = x0 * cs.y + x1 * cs.x;
  }
}

// EPI_QKV: the (cos, sin) of the 16 rotary pairs of columns [col0, col0 + 32) of `row`, loaded
// ahead of their use (the table rows of a tile's 128 rows do not fit in L1, so these are L2
// reads whose latency the previous chunk's work hides).
__device__ __forceinline__ void epi_rope_load(const EpiParams& p, int row, int col0, float4 (&cs)[8]) {
  const int l = row % p.rows_per_batch;
  const float4* rt = reinterpret_cast<const float4*>(p.rope + (long)l * 64 + (((col0 % p.dim) & 127) >> 1));
#pragma unroll
  for (int k = 0; k < 8; ++k) cs[k] = rt[k];
}
// epi_rope with the pairs' (cos, sin) already in registers
__device__ __forceinline__ void epi_rope_apply(const float4 (&cs)[8], float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float x0 = v[4 * k], x1 = v[4 * k + 1];
    v[4 * k] = x0 * cs[k].x - x1 * cs[k].y;
    v[4 * k + 1] = x0 * cs[k].y + x1 * cs[k].x;
    x0 = v[4 * k + 2];
    x1 = v[4 * k + 3];
    v[4 * k + 2] = x0 * cs[k].z - x1 * cs[k].w;
    v[4 * k + 3] = x0 * cs[k].w + x1 * cs[k].z;
  }
}

// Prefetch into L1 the per-column vectors the epilogue of columns [col0, col0 + n) of
// `row` will read (bias; gate of the row's stream for EPI_RESID; gain for EPI_NORM/QKV),
// so that their loads, issued after the accumulator is ready, hit L1. One 128-byte line
// per 32 columns and vector.
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}
template <int KIND>
__device__ __forceinline__ void epi_prefetch(const EpiParams& p, int row, int col0, int n) {
  for (int c = 0; c < n; c += 32) {
    prefetch_l1(p.bias + col0 + c);
    if constexpr (KIND == EPI_RESID) {
      if (p.gate) prefetch_l1(p.gate + (long)(row / p.rows_per_batch) * p.gate_bstride + col0 + c);
    } else if constexpr (KIND == EPI_NORM || KIND == EPI_QKV) {
      if (epi_normed(p, col0 + c)) prefetch_l1(p.gain + col0 + c);
    }
  }
  if constexpr (KIND == EPI_QKV) {  // the row's rotary angles (64 (cos, sin) pairs, 4 lines)
    const float2* rt = p.rope + (long)(row % p.rows_per_batch) * 64;
    for (int c = 0; c < 64; c += 16) prefetch_l1(rt + c);
  }
}

// epi_math plus the store by the owning thread (row-major outputs, the residual update,
// or the head-major q/k/v scatter with rotary).
template <int KIND, typename OutT>
__device__ __forceinline__ void epi_chunk(const EpiParams& p, int row, int col0, float (&v)[32],
                                          float& ssq_acc) {
  epi_math<KIND, OutT>(p, row, col0, v, ssq_acc);
  if constexpr (KIND == EPI_STORE || KIND == EPI_GELU) {
    OutT* dst = reinterpret_cast<OutT*>(p.out) + (long)row * p.ldo + col0;
#pragma unroll
    for (int j = 0; j < 32; j += 8) store8(dst + j, v + j);
  } else if constexpr (KIND == EPI_RESID) {
    float* r = p.resid + (long)row * p.ldr + col0;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      float4 x = *reinterpret_cast<float4*>(r + j);
      x.x += v[j]; x.y += v[j + 1]; x.z += v[j + 2]; x.w += v[j + 3];
      *reinterpret_cast<float4*>(r + j) = x;
    }
  } else {  // EPI_NORM, EPI_QKV
    const bool normed = epi_normed(p, col0);
    if constexpr (KIND == EPI_NORM) {
      OutT* dst = reinterpret_cast<OutT*>(p.out) + (long)row * p.ldo + col0;
#pragma unroll
      for (int j = 0; j < 32; j += 8) store8(dst + j, v + j);
    } else {
      const int l = row % p.rows_per_batch;
      const int bidx = row / p.rows_per_batch;
      const int sec = col0 / p.dim;
      const int cin = col0 - sec * p.dim;
      const int head = cin >> 7;
      const int d0 = cin & 127;
      if (normed) epi_rope(p, row, col0, v);
      const int heads = p.dim >> 7;
      OutT* dst = reinterpret_cast<OutT*>(p.out) + (long)sec * p.sec_stride +
                  (((long)bidx * heads + head) * p.rows_per_batch + l) * 128 + d0;
      if (std::is_same<OutT, bf16>::value && sec == 2) {  // v in fp16 (see EPI_QKV above)
#pragma unroll
        for (int j = 0; j < 32; j += 8) store8(reinterpret_cast<__half*>(dst) + j, v + j);
      } else {
#pragma unroll
        for (int j = 0; j < 32; j += 8) store8(dst + j, v + j);
      }
    }
  }
}

// EPI_RESID with the row's residual already in registers (xr: 8 float4 = these 32 columns):
// x += gate * (acc + bias), stored back.
__device__ __forceinline__ void epi_resid_chunk_pref(const EpiParams& p, int row, int col0, float (&v)[32],
                                                     float4* xr) {
  const float* b = p.bias + col0;
  float* r = p.resid + (long)row * p.ldr + col0;
  const float* g = p.gate ? p.gate + (long)(row / p.rows_per_batch) * p.gate_bstride + col0 : nullptr;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 bb = *reinterpret_cast<const float4*>(b + j);
    float4 a = make_float4(v[j] + bb.x, v[j + 1] + bb.y, v[j + 2] + bb.z, v[j + 3] + bb.w);
    if (g) {
      const float4 gg = *reinterpret_cast<const float4*>(g + j);
      a.x *= gg.x; a.y *= gg.y; a.z *= gg.z; a.w *= gg.w;
    }
    float4 x = xr[j >> 2];
    x.x += a.x; x.y += a.y; x.z += a.z; x.w += a.w;
    *reinterpret_cast<float4*>(r + j) = x;
  }
}

// Row `r` (0..31) of a 32-row staging box for a TMA store: 32 values, fp32 rows of 128 bytes
// in the 128-byte swizzle or bf16 rows of 64 bytes in the 64-byte swizzle (16-byte chunk
// index XOR address bits 7-9 resp. 7-8), so the 32 lanes' chunks spread over all banks.
// `box` is aligned to 1024 bytes.
__device__ __forceinline__ void stage_row(uint8_t* box, int r, const float (&v)[32], float*) {
  uint8_t* row = box + r * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(row + ((j ^ (r & 7)) << 4)) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}
__device__ __forceinline__ void stage_row(uint8_t* box, int r, const float (&v)[32], bf16*) {
  uint8_t* row = box + r * 64;
#pragma unroll
  for (int j = 0; j < 4; ++j) store8(reinterpret_cast<bf16*>(row + ((j ^ ((r >> 1) & 3)) << 4)), v + 8 * j);
}
__device__ __forceinline__ void stage_row(uint8_t* box, int r, const float (&v)[32], __half*) {
  uint8_t* row = box + r * 64;
#pragma unroll
  for (int j = 0; j < 4; ++j) store8(reinterpret_cast<__half*>(row + ((j ^ ((r >> 1) & 3)) << 4)), v + 8 * j);
}

template <int KIND>
__device__ __forceinline__ void epi_group_end(const EpiParams& p, int row, int gcol0, float ssq_acc) {
  if constexpr (KIND == EPI_NORM || KIND == EPI_QKV) {
    if (epi_normed(p, gcol0)) p.ssq[(long)row * p.ssq_ld + (gcol0 >> 7)] = ssq_acc;
  }
}

}  // namespace fh
