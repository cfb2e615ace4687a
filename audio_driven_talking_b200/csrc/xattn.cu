// xattn.cu - per-frame audio cross-attention on the tensor cores (bf16, sm_100a).
//
// A token of latent frame f attends to that frame's A = 32 audio tokens only
// (gizai:flashhead, opening paragraph: 5 latent frames of 32 audio tokens; reading R5):
//   O_n = sum_a softmax_a(r_n r_a (q_n . k_a) / sqrt(128)) v_a
// per (stream, frame, head), with q the gain-scaled cross-attention query and r the
// token's full-width RMS factor from the per-head sums of squares (reading R4), exactly
// as in the self-attention kernel.
//
// xattn_tc_kernel: one CTA per 128 queries of one (stream, frame, head), 192 threads.
//   warp 0     TMA: the Q tile (3D map [frames][HW][D], rows past the frame read as
//              zero) and the frame's K and V (32 rows each); its lanes compute the 32
//              keys' RMS factors.
//   warp 1     allocates TMEM; one thread issues S = Q K^T (M=128, N=32, fp32 in TMEM)
//              and, once P is in TMEM, O = P V (M=128, N=128; P as the A operand from
//              TMEM, V read MN-major from its [key][d] layout).
//   warps 2-5  one query row per thread: the 32 scores, softmax in base 2, P split into
//              two bf16 parts P = P_hi + P_lo packed into the TMEM columns of S (so P V
//              carries P to about 16 bits for one more 128x128x32 MMA), then O / l
//              staged as bf16 in the Q tile's shared memory (free once S is computed) and
//              written by TMA stores (3D map: rows past the frame are clipped).
#include "common.cuh"
#include "kernels.h"

namespace fh {

namespace {

constexpr int XT_BQ = 128;
constexpr int XT_A = 32;
constexpr int XT_THREADS = 192;
constexpr uint32_t XT_PANEL_Q = XT_BQ * 128;  // [128 rows x 64 bf16], 128-byte rows
constexpr uint32_t XT_PANEL_KV = XT_A * 128;  // [32 rows x 64 bf16]
constexpr uint32_t XT_OFF_Q = 0;
constexpr uint32_t XT_OFF_K = XT_OFF_Q + 2 * XT_PANEL_Q;
constexpr uint32_t XT_OFF_V = XT_OFF_K + 2 * XT_PANEL_KV;
constexpr uint32_t XT_OFF_RK = XT_OFF_V + 2 * XT_PANEL_KV;
constexpr uint32_t XT_OFF_BAR = XT_OFF_RK + XT_A * 4;
constexpr uint32_t XT_SMEM = XT_OFF_BAR + 128 + 1024;
constexpr uint32_t XT_TMEM_COLS = 256;  // S in columns 0-31, O in 128-255

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(XT_THREADS, 1)
    xattn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                    const __grid_constant__ CUtensorMap tmO, const float* __restrict__ ssq_q,
                    const float* __restrict__ ssq_k, int ssq_k_ld, int ssq_k_off, int koff, int voff, int heads,
                    int HW, int F, int nqt, float eps, float scale_log2, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + XT_OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;
  uint64_t* rk_full = bars + 2;
  uint64_t* s_full = bars + 3;
  uint64_t* p_full = bars + 4;
  uint64_t* o_full = bars + 5;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* rks = reinterpret_cast<float*>(smem + XT_OFF_RK);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int f = blockIdx.x / nqt, qt = blockIdx.x % nqt;
  const int h = blockIdx.y, b = blockIdx.z;
  const int D = heads * 128;
  const float inv_d = 1.f / (float)D;
  const int frame = b * F + f;            // index into the [frames][HW] views
  const long kv_row0 = (long)frame * XT_A;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(kv_full, 1);
    mbar_init(rk_full, XT_A);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmKV);
    prefetch_tmap(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, XT_TMEM_COLS);
    tmem_relinquish();
  }
  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();  // q, its sums of squares, and the cross keys/values come from earlier kernels

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(q_full, 2 * XT_PANEL_Q);
      tma_load_3d(&tmQ, q_full, smem + XT_OFF_Q, h * 128, qt * XT_BQ, frame);
      tma_load_3d(&tmQ, q_full, smem + XT_OFF_Q + XT_PANEL_Q, h * 128 + 64, qt * XT_BQ, frame);
      mbar_expect_tx(kv_full, 4 * XT_PANEL_KV);
      tma_load_2d(&tmKV, kv_full, smem + XT_OFF_K, koff + h * 128, (int)kv_row0);
      tma_load_2d(&tmKV, kv_full, smem + XT_OFF_K + XT_PANEL_KV, koff + h * 128 + 64, (int)kv_row0);
      tma_load_2d(&tmKV, kv_full, smem + XT_OFF_V, voff + h * 128, (int)kv_row0);
      tma_load_2d(&tmKV, kv_full, smem + XT_OFF_V + XT_PANEL_KV, voff + h * 128 + 64, (int)kv_row0);
    }
    // key `lane`'s RMS factor over the full width (all heads' partial sums)
    rks[lane] = rsqrtf(sum_heads(ssq_k + (kv_row0 + lane) * ssq_k_ld + ssq_k_off, heads) * inv_d + eps);
    mbar_arrive(rk_full);
    if (lane == 0) {
      // the CTA's shared memory must outlive the copies: wait for them whatever happened
      drain_wait(q_full, 0);
      drain_wait(kv_full, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(smem + XT_OFF_Q);
      const uint32_t k_addr = smem_u32(smem + XT_OFF_K);
      const uint32_t v_addr = smem_u32(smem + XT_OFF_V);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN) &&
                mbar_wait(kv_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      if (ok) {
        tc_fence_after();
        const uint32_t id_s = idesc_bf16_f32(XT_BQ, XT_A, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 128 dims in 8 steps of 16 (two 64-wide panels)
          const uint32_t qo = (kk >> 2) * XT_PANEL_Q + (kk & 3) * 32;
          const uint32_t ko = (kk >> 2) * XT_PANEL_KV + (kk & 3) * 32;
          tc_mma_f16(tmem, sdesc_kmajor_sw128(q_addr + qo), sdesc_kmajor_sw128(k_addr + ko), id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        ok = mbar_wait(p_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      }
      if (ok) {
        tc_fence_after();
        const uint32_t id_o = idesc_bf16_f32(XT_BQ, 128, true);
        // 32 keys in 2 steps of 16, P packed 2 per column: P_hi in columns 0-15, P_lo in 16-31
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_f16_ts(tmem + 128, tmem + kk * 8, sdesc_mnmajor_sw128(v_addr + (kk & 1) * 16 * 128, XT_PANEL_KV),
                        id_o, kk > 0 ? 1u : 0u);
        tc_commit(o_full);
        // the commit's arrival must land before the CTA can leave
        mbar_wait(o_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;      // row of the tile = TMEM lane
    const int n = qt * XT_BQ + r;           // query index within the frame
    const bool valid = n < HW;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float rq = 1.f;
    if (valid) {
      rq = rsqrtf(sum_heads(ssq_q + ((long)frame * HW + n) * heads, heads) * inv_d + eps);
    }
    const float qscale = rq * scale_log2;
    bool ok = mbar_wait(rk_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
    ok = ok && mbar_wait(s_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      float sc[32];
      tmem_ld32(tmem + lane_off, sc);
      tc_wait_ld();
      float m8[8];
#pragma unroll
      for (int a = 0; a < 32; ++a) sc[a] *= rks[a] * qscale;
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = fmaxf(fmaxf(sc[u], sc[u + 8]), fmaxf(sc[u + 16], sc[u + 24]));
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[16], pl[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float p0 = ex2f(sc[2 * u] - mx), p1 = ex2f(sc[2 * u + 1] - mx);
        l4[u & 3] += p0 + p1;
        const __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
        const float2 hf = __bfloat1622float2(hp);
        const __nv_bfloat162 lp = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
        pk[u] = *reinterpret_cast<const uint32_t*>(&hp);
        pl[u] = *reinterpret_cast<const uint32_t*>(&lp);
      }
      const float inv_l = 1.f / ((l4[0] + l4[1]) + (l4[2] + l4[3]));
      tmem_st16(tmem + lane_off, pk);       // keys 2u, 2u+1 -> column u (S columns already read)
      tmem_st16(tmem + lane_off + 16, pl);  // the remainders -> column 16 + u
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      ok = mbar_wait(o_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        // O / l as bf16 into the Q tile's shared memory (S is done, so Q is no longer
        // read), in the TMA layout: two 64-wide panels of 128-byte rows, 128-byte swizzle
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_off + 128 + c, o);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= inv_l;
          uint8_t* row = smem + XT_OFF_Q + (c >> 6) * XT_PANEL_Q + r * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int chunk = ((c & 63) >> 3) + j;  // 16-byte chunk of the 128-byte row
            store8(reinterpret_cast<bf16*>(row + ((chunk ^ (r & 7)) << 4)), o + 8 * j);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        // this warp's 32 rows of both panels; rows past the frame are clipped by the map
        const int n0 = qt * XT_BQ + quarter * 32;
        if (lane == 0 && n0 < HW) {
          tma_store_3d(&tmO, smem + XT_OFF_Q + quarter * 32 * 128, h * 128, n0, frame);
          tma_store_3d(&tmO, smem + XT_OFF_Q + XT_PANEL_Q + quarter * 32 * 128, h * 128 + 64, n0, frame);
          bulk_commit();
          bulk_wait_all();
        }
        __syncwarp();
      }
    }
  }

  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, XT_TMEM_COLS);
  }
}

}  // namespace

cudaError_t xattn_tc_prepare() {
  return cudaFuncSetAttribute(xattn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)XT_SMEM);
}

cudaError_t xattn_tc(const CUtensorMap& q, const CUtensorMap& kv, const CUtensorMap& o, const float* ssq_q,
                     const float* ssq_k, int ssq_k_ld, int ssq_k_off, int koff, int voff, int batch, int heads, int L,
                     int F, int A, float eps, unsigned* err, cudaStream_t st) {
  if (A != XT_A || F < 1 || L % F != 0 || koff % 64 != 0 || voff % 64 != 0) return cudaErrorInvalidValue;
  const int HW = L / F;
  const int nqt = (HW + XT_BQ - 1) / XT_BQ;
  const float scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  dim3 grid(F * nqt, heads, batch);
  return launch_pdl(xattn_tc_kernel, grid, dim3(XT_THREADS), XT_SMEM, st, q, kv, o, ssq_q, ssq_k, ssq_k_ld,
                    ssq_k_off, koff, voff, heads, HW, F, nqt, eps, scale_log2, err);
}

}  // namespace fh
