// attention.cu - non-causal self-attention over all L tokens of a stream.
//
// O_i = sum_j softmax_j(r_i r_j (q_i . k_j) / sqrt(128)) v_j per (stream, head),
// with q, k the rotated, gain-scaled but not yet RMS-normalised projections and
// r the per-token full-width RMS factor (sum over heads of the partial sums of
// squares written by the QKV epilogue): reading R4 of the Wan-style block, whose
// self-attention the gizai:flashhead page (opening paragraph) describes as running
// over the whole latent with rotary over frame, row and column.
//
// attn_tc_kernel (bf16, sm_100a): one CTA per 128-query tile of one (stream, head).
//   warp 0     TMA: the Q tile once, then K and V tiles (128 keys) double-buffered.
//   warp 1     one thread issues tcgen05.mma: S_j = Q K_j^T into TMEM (double
//              buffered), then O_j = P_j V_j into TMEM (double buffered) with P_j
//              read from TMEM as the A operand and V read MN-major straight from
//              its [key][d] layout.
//   warps 2-9  two threads per query row (one per warpgroup, 64 keys and 64 output
//              dims each): S_j from TMEM, online softmax in base 2, P_j written as
//              packed bf16 back into TMEM over the S_j columns it has consumed (so P
//              is double-buffered with S at no cost), and O_j folded into a register
//              accumulator that carries the running max correction.
//   The MMA thread issues S_{j+1} before P_j V_j so the tensor core works while the
//   softmax warps exponentiate.
// attn_simt_kernel (fp32 or bf16 inputs, CUDA cores): one query row per thread, a
// plain online-softmax loop; used by the fp32 configuration.
#include "common.cuh"
#include "kernels.h"

namespace fh {

namespace {

constexpr int AT_BQ = 128;
constexpr int AT_BK = 128;
constexpr int AT_SOFTMAX_THREADS = 256;           // warps 2-9
constexpr int AT_THREADS = 64 + AT_SOFTMAX_THREADS;
constexpr uint32_t PANEL = 128 * 128;           // bytes of one [128 rows x 64 bf16] panel
constexpr uint32_t TILE = 2 * PANEL;            // [128 rows x 128 bf16]
// shared memory map (offsets from the 1024-aligned base)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE;        // 2 buffers
constexpr uint32_t OFF_V = OFF_K + 2 * TILE;    // 2 buffers
constexpr uint32_t OFF_MX = OFF_V + 2 * TILE;   // float [2][2][128] partial row maxima
constexpr uint32_t OFF_LS = OFF_MX + 4 * 128 * 4;  // float [2][128] partial row sums
constexpr uint32_t OFF_BAR = OFF_LS + 2 * 128 * 4;
constexpr uint32_t OFF_RKALL = OFF_BAR + 256;   // float rk[round_up(L, 128)]: every key's RMS factor
constexpr int AT_MAX_L = 8192;
constexpr uint32_t AT_SMEM = OFF_RKALL + AT_MAX_L * 4 + 1024;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float row_rms(const float* ssq, int ssq_ld, long row, int off, int heads, float inv_d,
                                         float eps) {
  const float* p = ssq + row * ssq_ld + off;
  float s = 0.f;
  for (int h = 0; h < heads; ++h) s += p[h];
  return rsqrtf(s * inv_d + eps);
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const float* __restrict__ ssq, int ssq_ld, int heads,
                   int L, float eps, float scale_log2, bf16* __restrict__ out, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* k_empty = bars + 5;   // [2] K buffer free (S MMA done)
  uint64_t* v_empty = bars + 9;   // [2] V buffer free (P.V MMA done); also orders S-buffer reuse
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* o_full = bars + 11;   // [2]
  uint64_t* o_free = bars + 13;   // [2]
  uint64_t* p_full = bars + 15;
  uint64_t* rk_full = bars + 17;  // every key's RMS factor staged
  uint64_t* mx_bar = bars + 21;   // [2]
  uint64_t* l_bar = bars + 23;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int D = heads * 128;
  const int nkv = (L + AT_BK - 1) / AT_BK;
  const int bh_row0 = (b * heads + h) * L;  // first row of this (stream, head) in the 2D views

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], AT_SOFTMAX_THREADS);
    }
    mbar_init(p_full, AT_SOFTMAX_THREADS);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&mx_bar[i], AT_SOFTMAX_THREADS);
    }
    mbar_init(l_bar, AT_SOFTMAX_THREADS);
    mbar_init(rk_full, AT_SOFTMAX_THREADS);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();  // q, k, v and the sums of squares come from the preceding QKV projection

  if (warp == 0) {
    if (lane == 0) {
      int kiss = 0, viss = 0;  // K and V tiles issued
      mbar_expect_tx(q_full, TILE);
      tma_load_2d(&tmQ, q_full, smem + OFF_Q, 0, bh_row0 + qt * AT_BQ);
      tma_load_2d(&tmQ, q_full, smem + OFF_Q + PANEL, 64, bh_row0 + qt * AT_BQ);
      // order K_0, K_1, V_0, K_2, V_1, ...: the MMA issues S_{j+1} before P_j V_j
      auto load_k = [&](int j) -> bool {
        const int bf = j & 1;
        if (!mbar_wait(&k_empty[bf], ((j >> 1) & 1) ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) return false;
        const int r0 = bh_row0 + j * AT_BK;
        mbar_expect_tx(&k_full[bf], TILE);
        tma_load_2d(&tmK, &k_full[bf], smem + OFF_K + bf * TILE, 0, r0);
        tma_load_2d(&tmK, &k_full[bf], smem + OFF_K + bf * TILE + PANEL, 64, r0);
        kiss = j + 1;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int bf = j & 1;
        if (!mbar_wait(&v_empty[bf], ((j >> 1) & 1) ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) return false;
        const int r0 = bh_row0 + j * AT_BK;
        mbar_expect_tx(&v_full[bf], TILE);
        tma_load_2d(&tmV, &v_full[bf], smem + OFF_V + bf * TILE, 0, r0);
        tma_load_2d(&tmV, &v_full[bf], smem + OFF_V + bf * TILE + PANEL, 64, r0);
        viss = j + 1;
        return true;
      };
      if (load_k(0)) {
        for (int j = 0; j < nkv; ++j) {
          if (j + 1 < nkv && !load_k(j + 1)) break;
          if (!load_v(j)) break;
        }
      }
      // tail: the MMA's release commits for the last K and V tiles have landed
      for (int j = kiss - 2 < 0 ? 0 : kiss - 2; !*abort_flag && j < kiss; ++j)
        mbar_wait(&k_empty[j & 1], (j >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      for (int j = viss - 2 < 0 ? 0 : viss - 2; !*abort_flag && j < viss; ++j)
        mbar_wait(&v_empty[j & 1], (j >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      if (*abort_flag) {
        uint64_t t0 = globaltimer();
        while (!mbar_try_wait(q_full, 0) && globaltimer() - t0 < FH_WAIT_LIMIT_NS) {
        }
        for (int j = kiss - 2 < 0 ? 0 : kiss - 2; j < kiss; ++j) {
          t0 = globaltimer();
          while (!mbar_try_wait(&k_full[j & 1], (j >> 1) & 1) && globaltimer() - t0 < FH_WAIT_LIMIT_NS) {
          }
        }
        for (int j = viss - 2 < 0 ? 0 : viss - 2; j < viss; ++j) {
          t0 = globaltimer();
          while (!mbar_try_wait(&v_full[j & 1], (j >> 1) & 1) && globaltimer() - t0 < FH_WAIT_LIMIT_NS) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, false);
      const uint32_t id_o = idesc_bf16_f32(128, 128, true);
      const uint32_t q_addr = smem_u32(smem + OFF_Q);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      tc_fence_after();
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {  // S_j = Q K_j^T
          const int bf = j & 1;
          const uint32_t par = (j >> 1) & 1;
          if (!mbar_wait(&k_full[bf], par, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) break;
          // S_j overwrites the TMEM buffer that held S_{j-2} and P_{j-2}: wait for P_{j-2} V_{j-2}
          if (j >= 2 && !mbar_wait(&v_empty[bf], par ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + OFF_K + bf * TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
            tc_mma_f16(tmem + bf * 128, sdesc_kmajor_sw128(q_addr + off), sdesc_kmajor_sw128(k_addr + off), id_s,
                       kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[bf]);
          tc_commit(&k_empty[bf]);
        }
        if (j >= 1) {  // O_i = P_i V_i for i = j - 1
          const int i = j - 1;
          const int bf = i & 1;
          const uint32_t par = (i >> 1) & 1;
          if (!mbar_wait(p_full, i & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) break;
          if (!mbar_wait(&v_full[bf], par, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) break;
          if (!mbar_wait(&o_free[bf], par ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(smem + OFF_V + bf * TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // keys 16kk..16kk+15 of P_i: packed in columns 64*(kk/4) + 8*(kk%4) of S_i's buffer
            const uint32_t a_tmem = tmem + bf * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
            const uint32_t b_off = kk * 16 * 128;                      // 16 key rows of V
            tc_mma_f16_ts(tmem + 256 + bf * 128, a_tmem, sdesc_mnmajor_sw128(v_addr + b_off, PANEL), id_o,
                          kk > 0 ? 1u : 0u);
          }
          tc_commit(&o_full[bf]);
          tc_commit(&v_empty[bf]);
        }
      }
    }
  } else {
    // softmax / correction / output, warps 2-9: each query row belongs to one thread of each
    // warpgroup; half 0 (warps 2-5) takes keys and output dims 0-63, half 1 (warps 6-9)
    // takes 64-127. Only the partial row maxima cross between the halves (per tile, through
    // shared memory and an mbarrier); the partial row sums are combined once at the end.
    const int quarter = warp & 3;                      // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;
    const int t = threadIdx.x - 64;                    // 0..255 among the softmax threads
    const int rl = quarter * 32 + lane;                // row within the tile
    const int qi = qt * AT_BQ + rl;                    // query index within the stream
    const bool qvalid = qi < L;
    const float inv_d = 1.f / (float)D;
    const float rq = row_rms(ssq, ssq_ld, (long)b * L + (qvalid ? qi : L - 1), 0, heads, inv_d, eps);
    const float qscale = rq * scale_log2;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* mxs = reinterpret_cast<float*>(smem + OFF_MX);  // [2 tiles][2 halves][128 rows]
    float* lss = reinterpret_cast<float*>(smem + OFF_LS);  // [2 halves][128 rows]

    // every key's RMS factor, once per CTA (the keys are shared by all tiles of the row)
    float* rk_all = reinterpret_cast<float*>(smem + OFF_RKALL);
    for (int key = t; key < nkv * AT_BK; key += AT_SOFTMAX_THREADS)
      rk_all[key] = key < L ? row_rms(ssq, ssq_ld, (long)b * L + key, heads, heads, inv_d, eps) : 0.f;
    mbar_arrive(&rk_full[0]);
    float o[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) o[d] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;

    ok = mbar_wait(&rk_full[0], 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
    ok = __all_sync(0xffffffffu, ok);
    for (int j = 0; ok && j < nkv; ++j) {
      const float* rk = rk_all + j * AT_BK + half * 64;
      const int bf = j & 1;
      const uint32_t par = (j >> 1) & 1;
      ok = mbar_wait(&s_full[bf], par, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_t = tmem + lane_off + bf * 128 + half * 64;
      const int kvalid = L - j * AT_BK - half * 64;  // keys of this half-tile that exist
      // this half's 64 scores of the row, one batched TMEM read kept in registers for both passes
      float sa[32], sb[32];
      tmem_ld32(s_t, sa);
      tmem_ld32(s_t + 32, sb);
      tc_wait_ld();
      // scaled scores r_k * (q.k); keys past the end of the sequence get -inf (only the last tile)
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        sa[e] *= rk[e];
        sb[e] *= rk[e + 32];
      }
      if (kvalid < 64) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if (e >= kvalid) sa[e] = -INFINITY;
          if (e + 32 >= kvalid) sb[e] = -INFINITY;
        }
      }
      // row max as a tree (independent chains)
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        m8[u] = fmaxf(fmaxf(sa[u], sa[u + 8]), fmaxf(sa[u + 16], sa[u + 24]));
        m8[u] = fmaxf(m8[u], fmaxf(fmaxf(sb[u], sb[u + 8]), fmaxf(sb[u + 16], sb[u + 24])));
      }
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      float* mxt = mxs + (j & 1) * 256;
      mxt[half * 128 + rl] = mx;
      mbar_arrive(&mx_bar[j & 1]);
      ok = mbar_wait(&mx_bar[j & 1], (j >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      mx = fmaxf(mx, mxt[(1 - half) * 128 + rl]);
      const float m_new = fmaxf(m_run, mx * qscale);
      const float alpha = ex2(m_run - m_new);
      // probabilities (ex2 of -inf is 0), four independent partial sums, packed bf16 P
      // written over the consumed S columns
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pa[16], pb2[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float p0 = ex2(fmaf(sa[2 * u], qscale, -m_new));
        const float p1 = ex2(fmaf(sa[2 * u + 1], qscale, -m_new));
        const float q0 = ex2(fmaf(sb[2 * u], qscale, -m_new));
        const float q1 = ex2(fmaf(sb[2 * u + 1], qscale, -m_new));
        rs4[u & 3] += (p0 + p1) + (q0 + q1);
        __nv_bfloat162 h0 = __floats2bfloat162_rn(p0, p1);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(q0, q1);
        pa[u] = *reinterpret_cast<uint32_t*>(&h0);
        pb2[u] = *reinterpret_cast<uint32_t*>(&h1);
      }
      const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      tmem_st16(s_t, pa);        // keys 0..31 of this half -> columns 0..15 (already read)
      tmem_st16(s_t + 16, pb2);  // keys 32..63 -> columns 16..31
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      l_run = l_run * alpha + rs;
      m_run = m_new;
      // fold this half's 64 dims of O_{j-1} (relative to the previous max), rescale to the new max
      if (j >= 1) {
        const int pb = (j - 1) & 1;
        ok = mbar_wait(&o_full[pb], ((j - 1) >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t o_t = tmem + lane_off + 256 + pb * 128 + half * 64;
        {
          float oa[32], ob[32];
          tmem_ld32(o_t, oa);
          tmem_ld32(o_t + 32, ob);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            o[e] = (o[e] + oa[e]) * alpha;
            o[e + 32] = (o[e + 32] + ob[e]) * alpha;
          }
        }
        tc_fence_before();
        mbar_arrive(&o_free[pb]);
      }
    }
    if (ok) {
      const int pb = (nkv - 1) & 1;
      ok = mbar_wait(&o_full[pb], ((nkv - 1) >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const uint32_t o_t = tmem + lane_off + 256 + pb * 128 + half * 64;
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          float v[32];
          tmem_ld32(o_t + c, v);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[c + e] += v[e];
        }
        // the row's normaliser is the sum of both halves' partial sums
        lss[half * 128 + rl] = l_run;
        mbar_arrive(l_bar);
        ok = mbar_wait(l_bar, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && qvalid) {
          const float inv_l = 1.f / (l_run + lss[(1 - half) * 128 + rl]);
          bf16* dst = out + ((long)b * L + qi) * D + h * 128 + half * 64;
#pragma unroll
          for (int d = 0; d < 64; d += 8) {
            float w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = o[d + e] * inv_l;
            store8(dst + d, w);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- SIMT version
constexpr int SA_KC = 32;  // keys staged per round

template <typename T>
__global__ void __launch_bounds__(64) attn_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                       const T* __restrict__ V, const float* __restrict__ ssq,
                                                       int ssq_ld, int heads, int L, float eps, float scale,
                                                       T* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float ks[SA_KC][128];
  __shared__ float vs[SA_KC][128];
  __shared__ float rks[SA_KC];
  const int h = blockIdx.y, b = blockIdx.z;
  const int D = heads * 128;
  const float inv_d = 1.f / (float)D;
  const int qi = blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = qi < L;
  const long base = ((long)(b * heads + h)) * L * 128;
  float q[128], o[128];
  float rq = 0.f;
  if (valid) {
    const float* p = ssq + ((long)b * L + qi) * ssq_ld;
    float s = 0.f;
    for (int i = 0; i < heads; ++i) s += p[i];
    rq = rsqrtf(s * inv_d + eps) * scale;
  }
#pragma unroll
  for (int d = 0; d < 128; ++d) {
    q[d] = valid ? to_f(Q[base + (long)qi * 128 + d]) : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < L; k0 += SA_KC) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < SA_KC * 128; idx += blockDim.x) {
      const int kj = idx / 128, d = idx % 128;
      const int key = k0 + kj;
      ks[kj][d] = key < L ? to_f(K[base + (long)key * 128 + d]) : 0.f;
      vs[kj][d] = key < L ? to_f(V[base + (long)key * 128 + d]) : 0.f;
    }
    for (int kj = threadIdx.x; kj < SA_KC; kj += blockDim.x) {
      const int key = k0 + kj;
      float r = 0.f;
      if (key < L) {
        const float* p = ssq + ((long)b * L + key) * ssq_ld + heads;
        float s = 0.f;
        for (int i = 0; i < heads; ++i) s += p[i];
        r = rsqrtf(s * inv_d + eps);
      }
      rks[kj] = r;
    }
    __syncthreads();
    const int nk = min(SA_KC, L - k0);
    for (int kj = 0; kj < nk; ++kj) {
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < 128; ++d) s = fmaf(q[d], ks[kj][d], s);
      s *= rq * rks[kj];
      const float mn = fmaxf(m, s);
      const float a = expf(m - mn);
      const float p = expf(s - mn);
      l = l * a + p;
#pragma unroll
      for (int d = 0; d < 128; ++d) o[d] = fmaf(o[d], a, p * vs[kj][d]);
      m = mn;
    }
  }
  if (valid) {
    T* dst = out + ((long)b * L + qi) * D + h * 128;
    const float inv = 1.f / l;
#pragma unroll
    for (int d = 0; d < 128; ++d) dst[d] = from_f<T>(o[d] * inv);
  }
}

}  // namespace

cudaError_t attn_tc_prepare() {
  return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AT_SMEM);
}

cudaError_t attn_tc(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const float* ssq,
                    int ssq_ld, int batch, int heads, int L, float eps, bf16* out, unsigned* err,
                    cudaStream_t st) {
  if (L > AT_MAX_L) return cudaErrorInvalidValue;
  const float scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  dim3 grid((L + AT_BQ - 1) / AT_BQ, heads, batch);
  { cudaError_t e_ = launch_pdl(attn_tc_kernel, dim3(grid), dim3(AT_THREADS), AT_SMEM, st, q, k, v, ssq, ssq_ld, heads, L, eps, scale_log2, out, err); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

template <typename T>
cudaError_t attn_simt(const T* q, const T* k, const T* v, const float* ssq, int ssq_ld, int batch, int heads, int L,
                      float eps, T* out, cudaStream_t st) {
  dim3 grid((L + 63) / 64, heads, batch);
  { cudaError_t e_ = launch_pdl(attn_simt_kernel<T>, dim3(grid), dim3(64), 0, st, q, k, v, ssq, ssq_ld, heads, L, eps, 1.f / sqrtf(128.f), out); if (e_ != cudaSuccess) return e_; }
  return cudaGetLastError();
}

template cudaError_t attn_simt<float>(const float*, const float*, const float*, const float*, int, int, int, int,
                                      float, float*, cudaStream_t);
template cudaError_t attn_simt<bf16>(const bf16*, const bf16*, const bf16*, const float*, int, int, int, int, float,
                                     bf16*, cudaStream_t);

}  // namespace fh
