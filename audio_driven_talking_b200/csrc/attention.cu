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
//   warp 1     one thread issues tcgen05.mma: S_j = Q K_j^T into TMEM (double buffered),
//              then for each key half w of tile j the product O_w += P_{j,w} V_{j,w}
//              (P read from TMEM as the A operand, V MN-major from its [key][d] layout)
//              into one of two TMEM accumulators O_0, O_1.
//   warps 2-9  two warpgroups; warpgroup w owns keys 64w..64w+63 of every tile, one
//              query row per thread, and runs its own online softmax over them (base 2,
//              its own running max and sum): the two halves are two independent
//              partial attentions over disjoint key sets, combined once at the end with
//              their maxima and sums (O = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1)).
//              P is written over the S columns it has consumed as packed fp16 (11-bit
//              significand; p <= 2^8 by the rescale rule below) and multiplied by V, which
//              the QKV epilogue stores in fp16 for this (a tensor-core product takes A and
//              B of one type): the weights carry 8 times less rounding than bf16 P, which
//              alone was the kernel's whole error, for one P.V product per key. O_w stays
//              in TMEM; it is rescaled only when a row's running max grows by more than
//              2^8 (then p <= 256 against the stale max, exact after the final division),
//              so most tiles need no correction pass and the warpgroups never wait for
//              each other inside the loop.
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
constexpr uint32_t OFF_ML = OFF_V + 2 * TILE;   // float [2 halves][2 (m, l)][128 rows]
constexpr uint32_t OFF_BAR = OFF_ML + 4 * 128 * 4;
constexpr uint32_t OFF_RKALL = OFF_BAR + 256;   // float rk[round_up(L, 128)]: every key's RMS factor
constexpr int AT_MAX_L = 8192;
constexpr uint32_t AT_SMEM = OFF_RKALL + AT_MAX_L * 4 + 1024;
constexpr float AT_RESCALE = 8.f;               // log2 growth of a row max that forces a rescale
// TMEM columns: S_0 0-127, S_1 128-255 (P over them), O_0 256-383, O_1 384-511

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float row_rms(const float* ssq, int ssq_ld, long row, int off, int heads, float inv_d,
                                         float eps) {
  return rsqrtf(sum_heads(ssq + row * ssq_ld + off, heads) * inv_d + eps);
}

// Every key's RMS factor rk[key] (0 past L) for keys [0, nkeys), by `nthreads` threads: with
// 12 heads (the model's width) each row's 12 partial sums are three 16-byte loads, and a
// thread issues the loads of its four rows before it adds any of them, so the prologue
// costs about one round trip to L2 instead of one per row and head.
__device__ __forceinline__ void key_rms_all(float* rk, const float* ssq, int ssq_ld, long row0, int heads, int L,
                                            int nkeys, float inv_d, float eps, int t, int nthreads) {
  if (heads == 12 && (ssq_ld & 3) == 0 && (reinterpret_cast<uintptr_t>(ssq) & 15) == 0) {
    for (int base = 0; base < nkeys; base += 4 * nthreads) {
      float4 v[4][3];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int key = base + u * nthreads + t;
        const float4* p = reinterpret_cast<const float4*>(ssq + (row0 + (key < L ? key : 0)) * ssq_ld + heads);
#pragma unroll
        for (int c = 0; c < 3; ++c) v[u][c] = p[c];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int key = base + u * nthreads + t;
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < 3; ++c) s += (v[u][c].x + v[u][c].y) + (v[u][c].z + v[u][c].w);
        if (key < nkeys) rk[key] = key < L ? rsqrtf(s * inv_d + eps) : 0.f;
      }
    }
  } else {
    for (int key = t; key < nkeys; key += nthreads)
      rk[key] = key < L ? row_rms(ssq, ssq_ld, row0 + key, heads, heads, inv_d, eps) : 0.f;
  }
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
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* v_empty = bars + 9;   // [2] V buffer free (both halves' P.V done); also orders S-buffer reuse
  // [2 halves][2 tiles by parity] P written. Two per half: a warpgroup no longer waits for
  // each tile's P.V, so it can publish P_{i+1} before the MMA thread has waited for P_i
  // (never P_{i+2}: S_{i+2} waits for P_i V_i), which one phase bit could not tell apart.
  uint64_t* p_full = bars + 11;
  // [2 halves][2 tiles by parity] P.V of a tile accumulated into O_w. A warpgroup waits for
  // one only to rescale O_w or at the end, so it may skip phases; per parity, the phase two
  // tiles back is always complete (S_j waits for P_{j-2} V_{j-2}) and the one two tiles
  // ahead cannot start, so each wait names one phase.
  uint64_t* pv_done = bars + 15;
  uint64_t* rk_full = bars + 19;  // the first key RMS factors staged
  uint64_t* fin_bar = bars + 20;  // both halves' (m, l) published
  uint64_t* rk_bar = bars + 21;   // [2 halves][2 tiles by parity] a later tile's key RMS factors staged
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 25);
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
      mbar_init(&p_full[2 * i], AT_SOFTMAX_THREADS / 2);
      mbar_init(&p_full[2 * i + 1], AT_SOFTMAX_THREADS / 2);
      mbar_init(&pv_done[2 * i], 1);
      mbar_init(&pv_done[2 * i + 1], 1);
    }
    mbar_init(rk_full, AT_SOFTMAX_THREADS);
    mbar_init(fin_bar, AT_SOFTMAX_THREADS);
    for (int i = 0; i < 4; ++i) mbar_init(&rk_bar[i], AT_SOFTMAX_THREADS / 2);
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
  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
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
      const uint32_t id_o = idesc_f16_f32(128, 128, true);  // fp16 P (TMEM) and V (smem)
      const uint32_t q_addr = smem_u32(smem + OFF_Q);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      tc_fence_after();
      int pv_issued = 0;  // tiles whose P.V was issued (for the tail)
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
        if (j >= 1) {  // O_w += P_{i,w} V_{i,w} for i = j - 1, each half as soon as its P is written
          const int i = j - 1;
          const int bf = i & 1;
          const uint32_t par = (i >> 1) & 1;
          if (!mbar_wait(&v_full[bf], par, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) break;
          const uint32_t v_addr = smem_u32(smem + OFF_V + bf * TILE);
          bool hok = true;
          for (int w = 0; w < 2; ++w) {
            if (!mbar_wait(&p_full[2 * w + bf], par, abort_flag, err, ERRBIT_TIMEOUT_ATTN)) {
              hok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // keys 64w + 16kk .. +15: their P (fp16 pairs) in columns 64w + 8kk .. +7
              const uint32_t a_tmem = tmem + bf * 128 + w * 64 + kk * 8;
              const uint32_t b_off = (w * 64 + kk * 16) * 128;  // 16 key rows of V
              tc_mma_f16_ts(tmem + 256 + w * 128, a_tmem, sdesc_mnmajor_sw128(v_addr + b_off, PANEL), id_o,
                            (i > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&pv_done[2 * w + bf]);
          }
          if (!hok) break;
          tc_commit(&v_empty[bf]);
          pv_issued = j;
        }
      }
      // tail: the last P.V commits have landed before the CTA can leave
      if (pv_issued > 0) {
        const int last = pv_issued - 1;
        mbar_wait(&pv_done[0 + (last & 1)], (last >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
        mbar_wait(&pv_done[2 + (last & 1)], (last >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      }
    }
  } else {
    // softmax, warps 2-9: warpgroup `half` owns keys 64*half .. 64*half + 63 of every tile
    const int quarter = warp & 3;                      // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;
    const int t = threadIdx.x - 64;                    // 0..255 among the softmax threads
    const int rl = quarter * 32 + lane;                // row within the tile
    const int qi = qt * AT_BQ + rl;                    // query index within the stream
    const bool qvalid = qi < L;
    const float inv_d = 1.f / (float)D;
    // the query's own partial sums, loaded now and added after the keys' loads are issued, so
    // that the prologue waits for one round trip to L2, not two
    const float* qrow = ssq + ((long)b * L + (qvalid ? qi : L - 1)) * ssq_ld;
    const bool qvec = heads == 12 && (reinterpret_cast<uintptr_t>(qrow) & 15) == 0;
    float4 qv[3];
    if (qvec) {
#pragma unroll
      for (int c = 0; c < 3; ++c) qv[c] = reinterpret_cast<const float4*>(qrow)[c];
    }
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t o_t = tmem + lane_off + 256 + half * 128;  // this half's O accumulator row
    float* mls = reinterpret_cast<float*>(smem + OFF_ML);    // [2 halves][m, l][128 rows]

    // The keys' RMS factors, staged in shared memory (every row of the tile uses them). With
    // 12 heads only the first two tiles' are computed before the loop; each later tile's are
    // loaded by its half's threads two tiles ahead (one key per thread, three 16-byte loads
    // issued at the start of a tile and summed at its end, so their L2 latency hides behind
    // the exponentials). Otherwise every key's, before the loop.
    float* rk_all = reinterpret_cast<float*>(smem + OFF_RKALL);
    const bool lazy = heads == 12 && (ssq_ld & 3) == 0 && (reinterpret_cast<uintptr_t>(ssq) & 15) == 0;
    key_rms_all(rk_all, ssq, ssq_ld, (long)b * L, heads, L, (lazy && nkv > 2 ? 2 : nkv) * AT_BK, inv_d, eps, t,
                AT_SOFTMAX_THREADS);
    mbar_arrive(rk_full);
    float qs = 0.f;  // head by head in order, as sum_heads adds them
    if (qvec) {
#pragma unroll
      for (int c = 0; c < 3; ++c) qs = (((qs + qv[c].x) + qv[c].y) + qv[c].z) + qv[c].w;
    } else {
      qs = sum_heads(qrow, heads);
    }
    const float qscale = rsqrtf(qs * inv_d + eps) * scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = mbar_wait(rk_full, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
    ok = __all_sync(0xffffffffu, ok);
    for (int j = 0; ok && j < nkv; ++j) {
      const float* rk = rk_all + j * AT_BK + half * 64;
      const int bf = j & 1;
      ok = mbar_wait(&s_full[bf], (j >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      // tile j + 2's key factors (this half's 64 keys, one per thread of its first 64)
      float4 kp[3];
      const int kkey = (lazy && j + 2 < nkv && (t & 127) < 64) ? (j + 2) * AT_BK + half * 64 + (t & 127) : -1;
      if (kkey >= 0) {
        const float4* p = reinterpret_cast<const float4*>(ssq + ((long)b * L + (kkey < L ? kkey : 0)) * ssq_ld + heads);
#pragma unroll
        for (int c = 0; c < 3; ++c) kp[c] = p[c];
      }
      // this tile's key factors, staged two tiles ago
      if (ok && lazy && j >= 2)
        ok = mbar_wait(&rk_bar[2 * half + (j & 1)], ((j - 2) >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_t = tmem + lane_off + bf * 128 + half * 64;
      const int kvalid = L - j * AT_BK - half * 64;  // keys of this half-tile that exist
      float sa[32], sb[32];
      tmem_ld32(s_t, sa);
      tmem_ld32(s_t + 32, sb);
      tc_wait_ld();
      // r_k (q.k) per key; the row factor r_q / sqrt(128) * log2(e) (qscale > 0) is applied
      // to the max and inside the exponent's FMA; missing keys get -inf
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
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        m8[u] = fmaxf(fmaxf(sa[u], sa[u + 8]), fmaxf(sa[u + 16], sa[u + 24]));
        m8[u] = fmaxf(m8[u], fmaxf(fmaxf(sb[u], sb[u + 8]), fmaxf(sb[u + 16], sb[u + 24])));
      }
      const float mt = qscale * fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                      fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      // the running max moves only when it must (first tile, or growth beyond 2^8); the
      // warp rescales together so its TMEM accesses stay collective
      const bool grow = __any_sync(0xffffffffu, mt > m_run + AT_RESCALE);
      if (grow) {
        const float m_new = fmaxf(m_run, mt);
        if (j > 0) {
          // 0 for a row that had only missing keys so far (its O and l are 0); 1 if still none
          const float alpha = m_new == -INFINITY ? 1.f : ex2(m_run - m_new);
          l_run *= alpha;
          // O_w holds P V up to tile j-1: wait for that product, then scale it in place
          ok = mbar_wait(&pv_done[2 * half + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort_flag, err,
                         ERRBIT_TIMEOUT_ATTN);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            float o[32];
            tmem_ld32(o_t + c, o);
            tc_wait_ld();
            uint32_t lo[16], hi[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              lo[e] = __float_as_uint(o[e] * alpha);
              hi[e] = __float_as_uint(o[e + 16] * alpha);
            }
            tmem_st16(o_t + c, lo);
            tmem_st16(o_t + c + 16, hi);
          }
          tc_wait_st();
        }
        m_run = m_new;
      }
      // probabilities against the (possibly stale) running max, packed as fp16 pairs; a row
      // whose keys so far are all missing uses 0 as its reference (ex2(-inf) = 0)
      const float mref = m_run == -INFINITY ? 0.f : m_run;
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pa[16], pb2[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float p0 = ex2(fmaf(sa[2 * u], qscale, -mref));
        const float p1 = ex2(fmaf(sa[2 * u + 1], qscale, -mref));
        const float q0 = ex2(fmaf(sb[2 * u], qscale, -mref));
        const float q1 = ex2(fmaf(sb[2 * u + 1], qscale, -mref));
        rs4[u & 3] += (p0 + p1) + (q0 + q1);
        __half2 h0 = __floats2half2_rn(p0, p1);
        __half2 h1 = __floats2half2_rn(q0, q1);
        pa[u] = *reinterpret_cast<uint32_t*>(&h0);
        pb2[u] = *reinterpret_cast<uint32_t*>(&h1);
      }
      l_run += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      tmem_st16(s_t, pa);        // P of keys 0..31 of this half -> columns 0..15 (already read)
      tmem_st16(s_t + 16, pb2);  // P of keys 32..63 -> columns 16..31
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[2 * half + bf]);
      if (lazy && j + 2 < nkv) {
        if (kkey >= 0) {
          float s2 = 0.f;
#pragma unroll
          for (int c = 0; c < 3; ++c) s2 += (kp[c].x + kp[c].y) + (kp[c].z + kp[c].w);
          rk_all[kkey] = kkey < L ? rsqrtf(s2 * inv_d + eps) : 0.f;
        }
        mbar_arrive(&rk_bar[2 * half + (j & 1)]);
      }
    }
    if (ok) {
      // this half's last product, then both halves' (m, l) for the combination
      ok = mbar_wait(&pv_done[2 * half + ((nkv - 1) & 1)], ((nkv - 1) >> 1) & 1, abort_flag, err,
                     ERRBIT_TIMEOUT_ATTN);
      mls[(half * 2 + 0) * 128 + rl] = m_run;
      mls[(half * 2 + 1) * 128 + rl] = l_run;
      mbar_arrive(fin_bar);
      ok = ok && mbar_wait(fin_bar, 0, abort_flag, err, ERRBIT_TIMEOUT_ATTN);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const float m0 = mls[0 * 128 + rl], l0 = mls[1 * 128 + rl];
        const float m1 = mls[2 * 128 + rl], l1 = mls[3 * 128 + rl];
        const float m = fmaxf(m0, m1);
        const float a0 = ex2(m0 - m), a1 = ex2(m1 - m);  // m1 = -inf (no key in half 1): a1 = 0
        const float inv_l = 1.f / (a0 * l0 + a1 * l1);
        const float c0 = a0 * inv_l, c1 = a1 * inv_l;
        // this warpgroup writes output dims 64*half .. +63 from both accumulators
        const uint32_t o0 = tmem + lane_off + 256 + half * 64, o1 = tmem + lane_off + 384 + half * 64;
        bf16* dst = out + ((long)b * L + qi) * D + h * 128 + half * 64;
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          float x0[32], x1[32];
          tmem_ld32(o0 + c, x0);
          tmem_ld32(o1 + c, x1);
          tc_wait_ld();
          if (qvalid) {
#pragma unroll
            for (int d = 0; d < 32; d += 8) {
              float w8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) w8[e] = x0[d + e] * c0 + x1[d + e] * c1;
              store8(dst + c + d, w8);
            }
          }
        }
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
