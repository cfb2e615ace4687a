// gemm_tc.cu - bf16 tensor-core GEMM with fused epilogues for sm_100a.
//
// out[M, N] = epilogue(A[M, K] * W[N, K]^T): A is an activation (bf16, row-major,
// K contiguous), W a Linear weight in nn.Linear layout [out, in] (bf16, K
// contiguous). This is every dense contraction of the DiT: patch embed, QKV,
// O-proj, cross-Q, cross-KV, cross-O, FFN1, FFN2 and the head.
//
// Three kernels, all warp-specialised:
//   warp 0     TMA producer: one thread streams 64-deep A and W tiles with the
//              128-byte swizzle into a STAGES-deep shared-memory ring (per-CTA
//              loads, no cluster multicast), the first stages' W before the
//              programmatic-launch dependency wait (W is never written).
//   warp 1     allocates TMEM and, from one thread, issues tcgen05.mma (fp32
//              accumulate in TMEM); each stage is released by tcgen05.commit to
//              its "empty" mbarrier and each finished tile by a commit to its
//              accumulator's "full" barrier.
//   warps 2-   epilogue: tcgen05.ld of 32 columns at a time (warp w reads TMEM
//              lanes 32*(w%4)..+31 = its 32 output rows) and the fused epilogue.
// gemm_tc_kernel    192 threads, one CTA per SM, persistent over 128 x BN tiles
//                   (cta_group::1), two accumulators so the epilogue of tile i
//                   overlaps the MMAs of tile i+1, direct 16-byte stores.
// gemm_tc2_kernel   320 threads, a CTA pair (cluster of 2) per 256 x BN tile
//                   (cta_group::2), persistent over whole tiles (one cluster per
//                   resident CTA pair), two accumulators, eight epilogue warps that
//                   stage 32 x 32 boxes in shared memory and store them by TMA (the
//                   residual as a TMA fp32 reduce-add into x).
// gemm_tc2s_kernel  320 threads, split-K over the two CTA pairs of a cluster of four
//                   for GEMMs with few 256 x 256 tiles, reduce-scatter of the fp32
//                   partial sums through distributed shared memory.
// Every wait is bounded (FH_WAIT_LIMIT_NS); on expiry the CTA latches an error
// bit, lets the producer's in-flight copies land, frees TMEM and exits.
#include <cstdio>
#include <type_traits>

#include "epilogue.cuh"
#include "kernels.h"

namespace fh {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct TcShape {
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

template <int BN, int KIND, typename OutT>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                   int N, int K, EpiParams ep, unsigned* err) {
  using S = TcShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::STAGES * S::STAGE_BYTES);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = N / BN;
  const int ntiles = num_m * num_n;
  const int nk = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 2 * BN);
    tmem_relinquish();
  }
  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // The weights W are never written by any kernel: start streaming the first stages'
      // W tiles before waiting for the kernels this one depends on (programmatic launch).
      int pre = 0;
      if ((int)blockIdx.x < ntiles) {
        const int n0 = ((int)blockIdx.x / num_m) * BN;
        pre = nk < S::STAGES ? nk : S::STAGES;
        for (int s = 0; s < pre; ++s) {
          mbar_expect_tx(&full[s], S::STAGE_BYTES);
          tma_load_2d(&tmB, &full[s], smem + s * S::STAGE_BYTES + S::A_BYTES, s * BK, n0);
        }
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      long issues = 0;
      bool first = true;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, first = false) {
        const int m0 = (tile % num_m) * BM;
        const int n0 = (tile / num_m) * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) goto producer_done;
          uint8_t* sa = smem + stage * S::STAGE_BYTES;
          if (!(first && kb < pre)) {
            mbar_expect_tx(&full[stage], S::STAGE_BYTES);
            tma_load_2d(&tmB, &full[stage], sa + S::A_BYTES, kb * BK, n0);
          }
          tma_load_2d(&tmA, &full[stage], sa, kb * BK, m0);
          ++issues;
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      pdl_launch_dependents();  // every tile load is issued: the next kernel may start its prologue
      // tail: wait until the MMA has released the stages filled last, so no commit arrival
      // is still in flight towards this CTA's barriers when it exits
      if (!*abort_flag) {
        for (int s = 0; s < S::STAGES && s < issues; ++s) {
          int st = stage - 1 - s;
          uint32_t ph = phase;
          if (st < 0) {
            st += S::STAGES;
            ph ^= 1u;
          }
          mbar_wait(&empty[st], ph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA's shared memory goes away;
        // W tiles issued ahead of the dependency wait whose A half never followed cannot
        // complete their barrier phase, so their wait simply runs out its bounded time
        for (long s = issues; s < pre; ++s) drain_wait(&full[s], 0);
        for (int s = 0; s < S::STAGES; ++s) {
          if (issues <= 0) break;
          int st = stage - 1 - s;
          uint32_t ph = phase;
          if (st < 0) {
            st += S::STAGES;
            ph ^= 1u;
          }
          drain_wait(&full[st], ph);
          --issues;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
          const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc_mma_f16(d_tmem, sdesc_kmajor_sw128(a_addr + k * 32), sdesc_kmajor_sw128(b_addr + k * 32), idesc,
                       (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      // tail: the epilogue has released the last accumulators (no arrival left in flight)
      for (int i = 0; i < 2 && i < local; ++i) {
        const int t = local - 1 - i;
        if (!mbar_wait(&tempty[t & 1], (t >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) break;
      }
    }
  } else {
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    pdl_wait();                    // the epilogue reads and writes global memory
    int local = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      const int m0 = (tile % num_m) * BM;
      const int n0 = (tile / num_m) * BN;
      const int row = m0 + quarter * 32 + lane;
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if constexpr (KIND == EPI_RESID && BN == 128) {
        // the residual row segment does not depend on the MMAs: fetch it while they run
        float4 xr[32];
        const float4* xrow = reinterpret_cast<const float4*>(ep.resid + (long)(row < M ? row : 0) * ep.ldr + n0);
#pragma unroll
        for (int i = 0; i < 32; ++i) xr[i] = xrow[i];
        bool ok = mbar_wait(&tfull[acc], aph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
        if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.ld below is warp-collective
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
          float v[32];
          tmem_ld32(tb + c, v);
          tc_wait_ld();
          if (row < M) epi_resid_chunk_pref(ep, row, n0 + c, v, &xr[c >> 2]);
        }
      } else {
        bool ok = mbar_wait(&tfull[acc], aph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
        if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.ld below is warp-collective
        tc_fence_after();
#pragma unroll 1
        for (int g = 0; g < BN; g += 128) {
          float ssq = 0.f;
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            float v[32];
            tmem_ld32(tb + g + c, v);
            tc_wait_ld();
            if (row < M) epi_chunk<KIND, OutT>(ep, row, n0 + g + c, v, ssq);
          }
          if (row < M) epi_group_end<KIND>(ep, row, n0 + g, ssq);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

template <int BN, int KIND, typename OutT>
cudaError_t launch_tc(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, const EpiParams& ep,
                      unsigned* err, int num_sms, cudaStream_t st) {
  using S = TcShape<BN>;
  const int tiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_pdl(gemm_tc_kernel<BN, KIND, OutT>, dim3(grid), dim3(192), S::SMEM, st, a, b, M, N, K, ep, err);
}


// ------------------------------------------------------------------ CTA-pair variant
// Two CTAs of a cluster compute a 256 x BN tile with tcgen05.mma.cta_group::2: each CTA
// loads its own 128 rows of A and half (BN/2 rows) of the W tile, the even CTA issues
// M=256 MMAs that read both CTAs' shared memory, and each CTA's TMEM receives its 128
// rows. Per unit of MMA work a CTA streams A + W/2 instead of A + W, which is what the
// per-SM operand bandwidth limits at these sizes. All loads are per-CTA (no multicast).
// Cluster c of a launch with ncl clusters takes tiles c, c + ncl, c + 2 ncl, ... (tiles in
// m-fastest order, so the clusters working at the same time share W n-tiles in L2).
//
// Eight epilogue warps, two per TMEM lane quarter (warp w reads lanes 32 * (w % 4)..+31):
// warps 2-5 take the tile's columns [0, EPI_SPLIT) and warps 6-9 [EPI_SPLIT, BN), so that
// each SM sub-partition has one warp's TMEM loads, L2 loads and stores in flight while
// the other computes. Where a 128-column norm group straddles EPI_SPLIT (BN = 128), the
// second warp hands its partial sum of squares to the first through shared memory.
constexpr int EPI_WARPS = 8;
constexpr int TC2_THREADS = 64 + 32 * EPI_WARPS;

template <int BN>
struct Tc2Shape {
  static constexpr int BNH = BN / 2;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BNH * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TX_BYTES = 2 * STAGE_BYTES;  // both CTAs' loads complete on the even CTA's barrier
  // two accumulators of BN columns, allocated as a power of two
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  // epilogue staging: per epilogue warp STG_BOXES 32-row boxes of up to 128-byte rows (one:
  // the ring's bytes in flight, not the epilogue, bound these main loops)
  static constexpr int STG_BOXES = 1;
  static constexpr uint32_t STG_BYTES = EPI_WARPS * STG_BOXES * 4096;
  static constexpr uint32_t AUX_BYTES = 2048;  // barriers and the norm hand-over
  // the operand ring takes what is left of the 227 KB a CTA may use (up to 8 stages)
  static constexpr int FIT = (int)((227u * 1024u - 1024u - AUX_BYTES - STG_BYTES) / STAGE_BYTES);
  static constexpr int STAGES = FIT < 8 ? FIT : 8;
  static constexpr uint32_t RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr uint32_t SMEM = RING_BYTES + STG_BYTES + 1024 /*align*/ + AUX_BYTES;
  // the first column of the second epilogue warp of a quarter
  static constexpr int EPI_SPLIT = ((BN / 32 + 1) / 2) * 32;
  static_assert(STAGES >= 4, "the operand ring needs at least four stages");
};

template <int BN, int KIND, typename OutT>
__global__ void __launch_bounds__(TC2_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, int M, int N, int K, EpiParams ep, unsigned* err) {
  using S = Tc2Shape<BN>;
  // element type of the staged boxes: the fp32 residual for EPI_RESID, else the output type
  using StageT = typename std::conditional<KIND == EPI_RESID, float, OutT>::type;
  // the 128-column group whose columns both warps of a quarter hold, or -1
  constexpr int SPLIT_GROUP = (S::EPI_SPLIT & 127) ? (S::EPI_SPLIT & ~127) : -1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* xssq = reinterpret_cast<float*>(smem + S::RING_BYTES + S::STG_BYTES);  // [2 slots][4 quarters][32 rows]
  uint64_t* full = reinterpret_cast<uint64_t*>(xssq + 2 * 4 * 32);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* xbar = tempty + 2;  // [2 slots][4 quarters]: the second warp's partial sums are in xssq
  uint64_t* dealloc_bar = xbar + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dealloc_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the pair's MMAs
  const int cl = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;
  const int num_m = (M + 2 * BM - 1) / (2 * BM);
  const int ntiles = num_m * (N / BN);
  const int nk = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * EPI_WARPS);  // both CTAs' epilogue threads
    }
    for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], 32);
    mbar_init(dealloc_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // The weights W are never written by any kernel: stream the first stages' W halves
      // of the first tile before waiting for the kernels this one depends on (programmatic
      // launch).
      const int pre = cl < ntiles ? (nk < S::STAGES ? nk : S::STAGES) : 0;
      for (int s = 0; s < pre; ++s) {
        if (rank == 0) mbar_expect_tx(&full[s], S::TX_BYTES);
        tma_load_2d_pair(&tmB, mapa_shared(smem_u32(&full[s]), 0), smem + s * S::STAGE_BYTES + S::A_BYTES, s * BK,
                         (cl / num_m) * BN + (int)rank * S::BNH);
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      int issues = 0;
      for (int tile = cl; tile < ntiles; tile += ncl) {
        const int m0 = (tile % num_m) * 2 * BM + (int)rank * BM;
        const int n0 = (tile / num_m) * BN + (int)rank * S::BNH;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) goto producer_done;
          uint8_t* sa = smem + stage * S::STAGE_BYTES;
          const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
          if (!(tile == cl && kb < pre)) {
            if (rank == 0) mbar_expect_tx(&full[stage], S::TX_BYTES);
            tma_load_2d_pair(&tmB, bar0, sa + S::A_BYTES, kb * BK, n0);
          }
          tma_load_2d_pair(&tmA, bar0, sa, kb * BK, m0);
          ++issues;
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      pdl_launch_dependents();
      // tail: the even CTA's MMA has released (multicast commit into this CTA) every stage
      // filled last, so no arrival is in flight towards this CTA when it exits
      if (!*abort_flag) {
        for (int s = 0; s < S::STAGES && s < issues; ++s) {
          int st = stage - 1 - s;
          uint32_t ph = phase;
          if (st < 0) {
            st += S::STAGES;
            ph ^= 1u;
          }
          mbar_wait(&empty[st], ph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
        }
      }
      if (*abort_flag) {  // give copies already issued time to land (their barrier is the even CTA's)
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = cl; tile < ntiles; tile += ncl, ++local) {
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
          const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc_mma_f16_pair(d_tmem, sdesc_kmajor_sw128(a_addr + k * 32), sdesc_kmajor_sw128(b_addr + k * 32), idesc,
                            (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(&tfull[acc], 0x3);
      }
      // tail: both CTAs' epilogues have released the last accumulators (their arrivals,
      // local and remote, have landed on this CTA's barriers)
      for (int i = 0; i < 2 && i < local; ++i) {
        const int t = local - 1 - i;
        if (!mbar_wait(&tempty[t & 1], (t >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) break;
      }
    }
  } else {
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;  // 0: columns [0, EPI_SPLIT), 1: [EPI_SPLIT, BN)
    const int cbeg = sub ? S::EPI_SPLIT : 0;
    const int cend = sub ? BN : S::EPI_SPLIT;
    uint8_t* stg = smem + S::RING_BYTES + (warp - 2) * (S::STG_BOXES * 4096);  // this warp's staging boxes
    uint32_t nchunk = 0;
    uint32_t nx = 0;  // norm hand-overs between this quarter's two warps so far
    pdl_wait();
    int local = 0;
    for (int tile = cl; tile < ntiles; tile += ncl, ++local) {
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      const int m0 = (tile % num_m) * 2 * BM + (int)rank * BM;
      const int n0 = (tile / num_m) * BN;
      const int row0 = m0 + quarter * 32;
      const int row = row0 + lane;
      const int rowc = row < M ? row : M - 1;
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      epi_prefetch<KIND>(ep, rowc, n0 + cbeg, cend - cbeg);  // while the MMAs run
      // EPI_QKV: the 32 rows stay inside one stream (row0 and L both multiples of 32 at
      // the usual sizes); otherwise this warp stores directly, row by row
      bool direct = false;
      int l0 = 0, bidx = 0;
      if constexpr (KIND == EPI_QKV) {
        l0 = row0 % ep.rows_per_batch;
        bidx = row0 / ep.rows_per_batch;
        direct = l0 + 32 > ep.rows_per_batch && row0 + (ep.rows_per_batch - l0) < M;
      }
      // EPI_QKV: the rotary (cos, sin) of the next chunk, loaded one chunk ahead (the first
      // chunk's while the MMAs run)
      float4 rope_cur[8], rope_nxt[8];
      const bool rope_rows = KIND == EPI_QKV && row0 < M && !direct;
      if (rope_rows && epi_normed(ep, n0 + cbeg)) epi_rope_load(ep, rowc, n0 + cbeg, rope_cur);
      bool ok = mbar_wait(&tfull[acc], aph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // one 32-column chunk of the tile: the epilogue and the store
      float ssq = 0.f;
      auto chunk = [&](float (&v)[32], int c) {
        if (rope_rows && c + 32 < cend && epi_normed(ep, n0 + c + 32)) epi_rope_load(ep, rowc, n0 + c + 32, rope_nxt);
        if (direct) {
          if (row < M) epi_chunk<KIND, OutT>(ep, row, n0 + c, v, ssq);
        } else {
          if (row < M) {
            epi_math<KIND, OutT>(ep, row, n0 + c, v, ssq);
            if constexpr (KIND == EPI_QKV)
              if (epi_normed(ep, n0 + c)) epi_rope_apply(rope_cur, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
          }
          // buffers alternate per committed store, so the one group that may still be
          // reading is the other buffer's (one buffer: no group may still be reading it)
          uint8_t* box = stg + (S::STG_BOXES == 2 ? (nchunk & 1) * 4096 : 0);
          if (lane == 0) bulk_wait_read<S::STG_BOXES - 1>();
          __syncwarp();
          if (KIND == EPI_QKV && std::is_same<OutT, bf16>::value && (n0 + c) / ep.dim == 2)
            stage_row(box, lane, v, (__half*)nullptr);  // v in fp16 (epilogue.cuh, EPI_QKV)
          else
            stage_row(box, lane, v, (StageT*)nullptr);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int col = n0 + c;
            if constexpr (KIND == EPI_RESID) {
              tma_reduce_add_2d(&tmC, box, col, row0);  // rows at or past M are clipped
            } else if constexpr (KIND == EPI_QKV) {
              const int sec = col / ep.dim, cin = col - sec * ep.dim;
              const int heads = ep.dim >> 7;
              const int nb = M / ep.rows_per_batch;
              tma_store_3d(&tmC, box, cin & 127, l0, (sec * nb + bidx) * heads + (cin >> 7));
            } else {
              tma_store_2d(&tmC, box, col, row0);
            }
            bulk_commit();
          }
          ++nchunk;
        }
        if constexpr (KIND == EPI_NORM || KIND == EPI_QKV) {
          if ((c & 127) == 96 || c + 32 == cend) {  // the end of this warp's part of a 128-column group
            const int g0 = c & ~127;
            if (g0 == SPLIT_GROUP) {
              // the quarter's two warps each summed part of the group: the second hands its
              // sums to the first, which writes the group's total
              // (two slots by hand-over count: the second warp reaches hand-over x + 2 only
              // after the first has read x and released that tile's accumulator)
              float* xs = xssq + ((nx & 1) * 4 + quarter) * 32;
              uint64_t* xb = &xbar[(nx & 1) * 4 + quarter];
              if (sub) {
                xs[lane] = ssq;
                mbar_arrive(xb);
              } else if (mbar_wait(xb, (nx >> 1) & 1, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) {
                if (row < M) epi_group_end<KIND>(ep, row, n0 + g0, ssq + xs[lane]);
              }
              ++nx;
            } else if (row < M) {
              epi_group_end<KIND>(ep, row, n0 + g0, ssq);
            }
            ssq = 0.f;
          }
        }
        if constexpr (KIND == EPI_QKV) {
#pragma unroll
          for (int k = 0; k < 8; ++k) rope_cur[k] = rope_nxt[k];
        }
      };
      if (row0 < M) {  // a quarter with no row below M stores nothing
#pragma unroll 1
        for (int c = cbeg; c < cend; c += 32) {
          float v[32];
          tmem_ld32(tb + c, v);
          tc_wait_ld();
          chunk(v, c);
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (*abort_flag) break;
    }
    if (lane == 0) bulk_wait_all();  // every store issued by this warp has been performed
    __syncwarp();
  }

  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // both CTAs are past their last TMEM access before the pair's allocation is released
    if (lane == 0) {
      mbar_arrive_cluster(mapa_shared(smem_u32(dealloc_bar), rank ^ 1u));
      drain_wait(dealloc_bar, 0);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

// CTA pairs of the pair GEMM, and clusters of four of the split-K kernel, that can be
// resident at once, per device (set by gemm_tc_prepare): the pair GEMM is persistent (one
// cluster per resident pair), and a split-K cluster's pairs wait for each other, so every
// cluster of a split-K launch must be able to run at the same time.
int g_pair_clusters[64] = {0};
int g_split_clusters[64] = {0};

// Clusters of a pair-GEMM launch: one per CTA pair that can be resident, or one per tile
// when there are fewer tiles.
inline int tc2_clusters(int M, int N, int bn, int num_sms) {
  const long tiles = (long)((M + 2 * BM - 1) / (2 * BM)) * (N / bn);
  int dev = 0;
  cudaGetDevice(&dev);
  int cap = num_sms / 2;
  const int resident = dev >= 0 && dev < 64 ? g_pair_clusters[dev] : 0;
  if (resident > 0 && resident < cap) cap = resident;
  return tiles < cap ? (int)tiles : cap;
}

template <int BN, int KIND, typename OutT>
cudaError_t launch_tc2(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, int M, int N, int K,
                       const EpiParams& ep, unsigned* err, int num_sms, cudaStream_t st) {
  using S = Tc2Shape<BN>;
  const int clusters = tc2_clusters(M, N, BN, num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(TC2_THREADS);
  cfg.dynamicSmemBytes = S::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<BN, KIND, OutT>, a, b, c, M, N, K, ep, err);
}

// ------------------------------------------------------------------ split-K over two CTA pairs
// GEMMs with few output tiles (M = 1280, N = 1536: 30 tiles of 256 x 256) run one tile per
// cluster of four CTAs. CTA pair s (cluster ranks 2s, 2s+1) computes the tile over half of
// the K range with cta_group::2 MMAs into its own TMEM accumulator, on 256-wide tiles whose
// operand traffic per MMA is the lowest the pair can have. The pairs then reduce-scatter
// through shared memory: each CTA finalises 128 of the 256 columns of its rows, receiving
// the partner pair's fp32 partial sums for them by bulk copies into its operand ring (free
// once its pair's MMAs are done), adding them to its own and running the staged epilogue.
// Eight epilogue warps as in the pair GEMM: the quarter's two warps take 64 of the 128
// columns each, in both the hand-over and the epilogue. One tile per cluster: the host
// launches this only when the tiles fit the clusters of four that can be resident at once.
struct Tc2sShape {
  static constexpr int BN = 256;
  static constexpr int STAGES = 6;
  static constexpr uint32_t STAGE_BYTES = BM * BK * 2 + (BN / 2) * BK * 2;
  static constexpr uint32_t RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr uint32_t HALF_COLS = BN / 2;
  static constexpr uint32_t QBYTES = HALF_COLS * 128;  // one quarter's rows of half the columns, fp32
  static constexpr uint32_t RX = 4 * QBYTES;           // ring offset of the partner's half
  // the staging boxes of the first four epilogue warps; the other four stage in the ring
  // past both halves (idle once the pair's MMAs are done)
  static constexpr uint32_t STG_BYTES = 4 * 2 * 4096;
  static constexpr uint32_t STG2 = 2 * RX;
  static constexpr uint32_t SMEM = RING_BYTES + STG_BYTES + 1024 /*align*/ + 2048 /*barriers*/;
  static_assert(STG2 + 4 * 2 * 4096 <= RING_BYTES, "both halves and four warps' boxes must fit in the ring");
  static_assert(SMEM <= 227u * 1024u, "shared memory per CTA");
};

template <int BN, int KIND, typename OutT>
__global__ void __launch_bounds__(TC2_THREADS, 1)
    gemm_tc2s_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, int M, int N, int K, EpiParams ep, unsigned* err) {
  using S = Tc2sShape;
  static_assert(KIND != EPI_QKV, "the head-major scatter runs on the plain pair kernel");
  static_assert(BN == S::BN, "each CTA finalises one 128-column group");
  constexpr uint32_t HALF_COLS = S::HALF_COLS, QBYTES = S::QBYTES, RX = S::RX;
  constexpr int BNH = BN / 2;
  constexpr uint32_t A_BYTES = BM * BK * 2;
  constexpr uint32_t TX_BYTES = 2 * S::STAGE_BYTES;
  using StageT = typename std::conditional<KIND == EPI_RESID, float, OutT>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* xssq = reinterpret_cast<float*>(smem + S::RING_BYTES + S::STG_BYTES);  // [4 quarters][32 rows]
  uint64_t* full = reinterpret_cast<uint64_t*>(xssq + 4 * 32);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* ring_free = tfull + 1;       // the partner's MMAs are done: its ring may be written
  uint64_t* part_ready = ring_free + 1;  // [4 quarters][2 warps] the partner's 64 columns of them landed
  uint64_t* xbar = part_ready + 8;       // [4 quarters] the second warp's sums of squares are in xssq
  uint64_t* done = xbar + 4;             // every other CTA of the cluster is finished with this one
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t split = rank >> 1;      // which half of K
  const uint32_t half = rank & 1;        // which 128 rows of the tile
  const uint32_t lead = rank & 2;        // the pair's MMA-issuing CTA
  const uint16_t mask = (uint16_t)(0x3u << lead);
  const int tile = blockIdx.x >> 2;
  const int num_m = (M + 2 * BM - 1) / (2 * BM);
  const int m0 = (tile % num_m) * 2 * BM + (int)half * BM;
  const int n0 = (tile / num_m) * BN;
  const int nk = (K + BK - 1) / BK;
  const int kb0 = split ? nk / 2 : 0, kb1 = split ? nk : nk / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(ring_free, 1);
    for (int q = 0; q < 8; ++q) mbar_init(&part_ready[q], 1);
    for (int q = 0; q < 4; ++q) mbar_init(&xbar[q], 32);
    mbar_init(done, 3);
    *abort_flag = 0;
    fence_mbar_init();
    // each warp's 64 columns of a quarter's rows arrive as one bulk copy
    for (int q = 0; q < 8; ++q) mbar_expect_tx(&part_ready[q], QBYTES / 2);
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, BN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // all four CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // the first stages' W halves before the dependency wait (W is never written)
      const int pre = kb1 - kb0 < S::STAGES ? kb1 - kb0 : S::STAGES;
      for (int s = 0; s < pre; ++s) {
        if (half == 0) mbar_expect_tx(&full[s], TX_BYTES);
        tma_load_2d_pair(&tmB, mapa_shared(smem_u32(&full[s]), lead), smem + s * S::STAGE_BYTES + A_BYTES,
                         (kb0 + s) * BK, n0 + (int)half * BNH);
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      int issues = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) goto producer_done;
        uint8_t* sa = smem + stage * S::STAGE_BYTES;
        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), lead);
        if (kb - kb0 >= pre) {
          if (half == 0) mbar_expect_tx(&full[stage], TX_BYTES);
          tma_load_2d_pair(&tmB, bar, sa + A_BYTES, kb * BK, n0 + (int)half * BNH);
        }
        tma_load_2d_pair(&tmA, bar, sa, kb * BK, m0);
        ++issues;
        if (++stage == S::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    producer_done:
      pdl_launch_dependents();
      // the lead CTA's release commits for the stages filled last have landed here
      if (!*abort_flag) {
        for (int s = 0; s < S::STAGES && s < issues; ++s) {
          int st = stage - 1 - s;
          uint32_t ph = phase;
          if (st < 0) {
            st += S::STAGES;
            ph ^= 1u;
          }
          mbar_wait(&empty[st], ph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
        }
      }
      if (*abort_flag) {  // give copies already issued time to land (their barrier is the lead CTA's)
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && half == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * BM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          tc_mma_f16_pair(tmem_base, sdesc_kmajor_sw128(a_addr + k * 32), sdesc_kmajor_sw128(b_addr + k * 32), idesc,
                          (kb > kb0 || k > 0) ? 1u : 0u);
        tc_commit_pair(&empty[stage], mask);
        if (++stage == S::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) tc_commit_pair(tfull, mask);
    }
  } else {
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;  // which 64 of the 128 columns of each half
    const int row0 = m0 + quarter * 32;
    const int row = row0 + lane;
    const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16);
    pdl_wait();
    bool ok = mbar_wait(tfull, 0, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) tc_fence_after();
    // Reduce-scatter between the pairs: the CTA finalises columns [mine, mine + BN/2) of its
    // 128 rows and its partner (same rows, other half of K, cluster rank ^ 2) the other
    // half. Each stages the partner's half of its accumulator in its own ring (free: its
    // pair's MMAs are done) as [BN/64 chunks][32 rows][32 columns] fp32 per quarter with
    // the 16-byte pieces of each row swizzled by row, and one bulk copy per warp (its two
    // chunks) moves it into the partner's ring at offset RX once the partner's MMAs are
    // done with it.
    const uint32_t partner = rank ^ 2u;
    const int mine = (int)split * (int)HALF_COLS, theirs = (int)HALF_COLS - mine;
    const int c0 = sub * 64;  // this warp's columns within each half
    if (ok && quarter == 0 && sub == 0 && lane == 0)
      mbar_arrive_release_cluster(mapa_shared(smem_u32(ring_free), partner));
    epi_prefetch<KIND>(ep, row < M ? row : M - 1, n0 + mine + c0, 64);
    if (ok && row0 < M) {
      uint8_t* out = smem + quarter * QBYTES + sub * (QBYTES / 2);
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float v[32];
        tmem_ld32(tb + theirs + c0 + c, v);
        tc_wait_ld();
        uint8_t* prow = out + (c >> 5) * 4096 + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(prow + ((j ^ (lane & 7)) << 4)) =
              make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(ring_free, 0, abort_flag, err, ERRBIT_TIMEOUT_GEMM));
      if (ok && lane == 0)
        bulk_copy_to_cluster(mapa_shared(smem_u32(smem + RX + quarter * QBYTES + sub * (QBYTES / 2)), partner), out,
                             QBYTES / 2, mapa_shared(smem_u32(&part_ready[quarter * 2 + sub]), partner));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(&part_ready[quarter * 2 + sub], 0, abort_flag, err,
                                                             ERRBIT_TIMEOUT_GEMM));
    }
    // the finalised columns: own accumulator + the partner's, then the staged epilogue
    const uint8_t* part = smem + RX + quarter * QBYTES + sub * (QBYTES / 2);
    uint8_t* stg = sub ? smem + S::STG2 + quarter * 8192 : smem + S::RING_BYTES + quarter * 8192;
    uint32_t nchunk = 0;
    if (ok && row0 < M) {
      float ssq = 0.f;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float v[32];
        tmem_ld32(tb + mine + c0 + c, v);
        tc_wait_ld();
        const int col = n0 + mine + c0 + c;
        const uint8_t* prow = part + (c >> 5) * 4096 + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 pp = *reinterpret_cast<const float4*>(prow + ((j ^ (lane & 7)) << 4));
          v[4 * j] += pp.x;
          v[4 * j + 1] += pp.y;
          v[4 * j + 2] += pp.z;
          v[4 * j + 3] += pp.w;
        }
        if (row < M) {
          epi_math<KIND, OutT>(ep, row, col, v, ssq);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
        uint8_t* box = stg + (nchunk & 1) * 4096;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        stage_row(box, lane, v, (StageT*)nullptr);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (KIND == EPI_RESID)
            tma_reduce_add_2d(&tmC, box, col, row0);
          else
            tma_store_2d(&tmC, box, col, row0);
          bulk_commit();
        }
        ++nchunk;
      }
      if constexpr (KIND == EPI_NORM) {
        // the group's sum of squares: the second warp hands its part to the first
        if (sub) {
          xssq[quarter * 32 + lane] = ssq;
          mbar_arrive(&xbar[quarter]);
        } else if (mbar_wait(&xbar[quarter], 0, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) {
          if (row < M) epi_group_end<KIND>(ep, row, n0 + mine, ssq + xssq[quarter * 32 + lane]);
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // every role ends here with its warp converged again (a lane that did a role's work arrives
  // after the others), so the CTA barrier below counts each warp once, after all of its work
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every CTA of the cluster is past its last access to the others' shared memory and
    // TMEM before any of them leaves or frees the pair's TMEM
    if (lane == 0) {
      for (uint32_t r = 0; r < 4; ++r)
        if (r != rank) mbar_arrive_release_cluster(mapa_shared(smem_u32(done), r));
      drain_wait(done, 0);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, BN);
  }
}

template <int BN, int KIND, typename OutT>
cudaError_t launch_tc2s(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, int M, int N, int K,
                        const EpiParams& ep, unsigned* err, cudaStream_t st) {
  using S = Tc2sShape;
  const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * (N / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4 * tiles);
  cfg.blockDim = dim3(TC2_THREADS);
  cfg.dynamicSmemBytes = S::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 4;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_tc2s_kernel<BN, KIND, OutT>, a, b, c, M, N, K, ep, err);
}

template <int BN, int KIND, typename OutT>
cudaError_t prepare_tc2s() {
  return cudaFuncSetAttribute(gemm_tc2s_kernel<BN, KIND, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Tc2sShape::SMEM);
}

template <int BN, int KIND, typename OutT>
cudaError_t prepare_tc2() {
  return cudaFuncSetAttribute(gemm_tc2_kernel<BN, KIND, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Tc2Shape<BN>::SMEM);
}

template <int BN, int KIND, typename OutT>
cudaError_t prepare_tc() {
  return cudaFuncSetAttribute(gemm_tc_kernel<BN, KIND, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)TcShape<BN>::SMEM);
}

}  // namespace

cudaError_t gemm_tc_prepare() {
  const cudaError_t es[] = {
      prepare_tc<128, EPI_STORE, bf16>(), prepare_tc<256, EPI_STORE, bf16>(), prepare_tc<128, EPI_GELU, bf16>(),
      prepare_tc<256, EPI_GELU, bf16>(),  prepare_tc<128, EPI_NORM, bf16>(),  prepare_tc<256, EPI_NORM, bf16>(),
      prepare_tc<128, EPI_QKV, bf16>(),   prepare_tc<256, EPI_QKV, bf16>(),   prepare_tc<128, EPI_RESID, bf16>(),
      prepare_tc<256, EPI_RESID, bf16>(), prepare_tc<128, EPI_STORE, float>(), prepare_tc<256, EPI_STORE, float>(),
      prepare_tc2<128, EPI_STORE, bf16>(), prepare_tc2<256, EPI_STORE, bf16>(), prepare_tc2<128, EPI_GELU, bf16>(),
      prepare_tc2<256, EPI_GELU, bf16>(), prepare_tc2<128, EPI_NORM, bf16>(), prepare_tc2<256, EPI_NORM, bf16>(),
      prepare_tc2<128, EPI_QKV, bf16>(), prepare_tc2<256, EPI_QKV, bf16>(), prepare_tc2<128, EPI_RESID, bf16>(),
      prepare_tc2<256, EPI_RESID, bf16>(), prepare_tc2<128, EPI_STORE, float>(), prepare_tc2<256, EPI_STORE, float>(),
      prepare_tc2<224, EPI_GELU, bf16>(), prepare_tc2<224, EPI_STORE, float>()};
  for (cudaError_t e : es)
    if (e != cudaSuccess) return e;
  const cudaError_t es2[] = {prepare_tc2s<256, EPI_STORE, bf16>(), prepare_tc2s<256, EPI_NORM, bf16>(),
                             prepare_tc2s<256, EPI_RESID, bf16>(), prepare_tc2s<256, EPI_STORE, float>()};
  for (cudaError_t e : es2)
    if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 64);
  cfg.blockDim = dim3(TC2_THREADS);
  cfg.dynamicSmemBytes = Tc2Shape<256>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<256, EPI_RESID, bf16>, &cfg);
  if (e != cudaSuccess) return e;
  int n4 = 0;
  attr[0].val.clusterDim.x = 4;
  cfg.gridDim = dim3(4 * 64);
  cfg.dynamicSmemBytes = Tc2sShape::SMEM;
  e = cudaOccupancyMaxActiveClusters(&n4, gemm_tc2s_kernel<256, EPI_RESID, bf16>, &cfg);
  if (e != cudaSuccess) return e;
  int dev = 0;
  cudaGetDevice(&dev);
  if (n < 1) return cudaErrorInvalidConfiguration;
  if (dev >= 0 && dev < 64) {
    g_pair_clusters[dev] = n;
    g_split_clusters[dev] = n4;
  }
  return cudaSuccess;
}

cudaError_t gemm_tc(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap* c, int M, int N, int K, int bn,
                    int kind, bool out_bf16, const EpiParams& ep, unsigned* err, int num_sms, cudaStream_t st,
                    bool pair) {
  // the CTA-pair kernels store their epilogue through the output map `c`
  if (pair && !c) return cudaErrorInvalidValue;
  const CUtensorMap& cm = c ? *c : a;
  // few 256 x 256 tiles (one per cluster of four fits the GPU): split K over two CTA pairs
  // of a cluster
  const int tiles256 = ((M + 2 * BM - 1) / (2 * BM)) * (N / 256);
  int dev = 0;
  cudaGetDevice(&dev);
  const int resident4 = dev >= 0 && dev < 64 ? g_split_clusters[dev] : 0;
  if (pair && bn == 256 && N <= 4096 && 4 * tiles256 <= num_sms &&
      tiles256 <= resident4 && K >= 2 * BK && (kind == EPI_STORE || kind == EPI_NORM || kind == EPI_RESID)) {
    if (out_bf16) {
      if (kind == EPI_STORE) return launch_tc2s<256, EPI_STORE, bf16>(a, b, cm, M, N, K, ep, err, st);
      if (kind == EPI_NORM) return launch_tc2s<256, EPI_NORM, bf16>(a, b, cm, M, N, K, ep, err, st);
      return launch_tc2s<256, EPI_RESID, bf16>(a, b, cm, M, N, K, ep, err, st);
    }
    if (kind == EPI_STORE) return launch_tc2s<256, EPI_STORE, float>(a, b, cm, M, N, K, ep, err, st);
  }
#define FH_TC_CASE(BNV, KV, OT)                                                                     \
  if (bn == BNV && kind == KV)                                                                      \
    return pair ? launch_tc2<BNV, KV, OT>(a, b, cm, M, N, K, ep, err, num_sms, st)              \
                : launch_tc<BNV, KV, OT>(a, b, M, N, K, ep, err, num_sms, st);
  if (pair && bn == 224) {  // FFN1-shaped (8960 = 40 x 224 balances the waves)
    if (kind == EPI_GELU && out_bf16)
      return launch_tc2<224, EPI_GELU, bf16>(a, b, cm, M, N, K, ep, err, num_sms, st);
    if (kind == EPI_STORE && !out_bf16)
      return launch_tc2<224, EPI_STORE, float>(a, b, cm, M, N, K, ep, err, num_sms, st);
    return cudaErrorInvalidValue;
  }
  if (out_bf16) {
    FH_TC_CASE(128, EPI_STORE, bf16)
    FH_TC_CASE(256, EPI_STORE, bf16)
    FH_TC_CASE(128, EPI_GELU, bf16)
    FH_TC_CASE(256, EPI_GELU, bf16)
    FH_TC_CASE(128, EPI_NORM, bf16)
    FH_TC_CASE(256, EPI_NORM, bf16)
    FH_TC_CASE(128, EPI_QKV, bf16)
    FH_TC_CASE(256, EPI_QKV, bf16)
    FH_TC_CASE(128, EPI_RESID, bf16)
    FH_TC_CASE(256, EPI_RESID, bf16)
  } else {
    FH_TC_CASE(128, EPI_STORE, float)
    FH_TC_CASE(256, EPI_STORE, float)
  }
#undef FH_TC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fh
