// gemm_tc.cu - bf16 tensor-core GEMM with fused epilogues for sm_100a.
//
// out[M, N] = epilogue(A[M, K] * W[N, K]^T): A is an activation (bf16, row-major,
// K contiguous), W a Linear weight in nn.Linear layout [out, in] (bf16, K
// contiguous). This is every dense contraction of the DiT: patch embed, QKV,
// O-proj, cross-Q, cross-KV, cross-O, FFN1, FFN2 and the head.
//
// Two kernels, both warp-specialised with 192 threads:
//   warp 0     TMA producer: one thread streams 64-deep A and W tiles with the
//              128-byte swizzle into a STAGES-deep shared-memory ring (per-CTA
//              loads, no cluster multicast), the first stages' W before the
//              programmatic-launch dependency wait (W is never written).
//   warp 1     allocates TMEM and, from one thread, issues tcgen05.mma (fp32
//              accumulate in TMEM); each stage is released by tcgen05.commit to
//              its "empty" mbarrier and each finished tile by a commit to its
//              accumulator's "full" barrier.
//   warps 2-5  epilogue: tcgen05.ld of 32 columns at a time (warp w reads TMEM
//              lanes 32*(w%4)..+31 = its 32 output rows) and the fused epilogue.
// gemm_tc_kernel    one CTA per SM, persistent over 128 x BN tiles
//                   (cta_group::1), two accumulators so the epilogue of tile i
//                   overlaps the MMAs of tile i+1, direct 16-byte stores.
// gemm_tc2_kernel   a CTA pair (cluster of 2) per 256 x BN tile (cta_group::2),
//                   persistent over a stream-K share of the tiles' k-blocks (one
//                   cluster per CTA pair of the GPU, every share the same size;
//                   tiles cut between clusters are summed by the owner through
//                   fp32 partials in the workspace), two accumulators; the
//                   epilogue stages 32 x 32 boxes in shared memory and stores them
//                   by TMA (the residual as a TMA fp32 reduce-add into x).
// Every wait is bounded (FH_WAIT_LIMIT_NS); on expiry the CTA latches an error
// bit, lets the producer's in-flight copies land, frees TMEM and exits.
#include <cstdio>
#include <type_traits>

#include "epilogue.cuh"
#include "kernels.h"
#include "rownorm.cuh"

namespace fh {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int SK_COLS = 256;  // columns of a stream-K partial-sum slot row (the widest tile)

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
//
// Work split (stream-K): the tiles' 64-deep k-blocks, taken tile by tile (tiles in
// m-fastest order, so clusters working at the same time share W n-tiles in L2), form one
// range of units that is cut into equal contiguous shares, one per cluster. A cluster's
// share is a sequence of segments (tile, k-blocks [kb0, kb1)). A segment that covers a
// whole tile runs the epilogue. Where a tile is cut between clusters, the segment that
// starts at k-block 0 is its owner and the later ones are contributors: a contributor is
// always the first segment of its cluster's share and the owner the last of its own, so
// contributors finish early and no cluster waits on one that is waiting itself. A
// contributor stores its fp32 partial accumulator in its cluster's slot of the workspace
// (`sk_part`) and counts itself on the tile's flag; the owner waits for the count, adds
// the contributors' partials in k order (a fixed order: the result is deterministic),
// runs the epilogue and clears the flag for the next launch (flags are per 32-row quarter
// of a CTA's rows, so each epilogue warp waits only for the same rows). Without a partial buffer
// (`sk_part` null) the shares are whole tiles.
template <int BN>
struct Tc2Shape {
  static constexpr int BNH = BN / 2;
  static constexpr int STAGES = (BN >= 192) ? 6 : 8;
  // two accumulators of BN columns, allocated as a power of two
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BNH * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TX_BYTES = 2 * STAGE_BYTES;  // both CTAs' loads complete on the even CTA's barrier
  static constexpr uint32_t RING_BYTES = STAGES * STAGE_BYTES;
  // epilogue staging: per epilogue warp two 32-row boxes of up to 128-byte rows
  static constexpr uint32_t STG_BYTES = 4 * 2 * 4096;
  // a stream-K owner's epilogue warps receive the contributors' partial sums as 32 x 32 fp32
  // boxes in the operand ring (idle by then): PBOX boxes per warp, loaded ahead by TMA
  static constexpr int PBOX = RING_BYTES / (4 * 4096) < 12 ? RING_BYTES / (4 * 4096) : 12;
  static constexpr uint32_t SMEM = RING_BYTES + STG_BYTES + 1024 /*align*/ + 1024 /*barriers*/;
};

// One segment of a cluster's work: k-blocks [kb0, kb1) of one tile.
struct SkSeg {
  int tile, kb0, kb1;
};
// A cluster's segments. Stream-K (sk): the k-blocks of all tiles, tile by tile, form one range
// of units cut into equal contiguous shares, one per cluster. Whole tiles (!sk): cluster c takes
// tiles c, c + ncl, c + 2 ncl, ... (so the clusters working at the same time cover consecutive
// tiles, which share W n-tiles in L2).
struct SkRange {
  long total;  // stream-K units: k-blocks of all tiles
  int nk, ncl, ntiles;
  bool sk;
  __device__ __forceinline__ long lo(int c) const { return (long)c * total / ncl; }
  // the first position of cluster c's work, and whether position u is still inside it
  __device__ __forceinline__ long begin(int c) const { return sk ? lo(c) : c; }
  __device__ __forceinline__ bool more(int c, long u) const { return sk ? u < lo(c + 1) : u < ntiles; }
  // the segment at position u of cluster c's work; returns the next position
  __device__ __forceinline__ long seg(int c, long u, SkSeg& s) const {
    if (!sk) {
      s.tile = (int)u;
      s.kb0 = 0;
      s.kb1 = nk;
      return u + ncl;
    }
    const long uh = lo(c + 1);
    s.tile = (int)(u / nk);
    s.kb0 = (int)(u - (long)s.tile * nk);
    const long rem = uh - u;
    s.kb1 = (long)(nk - s.kb0) <= rem ? nk : s.kb0 + (int)rem;
    return u + (s.kb1 - s.kb0);
  }
  // clusters after `cl` whose shares hold later k-blocks of `tile` (its contributors)
  __device__ __forceinline__ int contributors(int tile, int cl) const {
    const long end = (long)(tile + 1) * nk;
    int n = 0;
    for (int c = cl + 1; c < ncl && lo(c) < end; ++c) ++n;
    return n;
  }
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int BN, int KIND, typename OutT>
__global__ void __launch_bounds__(192, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmP, int M, int N,
                    int K, EpiParams ep, unsigned* err) {
  using S = Tc2Shape<BN>;
  static_assert(BN <= SK_COLS, "a partial-sum slot row holds SK_COLS columns");
  // element type of the staged boxes: the fp32 residual for EPI_RESID, else the output type
  using StageT = typename std::conditional<KIND == EPI_RESID, float, OutT>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::RING_BYTES + S::STG_BYTES);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* dealloc_bar = tempty + 2;
  uint64_t* pbar = dealloc_bar + 1;  // [4 warps][PBOX] partial-sum boxes landed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(pbar + 4 * S::PBOX);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the pair's MMAs
  const int cl = blockIdx.x >> 1;
  const int num_m = (M + 2 * BM - 1) / (2 * BM);
  const int num_n = N / BN;
  const int ntiles = num_m * num_n;
  const int nk = (K + BK - 1) / BK;
  SkRange R;
  R.sk = ep.sk_part != nullptr;
  R.nk = nk;
  R.ncl = gridDim.x >> 1;
  R.ntiles = ntiles;
  R.total = (long)ntiles * nk;
  const long u_begin = R.begin(cl);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 128);  // both CTAs' epilogue threads
    }
    mbar_init(dealloc_bar, 1);
    for (int i = 0; i < 4 * S::PBOX; ++i) mbar_init(&pbar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    if (R.sk) prefetch_tmap(&tmP);
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
      // of the share's first segment before waiting for the kernels this one depends on
      // (programmatic launch).
      int pre = 0;
      if (R.more(cl, u_begin)) {
        SkSeg s0;
        R.seg(cl, u_begin, s0);
        const int n0 = (s0.tile / num_m) * BN + (int)rank * S::BNH;
        pre = s0.kb1 - s0.kb0 < S::STAGES ? s0.kb1 - s0.kb0 : S::STAGES;
        for (int s = 0; s < pre; ++s) {
          if (rank == 0) mbar_expect_tx(&full[s], S::TX_BYTES);
          tma_load_2d_pair(&tmB, mapa_shared(smem_u32(&full[s]), 0), smem + s * S::STAGE_BYTES + S::A_BYTES,
                           (s0.kb0 + s) * BK, n0);
        }
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      int issues = 0;
      bool first = true;
      for (long u = u_begin; R.more(cl, u); first = false) {
        SkSeg sg;
        u = R.seg(cl, u, sg);
        const int m0 = (sg.tile % num_m) * 2 * BM + (int)rank * BM;
        const int n0 = (sg.tile / num_m) * BN + (int)rank * S::BNH;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) goto producer_done;
          uint8_t* sa = smem + stage * S::STAGE_BYTES;
          const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
          if (!(first && kb - sg.kb0 < pre)) {
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
      for (long u = u_begin; R.more(cl, u); ++local) {
        SkSeg sg;
        u = R.seg(cl, u, sg);
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, err, ERRBIT_TIMEOUT_GEMM)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
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
                            (kb > sg.kb0 || k > 0) ? 1u : 0u);
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
    uint8_t* stg = smem + S::RING_BYTES + quarter * 8192;  // this warp's two staging boxes
    uint32_t nchunk = 0;
    pdl_wait();
    int local = 0;
    for (long u = u_begin; R.more(cl, u); ++local) {
      SkSeg sg;
      u = R.seg(cl, u, sg);
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      const int m0 = (sg.tile % num_m) * 2 * BM + (int)rank * BM;
      const int n0 = (sg.tile / num_m) * BN;
      const int row = m0 + quarter * 32 + lane;
      const int row0 = m0 + quarter * 32;
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      // one flag per (tile, CTA of the pair, 32-row quarter): the owner's warp for these rows
      // waits only for the contributors' warps that stored the same rows
      int* flag = R.sk ? ep.sk_flags + (2 * sg.tile + (int)rank) * 4 + quarter : nullptr;
      if (sg.kb0 > 0) {
        // contributor: each thread stores its row's raw fp32 partial sums straight from the
        // accumulator into this cluster's slot (row-major rows of SK_COLS floats, which the
        // owner reads back as 32 x 32 TMA boxes); once the warp's stores are visible the
        // quarter's flag counts them
        bool ok = mbar_wait(&tfull[acc], aph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        float* prow = ep.sk_part + ((size_t)(cl * 2 + (int)rank) * BM + quarter * 32 + lane) * SK_COLS;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld32(tb + c, v);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(reinterpret_cast<float4*>(prow + c + 4 * j), make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        }
        tc_fence_before();
        mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        __syncwarp();
        if (lane == 0) {
          __threadfence();  // the warp's partial sums are visible before the flag counts them
          atomicAdd(flag, 1);
        }
        __syncwarp();
        continue;
      }
      // whole tile, or the owner of a cut tile: wait for its contributors' partial sums
      const int ncontrib = (R.sk && sg.kb1 < nk) ? R.contributors(sg.tile, cl) : 0;
      epi_prefetch<KIND>(ep, row < M ? row : M - 1, n0, BN);  // while the MMAs run
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
      if (rope_rows && epi_normed(ep, n0)) epi_rope_load(ep, row < M ? row : M - 1, n0, rope_cur);
      bool ok = mbar_wait(&tfull[acc], aph, abort_flag, err, ERRBIT_TIMEOUT_GEMM);
      if (ncontrib > 0 && lane == 0 && ok) {
        const uint64_t t0 = globaltimer();
        while (ld_acquire(flag) < ncontrib) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          if (globaltimer() - t0 > FH_WAIT_LIMIT_NS) {
            *abort_flag = 1;
            if (err) atomicOr(err, ERRBIT_TIMEOUT_GEMM);
            ok = false;
            break;
          }
        }
        fence_proxy_async_global();
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // the contributors' boxes (32 rows x 32 columns each, box i = chunk * ncontrib + q) stream
      // into this warp's PBOX buffers in the ring (free: this owner segment is the share's last,
      // its MMAs are done), up to PBOX ahead of their use
      uint8_t* pbuf = smem + quarter * (S::PBOX * 4096);
      uint64_t* pb = pbar + quarter * S::PBOX;
      const int nbox = ncontrib * (BN / 32);
      auto issue_box = [&](int i) {
        const int q = i % ncontrib, ch = i / ncontrib;
        const int slot = i % S::PBOX;
        mbar_expect_tx(&pb[slot], 4096);
        tma_load_2d(&tmP, &pb[slot], pbuf + slot * 4096, ch * 32, ((cl + 1 + q) * 2 + (int)rank) * BM + quarter * 32);
      };
      int nissued = 0;  // boxes issued (lane 0) and waited for
      if (lane == 0)
        for (; nissued < nbox && nissued < S::PBOX; ++nissued) issue_box(nissued);
      int nwait = 0;
      bool pok = true;  // every box arrived in time
      // one 32-column chunk of the tile: contributors' partial sums, the epilogue, the store
      float ssq = 0.f;
      auto chunk = [&](float (&v)[32], int c) {
        if (rope_rows && c + 32 < BN && epi_normed(ep, n0 + c + 32))
          epi_rope_load(ep, row < M ? row : M - 1, n0 + c + 32, rope_nxt);
        // contributors' partial sums of these 32 columns, in k order
        for (int q = 0; q < ncontrib && pok; ++q, ++nwait) {
          const int slot = nwait % S::PBOX;
          pok = __all_sync(0xffffffffu,
                           mbar_wait(&pb[slot], (nwait / S::PBOX) & 1, abort_flag, err, ERRBIT_TIMEOUT_GEMM));
          if (!pok) break;
          const uint8_t* prow = pbuf + slot * 4096 + lane * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 pp = *reinterpret_cast<const float4*>(prow + ((j ^ (lane & 7)) << 4));
            v[4 * j] += pp.x;
            v[4 * j + 1] += pp.y;
            v[4 * j + 2] += pp.z;
            v[4 * j + 3] += pp.w;
          }
          __syncwarp();
          if (lane == 0 && nissued < nbox) issue_box(nissued++);  // its buffer has been read
        }
        if (row0 >= M) return;  // a warp with no row below M stores nothing
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
          // reading is the other buffer's
          uint8_t* box = stg + (nchunk & 1) * 4096;
          if (lane == 0) bulk_wait_read<1>();
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
        if ((c & 127) == 96 || c + 32 == BN) {  // the end of a 128-column group
          if (row < M) epi_group_end<KIND>(ep, row, n0 + (c & ~127), ssq);
          ssq = 0.f;
        }
        if constexpr (KIND == EPI_QKV) {
#pragma unroll
          for (int k = 0; k < 8; ++k) rope_cur[k] = rope_nxt[k];
        }
      };
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tb + c, v);
        tc_wait_ld();
        chunk(v, c);
      }
      if (!pok) {
        // boxes still in flight land before the CTA's shared memory can go away
        if (lane == 0)
          for (int i = nwait; i < nissued; ++i) drain_wait(&pb[i % S::PBOX], (i / S::PBOX) & 1);
        __syncwarp();
        break;
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (ncontrib > 0 && lane == 0) *flag = 0;  // its only reader is done: clear it for the next launch
    }
    if (lane == 0) {
      bulk_wait_all();  // every store issued by this warp has been performed
      if (KIND == EPI_RESID && ep.ln_out) fence_proxy_async_global();  // ... before the rows are read back
    }
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
  if constexpr (KIND == EPI_RESID) {
    if (ep.ln_out && N == 12 * 128) {
      // the next norm of the updated rows: wait until every CTA of the launch (all resident:
      // one cluster per CTA pair that fits) has added its tiles, then each warp normalises rows
      if (threadIdx.x == 0 && !*abort_flag) {
        __threadfence();
        atomicAdd(ep.ln_ctr, 1);
        const uint64_t t0 = globaltimer();
        while (ld_acquire(ep.ln_ctr) < (int)gridDim.x) {
          if (globaltimer() - t0 > FH_WAIT_LIMIT_NS) {
            *abort_flag = 1;
            if (err) atomicOr(err, ERRBIT_TIMEOUT_GEMM);
            break;
          }
        }
        __threadfence();
      }
      __syncwarp();  // warp 0 converged again before the CTA barrier
      __syncthreads();
      if (!*abort_flag) {
        const int nw = blockDim.x >> 5;
        for (int r = blockIdx.x * nw + warp; r < M; r += gridDim.x * nw) {
          const long mb = (long)(r / ep.rows_per_batch) * ep.ln_bstride;
          norm_row<bf16, 12>(ep.resid + (long)r * ep.ldr, reinterpret_cast<bf16*>(ep.ln_out) + (long)r * N, lane,
                             ep.ln_mode, ep.ln_a + mb, ep.ln_c + mb, ep.ln_eps);
        }
      }
    }
  }
}

// CTA pairs of the pair GEMM, and clusters of four of the split-K kernel, that can be
// resident at once, per device (set by gemm_tc_prepare): a stream-K owner waits for
// contributors with higher cluster indices, and a split-K cluster's pairs wait for each
// other, so every cluster of a launch must be able to run at the same time.
int g_pair_clusters[64] = {0};
int g_split_clusters[64] = {0};

// Clusters of a pair-GEMM launch: one per CTA pair that can be resident, or fewer when there
// is less work than that (stream-K: fewer k-blocks; whole tiles: fewer tiles).
inline int tc2_clusters(int M, int N, int K, int bn, int num_sms, bool sk) {
  const long tiles = (long)((M + 2 * BM - 1) / (2 * BM)) * (N / bn);
  const long units = sk ? tiles * ((K + BK - 1) / BK) : tiles;
  int dev = 0;
  cudaGetDevice(&dev);
  int cap = num_sms / 2;
  const int resident = dev >= 0 && dev < 64 ? g_pair_clusters[dev] : 0;
  if (resident > 0 && resident < cap) cap = resident;
  return units < cap ? (int)units : cap;
}

template <int BN, int KIND, typename OutT>
cudaError_t launch_tc2(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, const CUtensorMap& p, int M,
                       int N, int K, const EpiParams& ep, unsigned* err, int num_sms, cudaStream_t st) {
  using S = Tc2Shape<BN>;
  const int clusters = tc2_clusters(M, N, K, BN, num_sms, ep.sk_part != nullptr);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(192);
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
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<BN, KIND, OutT>, a, b, c, p, M, N, K, ep, err);
}

// ------------------------------------------------------------------ split-K over two CTA pairs
// GEMMs with few output tiles (M = 1280, N = 1536: 30 tiles of 256 x 256) run one tile per
// cluster of four CTAs. CTA pair s (cluster ranks 2s, 2s+1) computes the tile over half of
// the K range with cta_group::2 MMAs into its own TMEM accumulator, on 256-wide tiles whose
// operand traffic per MMA is the lowest the pair can have. The pairs then reduce-scatter
// through shared memory: each CTA finalises 128 of the 256 columns of its rows, receiving
// the partner pair's fp32 partial sums for them by one bulk copy per warp into its operand
// ring (free once its pair's MMAs are done), adding them to its own and running the staged
// epilogue. One tile per cluster: the host launches this only when the tiles fit the
// clusters of four that can be resident at once.
template <int BN, int KIND, typename OutT>
__global__ void __launch_bounds__(192, 1)
    gemm_tc2s_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, int M, int N, int K, EpiParams ep, unsigned* err) {
  using S = Tc2Shape<BN>;
  static_assert(KIND != EPI_QKV, "the head-major scatter runs on the plain pair kernel");
  static_assert(BN == 256, "each CTA finalises one 128-column group");
  constexpr uint32_t HALF_COLS = BN / 2;
  constexpr uint32_t QBYTES = HALF_COLS * 128;   // one quarter's rows of half the columns, fp32
  constexpr uint32_t RX = 4 * QBYTES;            // ring offset of the partner's half
  static_assert(2 * RX <= S::RING_BYTES, "both halves must fit in the operand ring");
  using StageT = typename std::conditional<KIND == EPI_RESID, float, OutT>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::RING_BYTES + S::STG_BYTES);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* ring_free = tfull + 1;       // the partner's MMAs are done: its ring may be written
  uint64_t* part_ready = ring_free + 1;  // [4] the partner's half of a quarter's rows has landed
  uint64_t* done = part_ready + 4;   // every other CTA of the cluster is finished with this one
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
    for (int q = 0; q < 4; ++q) mbar_init(&part_ready[q], 1);
    mbar_init(done, 3);
    *abort_flag = 0;
    fence_mbar_init();
    // each quarter's rows of the columns this CTA finalises arrive as one bulk copy
    for (int q = 0; q < 4; ++q) mbar_expect_tx(&part_ready[q], QBYTES);
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
        if (half == 0) mbar_expect_tx(&full[s], S::TX_BYTES);
        tma_load_2d_pair(&tmB, mapa_shared(smem_u32(&full[s]), lead), smem + s * S::STAGE_BYTES + S::A_BYTES,
                         (kb0 + s) * BK, n0 + (int)half * S::BNH);
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
          if (half == 0) mbar_expect_tx(&full[stage], S::TX_BYTES);
          tma_load_2d_pair(&tmB, bar, sa + S::A_BYTES, kb * BK, n0 + (int)half * S::BNH);
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
        const uint32_t b_addr = a_addr + S::A_BYTES;
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
    // the 16-byte pieces of each row swizzled by row, and one bulk copy per warp moves it
    // into the partner's ring at offset RX once the partner's MMAs are done with it.
    const uint32_t partner = rank ^ 2u;
    const int mine = (int)split * (int)HALF_COLS, theirs = (int)HALF_COLS - mine;
    if (ok && quarter == 0 && lane == 0) mbar_arrive_release_cluster(mapa_shared(smem_u32(ring_free), partner));
    epi_prefetch<KIND>(ep, row < M ? row : M - 1, n0 + mine, HALF_COLS);
    if (ok && row0 < M) {
      uint8_t* out = smem + quarter * QBYTES;
      auto put = [&](const float (&v)[32], int c) {
        uint8_t* prow = out + (c >> 5) * 4096 + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(prow + ((j ^ (lane & 7)) << 4)) =
              make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      };
#pragma unroll 1
      for (int c = 0; c < (int)HALF_COLS; c += 32) {
        float v[32];
        tmem_ld32(tb + theirs + c, v);
        tc_wait_ld();
        put(v, c);
      }
      fence_proxy_async_smem();
      __syncwarp();
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(ring_free, 0, abort_flag, err, ERRBIT_TIMEOUT_GEMM));
      if (ok && lane == 0)
        bulk_copy_to_cluster(mapa_shared(smem_u32(smem + RX + quarter * QBYTES), partner), out, QBYTES,
                             mapa_shared(smem_u32(&part_ready[quarter]), partner));
      if (ok) ok = __all_sync(0xffffffffu,
                              mbar_wait_cluster(&part_ready[quarter], 0, abort_flag, err, ERRBIT_TIMEOUT_GEMM));
    }
    // the finalised half: own accumulator + the partner's, then the staged epilogue
    const uint8_t* part = smem + RX + quarter * QBYTES;
    uint8_t* stg = smem + S::RING_BYTES + quarter * 8192;
    uint32_t nchunk = 0;
    if (ok && row0 < M) {
      float ssq = 0.f;
      auto chunk = [&](float (&v)[32], int c) {
        const int col = n0 + mine + c;
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
      };
#pragma unroll 1
      for (int c = 0; c < (int)HALF_COLS; c += 32) {
        float v[32];
        tmem_ld32(tb + mine + c, v);
        tc_wait_ld();
        chunk(v, c);
      }
      if (row < M) epi_group_end<KIND>(ep, row, n0 + mine, ssq);
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
  using S = Tc2Shape<BN>;
  const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * (N / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4 * tiles);
  cfg.blockDim = dim3(192);
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
                              (int)Tc2Shape<BN>::SMEM);
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
  cfg.blockDim = dim3(192);
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

cudaError_t gemm_tc(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap* c, const CUtensorMap* p, int M,
                    int N, int K, int bn, int kind, bool out_bf16, const EpiParams& ep, unsigned* err, int num_sms,
                    cudaStream_t st, bool pair) {
  // the CTA-pair kernels store their epilogue through the output map `c`, and stream-K moves
  // partial sums through `p`
  if (pair && !c) return cudaErrorInvalidValue;
  if (pair && ep.sk_part && (!p || !ep.sk_flags)) return cudaErrorInvalidValue;
  const CUtensorMap& cm = c ? *c : a;
  const CUtensorMap& pm = p ? *p : cm;
  // few 256 x 256 tiles (one per cluster of four fits the GPU), whole tiles asked for: split K
  // over two CTA pairs of a cluster
  const int tiles256 = ((M + 2 * BM - 1) / (2 * BM)) * (N / 256);
  int dev = 0;
  cudaGetDevice(&dev);
  const int resident4 = dev >= 0 && dev < 64 ? g_split_clusters[dev] : 0;
  if (pair && !ep.sk_part && !ep.ln_out && bn == 256 && N <= 4096 && 4 * tiles256 <= num_sms &&
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
    return pair ? launch_tc2<BNV, KV, OT>(a, b, cm, pm, M, N, K, ep, err, num_sms, st)              \
                : launch_tc<BNV, KV, OT>(a, b, M, N, K, ep, err, num_sms, st);
  if (pair && bn == 224) {  // FFN1-shaped (8960 = 40 x 224 balances the waves)
    if (kind == EPI_GELU && out_bf16)
      return launch_tc2<224, EPI_GELU, bf16>(a, b, cm, pm, M, N, K, ep, err, num_sms, st);
    if (kind == EPI_STORE && !out_bf16)
      return launch_tc2<224, EPI_STORE, float>(a, b, cm, pm, M, N, K, ep, err, num_sms, st);
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
