// api.cu - the C ABI (include/fh.h, include/fh_ops.h) and the host runtime of the
// FlashHead Lite DiT: weight arena and seeded generation, workspace plan, TMA
// descriptors, the launch sequences of a block / a flow prediction / the slice
// sampler, and CUDA-graph capture of the sampler's step loop.
//
// The model follows gizai:flashhead (gizstack API reference): Functions > load
// binds a model to one GPU; Types > FlashHead lists its Linear layers, per-step
// headMods, the [1280, 768] rotary tables and the `work: Scratch` arena, which here
// is the caller-owned workspace; Methods > talk runs slice by slice. The launch
// sequence of one block is the Wan-style adaLN block of readings R1-R11.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "epilogue.cuh"
#include "fh.h"
#include "fh_ops.h"
#include "kernels.h"

using namespace fh;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define CK(call)                                                                                    \
  do {                                                                                              \
    cudaError_t e_ = (call);                                                                        \
    if (e_ != cudaSuccess) return fail(FH_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                                       __FILE__, __LINE__);                                          \
  } while (0)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool load_encode() {
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return true;
}

// 2D bf16 view [rows, cols] (cols contiguous), box 64 x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D view [rows, cols] with row pitch `ld` elements for the GEMM epilogue's TMA stores:
// box 32 x 32, fp32 with the 128-byte swizzle or bf16 with the 64-byte swizzle.
bool make_out_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, bool f32) {
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * es};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 view [d2][d1][d0] (d0 contiguous), box box0 x box1 x 1, 128-byte swizzle.
bool make_map_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                 uint32_t box1) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d1 * d0 * 2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 view of the head-major q/k/v workspace [planes = 3 * B * heads][L][128], box
// 32 x 32 x 1 with the 64-byte swizzle
bool make_qkv_map(CUtensorMap* map, const void* base, uint64_t L, uint64_t planes) {
  cuuint64_t dims[3] = {128, L, planes};
  cuuint64_t strides[2] = {128 * 2, L * 128 * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// output map of a CTA-pair GEMM epilogue
bool epi_out_map(CUtensorMap* map, int kind, bool out_bf16, const EpiParams& ep, int M, int N) {
  if (kind == EPI_QKV)
    return out_bf16 && make_qkv_map(map, ep.out, ep.rows_per_batch,
                                    3ull * (M / ep.rows_per_batch) * (ep.dim >> 7));
  if (kind == EPI_RESID) return make_out_map(map, ep.resid, M, N, ep.ldr, true);
  return make_out_map(map, ep.out, M, N, ep.ldo, !out_bf16);
}

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Tile shape per GEMM, from the weight's N and K. Deep projections (K >= 1024, N >= 1536:
// QKV, O-proj, cross-Q/O, FFN1, FFN2) run as 256-row tiles on CTA pairs (cta_group::2),
// each CTA streaming half of the W tile, 256 columns wide where N allows (the widest tile
// a pair accumulates, the least operand traffic per MMA); the rest (patch embed K = 256,
// head N = 128, the per-slice cross-KV with 160 rows) on single CTAs.
struct TileCfg {
  int bn;
  bool pair;
  int wbox;  // rows of the W tile each CTA loads
};
TileCfg tile_cfg(int N, int K, bool pair_ok = true) {
  TileCfg t;
  t.pair = pair_ok && K >= 1024 && N >= 1536 && N <= 16384;
  // 256 wide for the cross-KV (single CTAs), for QKV (N = 4608: the pair's operand bytes per
  // MMA, not its MMA rate, bound these main loops) and for the pair GEMMs of width up to 4096
  // (O-proj, cross-Q/O, FFN2), which then run split-K on clusters of four when their 256 x 256
  // tiles are few
  t.bn = (N % 256 == 0 && (N >= 4608 || (t.pair && N <= 4096))) ? 256 : 128;
  // FFN1 (N = 8960 = 40 x 224): at 1280 tokens 200 pair tiles of width 224 fill three rounds
  // of 74 CTA pairs better than 175 tiles of width 256
  if (t.pair && N >= 8192 && N % 224 == 0) t.bn = 224;
  t.wbox = t.pair ? t.bn / 2 : t.bn;
  return t;
}

// The audio projection's fixed sizes: the speech encoder's window (8 s at 25 states/s, 12
// layers of 768, wav2vec 2.0 base), 5 states per video frame, 8 video frames per latent
// frame after the first, hidden width 512 (readings of gizai:flashhead's opening paragraph).
constexpr int AU_STATES = 200, AU_LAYERS = 12, AU_CH = 768, AU_WIN = 5, AU_STRIDE = 8, AU_HID = 512;
constexpr int AU_PER_STATE = AU_LAYERS * AU_CH;
constexpr int AU_GROUP = AU_STRIDE + AU_WIN - 1;
constexpr int AU_K0 = AU_WIN * AU_PER_STATE, AU_KV = AU_GROUP * AU_PER_STATE;

struct TensorRec {
  int tid;
  void* ptr;
  long rows, cols, ld;
  bool mat;  // stored in the model dtype (else float32)
  int kind;  // 0: z / sqrt(fan), 1: 1 + 0.1 z, 2: 0.1 z
  int fan;
};

struct BlockW {
  void *wqkv, *wo, *wcq, *wco, *w1, *w2;
  float *bqkv, *gqkv, *bo, *bcq, *gcq, *bco, *ln3w, *ln3b, *b1, *b2;
  CUtensorMap m_qkv, m_o, m_cq, m_co, m_1, m_2, m_ckv;
};

struct WsLayout {
  size_t x, h, qkv, ssq_qk, attn, cq, ssq_cq, ckv, ssq_ckv, u, tok, lat, v, mods, hmods, tsin, thid, te, te0, audio,
      in_noise, in_ref, in_motion, out, au_win0, au_winv, au_part, au_h1, au_h2,
      au_tok, total;
};

struct Plan {
  void* ws = nullptr;
  int batch = 0;
  WsLayout lay{};
  CUtensorMap m_h, m_attn, m_u, m_tok, m_audio, m_q, m_k, m_v;
  CUtensorMap m_xq, m_xkv, m_xo;  // cross-attention: queries and output per frame, keys/values
};

struct GraphEntry {
  void* ws;
  const float* eps;  // the re-noising sampler's draws (null: Euler)
  int batch, nsteps, timing;
  std::vector<float> sigmas;
  cudaGraphExec_t exec;
  int launches;
  std::vector<int> ev_pairs;  // indices of event pairs recorded in this graph
};

}  // namespace

struct fh_dit {
  fh_config cfg;
  int device = 0, num_sms = 148;
  bool bf16 = true;
  int D, NH, FF, NB, C, F, HW, L, A;
  uint64_t seed;
  void* arena = nullptr;
  size_t arena_bytes = 0;
  std::vector<BlockW> blk;
  void* wckv = nullptr;
  float *bckv = nullptr, *gckv = nullptr, *modtab = nullptr;
  void *patch_w = nullptr, *head_w = nullptr, *t_w1 = nullptr, *t_w2 = nullptr, *t_wp = nullptr;
  float *patch_b = nullptr, *head_b = nullptr, *head_mod = nullptr, *t_b1 = nullptr, *t_b2 = nullptr,
        *t_bp = nullptr;
  float2* rope = nullptr;
  // audio projection: proj1 [HID, K0], proj1vf [HID, KV], proj2 [HID, HID], proj3 [32 D, HID]
  void *a_w1 = nullptr, *a_w1v = nullptr, *a_w2 = nullptr, *a_w3 = nullptr;
  float *a_b1 = nullptr, *a_b1v = nullptr, *a_b2 = nullptr, *a_b3 = nullptr, *a_nw = nullptr, *a_nb = nullptr;
  CUtensorMap m_ckv_all, m_patch, m_head;
  std::vector<TensorRec> recs;
  unsigned* err_host = nullptr;
  unsigned* err_dev = nullptr;
  Plan plan;
  std::vector<GraphEntry> graphs;
  cudaStream_t cap = nullptr;
  int launches = 0, last_launches = 0;
  // timing of one kernel class inside the sampler graph
  int timing = 0;
  std::vector<cudaEvent_t> events;
  int ev_used = 0;
  bool capturing = false;
  std::vector<int> last_pairs;
};

namespace {

size_t elt(const fh_dit* m) { return m->bf16 ? 2 : 4; }

WsLayout layout(const fh_dit* m, int B) {
  WsLayout w{};
  const size_t M = (size_t)B * m->L, Ma = (size_t)B * m->F * m->A, e = elt(m);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t r = o;
    o += al256(bytes);
    return r;
  };
  w.x = take(M * m->D * 4);
  w.h = take(M * m->D * e);
  w.qkv = take(3 * M * m->D * e);
  w.ssq_qk = take(M * 2 * m->NH * 4);
  w.attn = take(M * m->D * e);
  w.cq = take(M * m->D * e);
  w.ssq_cq = take(M * m->NH * 4);
  w.ckv = take(Ma * (size_t)m->NB * 2 * m->D * e);
  w.ssq_ckv = take(Ma * (size_t)m->NB * 2 * m->NH * 4);
  w.u = take(M * m->FF * e);
  w.tok = take(M * 2 * m->C * e);
  w.lat = take(M * m->C * 4);
  w.v = take(M * m->C * 4);
  w.mods = take((size_t)B * m->NB * 6 * m->D * 4);
  w.hmods = take((size_t)B * 2 * m->D * 4);
  w.tsin = take((size_t)B * 256 * 4);
  w.thid = take((size_t)B * m->D * 4);
  w.te = take((size_t)B * m->D * 4);
  w.te0 = take((size_t)B * 6 * m->D * 4);
  w.audio = take(Ma * m->D * e);
  w.in_noise = take((size_t)B * m->C * m->L * 4);
  w.in_ref = take((size_t)B * m->C * m->L * 4);
  w.in_motion = take((size_t)B * m->C * 2 * m->HW * 4);
  w.out = take((size_t)B * m->C * m->L * 4);
  // audio projection: the gathered states, split-K partial sums, hidden rows, fp32 tokens
  {
    const size_t R = (size_t)B * m->F, HID = AU_HID, TN = (size_t)m->A * m->D;
    w.au_win0 = take((size_t)B * AU_K0 * 4);
    w.au_winv = take((size_t)B * (m->F - 1) * AU_KV * 4);
    size_t part = (size_t)audio_gemv_chunks(AU_K0) * B * HID;
    part = std::max(part, (size_t)audio_gemv_chunks(AU_KV) * B * (m->F - 1) * HID);
    part = std::max(part, R * std::max(HID, TN));
    w.au_part = take(part * 4);
    w.au_h1 = take(R * HID * 4);
    w.au_h2 = take(R * HID * 4);
    w.au_tok = take(R * TN * 4);
  }
  w.total = o;
  return w;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(reinterpret_cast<uint8_t*>(ws) + off);
}

int get_plan(fh_dit* m, void* ws, int B, Plan** out) {
  Plan& p = m->plan;
  if (p.ws == ws && p.batch == B) {
    *out = &p;
    return FH_OK;
  }
  p.ws = ws;
  p.batch = B;
  p.lay = layout(m, B);
  if (m->bf16) {
    const WsLayout& w = p.lay;
    const uint64_t M = (uint64_t)B * m->L;
    bool ok = make_map(&p.m_h, at<void>(ws, w.h), M, m->D, 128) &&
              make_map(&p.m_attn, at<void>(ws, w.attn), M, m->D, 128) &&
              make_map(&p.m_u, at<void>(ws, w.u), M, m->FF, 128) &&
              make_map(&p.m_tok, at<void>(ws, w.tok), M, 2 * m->C, 128) &&
              make_map(&p.m_audio, at<void>(ws, w.audio), (uint64_t)B * m->F * m->A, m->D, 128);
    const uint64_t rows = (uint64_t)B * m->NH * m->L;
    const size_t sec = (size_t)M * m->D * 2;
    ok = ok && make_map(&p.m_q, at<void>(ws, w.qkv), rows, 128, 128) &&
         make_map(&p.m_k, at<void>(ws, w.qkv + sec), rows, 128, 128) &&
         make_map(&p.m_v, at<void>(ws, w.qkv + 2 * sec), rows, 128, 128);
    const uint64_t HW = m->L / m->F, frames = (uint64_t)B * m->F;
    ok = ok && make_map_3d(&p.m_xq, at<void>(ws, w.cq), m->D, HW, frames, 64, 128) &&
         make_map_3d(&p.m_xo, at<void>(ws, w.attn), m->D, HW, frames, 64, 32) &&
         make_map(&p.m_xkv, at<void>(ws, w.ckv), frames * m->A, (uint64_t)m->NB * 2 * m->D, 32);
    if (!ok) {
      p.ws = nullptr;
      return fail(FH_ERR_CUDA, "tensor map encoding failed for the workspace");
    }
  }
  *out = &p;
  return FH_OK;
}

// ------------------------------------------------------------ launch helpers
int timed_begin(fh_dit* m, int cls, cudaStream_t st) {
  if (!m->capturing || m->timing == 0 || cls != m->timing) return -1;
  if (m->ev_used + 2 > (int)m->events.size()) return -1;
  const int i = m->ev_used;
  m->ev_used += 2;
  cudaEventRecordWithFlags(m->events[i], st, cudaEventRecordExternal);
  return i;
}
void timed_end(fh_dit* m, int i, cudaStream_t st) {
  if (i < 0) return;
  cudaEventRecordWithFlags(m->events[i + 1], st, cudaEventRecordExternal);
  m->last_pairs.push_back(i);
}

int run_gemm(fh_dit* m, const CUtensorMap* amap, const void* A, long lda, const CUtensorMap* bmap, const void* W,
             long ldw, int M, int N, int K, int kind, bool out_bf16, const EpiParams& ep, cudaStream_t st,
             int tclass) {
  const int ti = timed_begin(m, tclass, st);
  cudaError_t e;
  if (m->bf16) {
    const TileCfg tc = tile_cfg(N, K);
    CUtensorMap cmap;
    if (tc.pair && !epi_out_map(&cmap, kind, out_bf16, ep, M, N)) {
      timed_end(m, ti, st);
      return fail(FH_ERR_CUDA, "tensor map encoding failed for a GEMM output");
    }
    e = gemm_tc(*amap, *bmap, tc.pair ? &cmap : nullptr, M, N, K, tc.bn, kind, out_bf16, ep, m->err_dev,
                m->num_sms, st, tc.pair);
  } else {
    e = gemm_simt(reinterpret_cast<const float*>(A), lda, reinterpret_cast<const float*>(W), ldw, M, N, K, kind,
                  ep, st);
  }
  timed_end(m, ti, st);
  m->launches++;
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "gemm launch (M=%d N=%d K=%d kind=%d): %s", M, N, K, kind,
                                    cudaGetErrorString(e));
  return FH_OK;
}

EpiParams epi0(int L) {
  EpiParams p;
  memset(&p, 0, sizeof p);
  p.rows_per_batch = L;
  p.norm_period = 1 << 30;
  p.norm_count = 0;
  return p;
}

#define RUN(x)          \
  do {                  \
    int r_ = (x);       \
    if (r_) return r_;  \
  } while (0)
#define LAUNCH(x)                                                                                    \
  do {                                                                                               \
    cudaError_t e_ = (x);                                                                            \
    m->launches++;                                                                                   \
    if (e_ != cudaSuccess) return fail(FH_ERR_CUDA, "%s: %s", #x, cudaGetErrorString(e_));           \
  } while (0)

// time conditioning for per-stream timesteps tv -> mods [B, NB, 6, D], hmods [B, 2, D]
int run_time_cond(fh_dit* m, Plan& P, TVals tv, cudaStream_t st) {
  const WsLayout& w = P.lay;
  void* ws = P.ws;
  const int B = P.batch;
  LAUNCH(time_sinusoid(at<float>(ws, w.tsin), B, tv, 256, st));
  if (m->bf16) {
    LAUNCH(gemv<bf16>((const bf16*)m->t_w1, at<float>(ws, w.tsin), m->t_b1, at<float>(ws, w.thid), m->D, 256, B, 0,
                      1, st));
    LAUNCH(gemv<bf16>((const bf16*)m->t_w2, at<float>(ws, w.thid), m->t_b2, at<float>(ws, w.te), m->D, m->D, B, 0,
                      0, st));
    LAUNCH(gemv<bf16>((const bf16*)m->t_wp, at<float>(ws, w.te), m->t_bp, at<float>(ws, w.te0), 6 * m->D, m->D, B,
                      1, 0, st));
  } else {
    LAUNCH(gemv<float>((const float*)m->t_w1, at<float>(ws, w.tsin), m->t_b1, at<float>(ws, w.thid), m->D, 256, B,
                       0, 1, st));
    LAUNCH(gemv<float>((const float*)m->t_w2, at<float>(ws, w.thid), m->t_b2, at<float>(ws, w.te), m->D, m->D, B,
                       0, 0, st));
    LAUNCH(gemv<float>((const float*)m->t_wp, at<float>(ws, w.te), m->t_bp, at<float>(ws, w.te0), 6 * m->D, m->D,
                       B, 1, 0, st));
  }
  LAUNCH(assemble_mods(m->modtab, at<float>(ws, w.te0), m->head_mod, at<float>(ws, w.te), at<float>(ws, w.mods),
                       at<float>(ws, w.hmods), B, m->NB, m->D, st));
  return FH_OK;
}

// cross-attention keys/values of blocks [k0, k0 + nb) from the staged audio tokens
int run_cross_kv(fh_dit* m, Plan& P, int k0, int nb, cudaStream_t st) {
  const WsLayout& w = P.lay;
  void* ws = P.ws;
  const int Ma = P.batch * m->F * m->A;
  const long ldkv = (long)m->NB * 2 * m->D;
  EpiParams ep = epi0(1 << 30);
  ep.bias = m->bckv + (long)k0 * 2 * m->D;
  ep.gain = m->gckv + (long)k0 * 2 * m->D;
  ep.out = at<uint8_t>(ws, w.ckv) + (size_t)k0 * 2 * m->D * elt(m);
  ep.ldo = ldkv;
  ep.ssq = at<float>(ws, w.ssq_ckv) + (long)k0 * 2 * m->NH;
  ep.ssq_ld = m->NB * 2 * m->NH;
  ep.norm_period = 2 * m->D;
  ep.norm_count = m->D;
  const CUtensorMap* bm = nb == m->NB ? &m->m_ckv_all : &m->blk[k0].m_ckv;
  const void* W = reinterpret_cast<const uint8_t*>(m->wckv) + (size_t)k0 * 2 * m->D * m->D * elt(m);
  return run_gemm(m, &P.m_audio, at<void>(ws, w.audio), m->D, bm, W, m->D, Ma, nb * 2 * m->D, m->D, EPI_NORM,
                  m->bf16, ep, st, 0);
}

// One block on the residual x.
template <typename T>
int run_block(fh_dit* m, Plan& P, int k, float* x, cudaStream_t st) {
  const WsLayout& w = P.lay;
  void* ws = P.ws;
  const int B = P.batch, L = m->L, D = m->D, NH = m->NH;
  const int M = B * L;
  const long mbs = (long)m->NB * 6 * D;
  const float* mods = at<float>(ws, w.mods) + (long)k * 6 * D;
  BlockW& bw = m->blk[k];
  T* h = at<T>(ws, w.h);
  T* attn = at<T>(ws, w.attn);
  T* qkv = at<T>(ws, w.qkv);
  float* ssq_qk = at<float>(ws, w.ssq_qk);
  const float eps = m->cfg.eps;

  // self-attention branch
  {
    const int ti = timed_begin(m, 6, st);
    cudaError_t e = norm_rows<T>(x, h, M, D, L, 0, mods + 0 * D, mods + 1 * D, mbs, nullptr, nullptr, eps, st);
    timed_end(m, ti, st);
    LAUNCH(e);
  }
  {
    EpiParams ep = epi0(L);
    ep.bias = bw.bqkv;
    ep.gain = bw.gqkv;
    ep.out = qkv;
    ep.ssq = ssq_qk;
    ep.ssq_ld = 2 * NH;
    ep.norm_period = 3 * D;
    ep.norm_count = 2 * D;
    ep.rope = m->rope;
    ep.dim = D;
    ep.sec_stride = (long)M * D;
    RUN(run_gemm(m, &P.m_h, h, D, &bw.m_qkv, bw.wqkv, D, M, 3 * D, D, EPI_QKV, m->bf16, ep, st, 3));
  }
  {
    const int ti = timed_begin(m, 4, st);
    cudaError_t e;
    if (m->bf16)
      e = attn_tc(P.m_q, P.m_k, P.m_v, ssq_qk, 2 * NH, B, NH, L, eps, (bf16*)attn, m->err_dev, st);
    else
      e = attn_simt<float>((const float*)qkv, (const float*)qkv + (long)M * D, (const float*)qkv + 2L * M * D,
                           ssq_qk, 2 * NH, B, NH, L, eps, (float*)attn, st);
    timed_end(m, ti, st);
    LAUNCH(e);
  }
  {
    // O-proj + gated residual, then the learned-affine LayerNorm before the cross-attention (R7)
    EpiParams ep = epi0(L);
    ep.bias = bw.bo;
    ep.resid = x;
    ep.ldr = D;
    ep.gate = mods + 2 * D;
    ep.gate_bstride = mbs;
    RUN(run_gemm(m, &P.m_attn, attn, D, &bw.m_o, bw.wo, D, M, D, D, EPI_RESID, m->bf16, ep, st, 1));
  }
  // audio cross-attention branch
  LAUNCH(norm_rows<T>(x, h, M, D, L, 1, nullptr, nullptr, 0, bw.ln3w, bw.ln3b, eps, st));
  {
    EpiParams ep = epi0(L);
    ep.bias = bw.bcq;
    ep.gain = bw.gcq;
    ep.out = at<T>(ws, w.cq);
    ep.ldo = D;
    ep.ssq = at<float>(ws, w.ssq_cq);
    ep.ssq_ld = NH;
    ep.norm_period = D;
    ep.norm_count = D;
    RUN(run_gemm(m, &P.m_h, h, D, &bw.m_cq, bw.wcq, D, M, D, D, EPI_NORM, m->bf16, ep, st, 7));
  }
  {
    const int ti = timed_begin(m, 5, st);
    cudaError_t e =
        m->bf16 ? xattn_tc(P.m_xq, P.m_xkv, P.m_xo, at<float>(ws, w.ssq_cq), at<float>(ws, w.ssq_ckv),
                           m->NB * 2 * NH, k * 2 * NH, k * 2 * D, k * 2 * D + D, B, NH, L, m->F, m->A, eps, m->err_dev,
                           st)
                : cross_attn<T>(at<T>(ws, w.cq), at<float>(ws, w.ssq_cq), at<T>(ws, w.ckv), (long)m->NB * 2 * D,
                                k * 2 * D, k * 2 * D + D, at<float>(ws, w.ssq_ckv), m->NB * 2 * NH, k * 2 * NH, B,
                                NH, L, m->F, m->A, eps, attn, st);
    timed_end(m, ti, st);
    LAUNCH(e);
  }
  {
    // cross-O + residual, then the FFN's LayerNorm and modulation
    EpiParams ep = epi0(L);
    ep.bias = bw.bco;
    ep.resid = x;
    ep.ldr = D;
    RUN(run_gemm(m, &P.m_attn, attn, D, &bw.m_co, bw.wco, D, M, D, D, EPI_RESID, m->bf16, ep, st, 1));
  }
  // FFN branch
  LAUNCH(norm_rows<T>(x, h, M, D, L, 0, mods + 3 * D, mods + 4 * D, mbs, nullptr, nullptr, eps, st));
  {
    EpiParams ep = epi0(L);
    ep.bias = bw.b1;
    ep.out = at<T>(ws, w.u);
    ep.ldo = m->FF;
    RUN(run_gemm(m, &P.m_h, h, D, &bw.m_1, bw.w1, D, M, m->FF, D, EPI_GELU, m->bf16, ep, st, 2));
  }
  {
    EpiParams ep = epi0(L);
    ep.bias = bw.b2;
    ep.resid = x;
    ep.ldr = D;
    ep.gate = mods + 5 * D;
    ep.gate_bstride = mbs;
    RUN(run_gemm(m, &P.m_u, at<T>(ws, w.u), m->FF, &bw.m_2, bw.w2, m->FF, M, D, m->FF, EPI_RESID, m->bf16, ep, st,
                 1));
  }
  return FH_OK;
}

// patch embed -> blocks -> output norm -> head; input tok, output v [B*L, C] float32
template <typename T>
int run_network(fh_dit* m, Plan& P, cudaStream_t st) {
  const WsLayout& w = P.lay;
  void* ws = P.ws;
  const int B = P.batch, L = m->L, D = m->D, C = m->C;
  const int M = B * L;
  float* x = at<float>(ws, w.x);
  {
    EpiParams ep = epi0(L);
    ep.bias = m->patch_b;
    ep.out = x;
    ep.ldo = D;
    RUN(run_gemm(m, &P.m_tok, at<T>(ws, w.tok), 2 * C, &m->m_patch, m->patch_w, 2 * C, M, D, 2 * C, EPI_STORE,
                 false, ep, st, 0));
  }
  float* hm = at<float>(ws, w.hmods);
  for (int k = 0; k < m->NB; ++k) RUN(run_block<T>(m, P, k, x, st));
  // the output norm with its modulation (R9)
  LAUNCH(norm_rows<T>(x, at<T>(ws, w.h), M, D, L, 2, hm, hm + D, 2L * D, nullptr, nullptr, m->cfg.eps, st));
  {
    EpiParams ep = epi0(L);
    ep.bias = m->head_b;
    ep.out = at<float>(ws, w.v);
    ep.ldo = C;
    RUN(run_gemm(m, &P.m_h, at<T>(ws, w.h), D, &m->m_head, m->head_w, D, M, C, D, EPI_STORE, false, ep, st, 0));
  }
  return FH_OK;
}

template <typename T>
int run_sampler_steps(fh_dit* m, Plan& P, const float* sig, int nsteps, const float* eps, cudaStream_t st) {
  const WsLayout& w = P.lay;
  RUN(run_cross_kv(m, P, 0, m->NB, st));
  const size_t draw = (size_t)P.batch * m->C * m->L;  // floats per step of the re-noising draws
  for (int s = 0; s < nsteps; ++s) {
    TVals tv;
    for (int b = 0; b < 8; ++b) tv.t[b] = sig[s];
    RUN(run_time_cond(m, P, tv, st));
    RUN(run_network<T>(m, P, st));
    if (eps)
      LAUNCH(renoise_step<T>(at<float>(P.ws, w.lat), at<float>(P.ws, w.v), eps + s * draw, sig[s], sig[s + 1],
                             2 * m->HW, at<T>(P.ws, w.tok), P.batch, m->C, m->L, st));
    else
      LAUNCH(euler_step<T>(at<float>(P.ws, w.lat), at<float>(P.ws, w.v), sig[s + 1] - sig[s], 2 * m->HW,
                           at<T>(P.ws, w.tok), P.batch, m->C, m->L, st));
  }
  return FH_OK;
}

int check_err_word(fh_dit* m) {
  unsigned e = *reinterpret_cast<volatile unsigned*>(m->err_host);
  if (e) {
    *m->err_host = 0;
    return fail(FH_ERR_TIMEOUT, "a kernel's bounded wait ran out (error bits 0x%x)", e);
  }
  return FH_OK;
}

int common_checks(fh_dit* m, int batch, void* ws) {
  if (!m) return fail(FH_ERR_ARG, "null model");
  if (batch < 1 || batch > m->cfg.max_batch) return fail(FH_ERR_SHAPE, "batch %d outside [1, %d]", batch,
                                                         m->cfg.max_batch);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return fail(FH_ERR_ARG, "workspace null or not 256-byte aligned");
  if (cudaSetDevice(m->device) != cudaSuccess) return fail(FH_ERR_CUDA, "cudaSetDevice(%d) failed", m->device);
  return check_err_word(m);
}

// kernels with more than 48 KB of dynamic shared memory need an attribute set per device,
// outside any stream capture; done once per device (ordinals below 64), under a lock so that
// first calls from several threads do not race on it
std::mutex g_prepare_mu;
bool g_prepared[64] = {};
int prepare_device(int dev) {
  if (dev < 0 || dev >= 64) return fail(FH_ERR_UNSUPPORTED, "device ordinal %d outside [0, 64)", dev);
  std::lock_guard<std::mutex> lock(g_prepare_mu);
  if (g_prepared[dev]) return FH_OK;
  cudaError_t e = gemm_tc_prepare();
  if (e == cudaSuccess) e = attn_tc_prepare();
  if (e == cudaSuccess) e = cross_attn_prepare();
  if (e == cudaSuccess) e = xattn_tc_prepare();
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "kernel attribute setup: %s", cudaGetErrorString(e));
  g_prepared[dev] = true;
  return FH_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* fh_last_error(void) { return g_err.c_str(); }

int fh_dit_create(const fh_config* cfg, uint64_t seed, void* stream, fh_dit** out) {
  if (!cfg || !out) return fail(FH_ERR_ARG, "null argument");
  *out = nullptr;
  const fh_config& c = *cfg;
  if (c.head_dim != 128 || c.heads * c.head_dim != c.dim || c.dim % 128 || c.ffn % 128 || c.latent_ch % 64 ||
      c.frames < 2 || c.lat_h < 1 || c.lat_w < 1 || c.blocks < 1 || c.audio_tokens != 32 || c.max_batch < 1 ||
      c.max_batch > 8 || c.rope_split[0] % 2 || c.rope_split[1] % 2 || c.rope_split[2] % 2 ||
      c.rope_split[0] + c.rope_split[1] + c.rope_split[2] != c.head_dim || (c.dtype != FH_F32 && c.dtype != FH_BF16) ||
      c.dim / 128 > 16 || c.dim > 1536 * 4)
    return fail(FH_ERR_SHAPE, "configuration outside the supported set");
  const int L = c.frames * c.lat_h * c.lat_w;
  if (L > 8192) return fail(FH_ERR_SHAPE, "token count %d above 8192", L);
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || c.device < 0 || c.device >= ndev)
    return fail(FH_ERR_UNSUPPORTED, "no CUDA device %d", c.device);
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, c.device) != cudaSuccess) return fail(FH_ERR_CUDA, "device query failed");
  if (prop.major != 10 || prop.minor != 0)
    return fail(FH_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100 (B200) only", c.device,
                prop.major, prop.minor);
  if (cudaSetDevice(c.device) != cudaSuccess) return fail(FH_ERR_CUDA, "cudaSetDevice failed");
  if (!load_encode()) return fail(FH_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled unavailable");
  RUN(prepare_device(c.device));

  fh_dit* m = new fh_dit();
  m->cfg = c;
  m->device = c.device;
  m->num_sms = prop.multiProcessorCount;
  m->bf16 = c.dtype == FH_BF16;
  m->D = c.dim;
  m->NH = c.heads;
  m->FF = c.ffn;
  m->NB = c.blocks;
  m->C = c.latent_ch;
  m->F = c.frames;
  m->HW = c.lat_h * c.lat_w;
  m->L = L;
  m->A = c.audio_tokens;
  m->seed = seed;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t e = elt(m);
  const long D = m->D, FF = m->FF, NB = m->NB, C = m->C;

  // ---- arena layout
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t r = off;
    off += al256(bytes);
    return r;
  };
  struct BO {
    size_t wqkv, wo, wcq, wco, w1, w2, bqkv, gqkv, bo, bcq, gcq, bco, ln3w, ln3b, b1, b2;
  };
  std::vector<BO> bo(NB);
  for (long k = 0; k < NB; ++k) {
    bo[k].wqkv = take(3 * D * D * e);
    bo[k].wo = take(D * D * e);
    bo[k].wcq = take(D * D * e);
    bo[k].wco = take(D * D * e);
    bo[k].w1 = take(FF * D * e);
    bo[k].w2 = take(D * FF * e);
    bo[k].bqkv = take(3 * D * 4);
    bo[k].gqkv = take(3 * D * 4);
    bo[k].bo = take(D * 4);
    bo[k].bcq = take(D * 4);
    bo[k].gcq = take(D * 4);
    bo[k].bco = take(D * 4);
    bo[k].ln3w = take(D * 4);
    bo[k].ln3b = take(D * 4);
    bo[k].b1 = take(FF * 4);
    bo[k].b2 = take(D * 4);
  }
  const size_t o_wckv = take(NB * 2 * D * D * e), o_bckv = take(NB * 2 * D * 4), o_gckv = take(NB * 2 * D * 4),
               o_mod = take(NB * 6 * D * 4), o_pw = take(D * 2 * C * e), o_pb = take(D * 4), o_hw = take(C * D * e),
               o_hb = take(C * 4), o_hm = take(2 * D * 4), o_tw1 = take(D * 256 * e), o_tb1 = take(D * 4),
               o_tw2 = take(D * D * e), o_tb2 = take(D * 4), o_twp = take(6 * D * D * e), o_tbp = take(6 * D * 4),
               o_rope = take((size_t)L * 64 * 8);
  const size_t o_aw1 = take((size_t)AU_HID * AU_K0 * e), o_ab1 = take(AU_HID * 4),
               o_aw1v = take((size_t)AU_HID * AU_KV * e), o_ab1v = take(AU_HID * 4),
               o_aw2 = take((size_t)AU_HID * AU_HID * e), o_ab2 = take(AU_HID * 4),
               o_aw3 = take((size_t)32 * D * AU_HID * e), o_ab3 = take((size_t)32 * D * 4), o_anw = take(D * 4),
               o_anb = take(D * 4);
  m->arena_bytes = off;
  if (cudaMalloc(&m->arena, off) != cudaSuccess) {
    cudaGetLastError();
    delete m;
    return fail(FH_ERR_OOM, "weight arena of %zu bytes", off);
  }
  uint8_t* a = reinterpret_cast<uint8_t*>(m->arena);
  m->blk.resize(NB);
  for (long k = 0; k < NB; ++k) {
    BlockW& b = m->blk[k];
    b.wqkv = a + bo[k].wqkv;
    b.wo = a + bo[k].wo;
    b.wcq = a + bo[k].wcq;
    b.wco = a + bo[k].wco;
    b.w1 = a + bo[k].w1;
    b.w2 = a + bo[k].w2;
    b.bqkv = (float*)(a + bo[k].bqkv);
    b.gqkv = (float*)(a + bo[k].gqkv);
    b.bo = (float*)(a + bo[k].bo);
    b.bcq = (float*)(a + bo[k].bcq);
    b.gcq = (float*)(a + bo[k].gcq);
    b.bco = (float*)(a + bo[k].bco);
    b.ln3w = (float*)(a + bo[k].ln3w);
    b.ln3b = (float*)(a + bo[k].ln3b);
    b.b1 = (float*)(a + bo[k].b1);
    b.b2 = (float*)(a + bo[k].b2);
  }
  m->wckv = a + o_wckv;
  m->bckv = (float*)(a + o_bckv);
  m->gckv = (float*)(a + o_gckv);
  m->modtab = (float*)(a + o_mod);
  m->patch_w = a + o_pw;
  m->patch_b = (float*)(a + o_pb);
  m->head_w = a + o_hw;
  m->head_b = (float*)(a + o_hb);
  m->head_mod = (float*)(a + o_hm);
  m->t_w1 = a + o_tw1;
  m->t_b1 = (float*)(a + o_tb1);
  m->t_w2 = a + o_tw2;
  m->t_b2 = (float*)(a + o_tb2);
  m->t_wp = a + o_twp;
  m->t_bp = (float*)(a + o_tbp);
  m->rope = (float2*)(a + o_rope);
  m->a_w1 = a + o_aw1;
  m->a_b1 = (float*)(a + o_ab1);
  m->a_w1v = a + o_aw1v;
  m->a_b1v = (float*)(a + o_ab1v);
  m->a_w2 = a + o_aw2;
  m->a_b2 = (float*)(a + o_ab2);
  m->a_w3 = a + o_aw3;
  m->a_b3 = (float*)(a + o_ab3);
  m->a_nw = (float*)(a + o_anw);
  m->a_nb = (float*)(a + o_anb);

  // ---- tensor records: id -> storage (the id scheme of fh.h)
  auto rec = [&](int tid, void* p, long rows, long cols, long ld, bool mat, int kind, int fan) {
    m->recs.push_back(TensorRec{tid, p, rows, cols, ld, mat, kind, fan});
  };
  const int LIN = 0, GAIN = 1, LNB = 2;
  for (long k = 0; k < NB; ++k) {
    BlockW& b = m->blk[k];
    auto T = [&](int s) { return (int)FH_BLOCK_TENSOR(k, s); };
    uint8_t* wqkv = (uint8_t*)b.wqkv;
    uint8_t* wckv_k = (uint8_t*)m->wckv + (size_t)k * 2 * D * D * e;
    rec(T(0), m->modtab + k * 6 * D, 6, D, D, false, LIN, (int)D);
    rec(T(1), wqkv, D, D, D, true, LIN, (int)D);
    rec(T(2), b.bqkv, 1, D, D, false, LIN, (int)D);
    rec(T(3), wqkv + D * D * e, D, D, D, true, LIN, (int)D);
    rec(T(4), b.bqkv + D, 1, D, D, false, LIN, (int)D);
    rec(T(5), wqkv + 2 * D * D * e, D, D, D, true, LIN, (int)D);
    rec(T(6), b.bqkv + 2 * D, 1, D, D, false, LIN, (int)D);
    rec(T(7), b.wo, D, D, D, true, LIN, (int)D);
    rec(T(8), b.bo, 1, D, D, false, LIN, (int)D);
    rec(T(9), b.gqkv, 1, D, D, false, GAIN, 1);
    rec(T(10), b.gqkv + D, 1, D, D, false, GAIN, 1);
    rec(T(11), b.ln3w, 1, D, D, false, GAIN, 1);
    rec(T(12), b.ln3b, 1, D, D, false, LNB, 1);
    rec(T(13), b.wcq, D, D, D, true, LIN, (int)D);
    rec(T(14), b.bcq, 1, D, D, false, LIN, (int)D);
    rec(T(15), wckv_k, D, D, D, true, LIN, (int)D);
    rec(T(16), m->bckv + k * 2 * D, 1, D, D, false, LIN, (int)D);
    rec(T(17), wckv_k + D * D * e, D, D, D, true, LIN, (int)D);
    rec(T(18), m->bckv + k * 2 * D + D, 1, D, D, false, LIN, (int)D);
    rec(T(19), b.wco, D, D, D, true, LIN, (int)D);
    rec(T(20), b.bco, 1, D, D, false, LIN, (int)D);
    rec(T(21), b.gcq, 1, D, D, false, GAIN, 1);
    rec(T(22), m->gckv + k * 2 * D, 1, D, D, false, GAIN, 1);
    rec(T(23), b.w1, FF, D, D, true, LIN, (int)D);
    rec(T(24), b.b1, 1, FF, FF, false, LIN, (int)D);
    rec(T(25), b.w2, D, FF, FF, true, LIN, (int)FF);
    rec(T(26), b.b2, 1, D, D, false, LIN, (int)FF);
  }
  rec(FH_GLOBAL_TENSOR(0), m->patch_w, D, 2 * C, 2 * C, true, LIN, (int)(2 * C));
  rec(FH_GLOBAL_TENSOR(1), m->patch_b, 1, D, D, false, LIN, (int)(2 * C));
  rec(FH_GLOBAL_TENSOR(2), m->head_w, C, D, D, true, LIN, (int)D);
  rec(FH_GLOBAL_TENSOR(3), m->head_b, 1, C, C, false, LIN, (int)D);
  rec(FH_GLOBAL_TENSOR(4), m->head_mod, 2, D, D, false, LIN, (int)D);
  rec(FH_GLOBAL_TENSOR(5), m->t_w1, D, 256, 256, true, LIN, 256);
  rec(FH_GLOBAL_TENSOR(6), m->t_b1, 1, D, D, false, LIN, 256);
  rec(FH_GLOBAL_TENSOR(7), m->t_w2, D, D, D, true, LIN, (int)D);
  rec(FH_GLOBAL_TENSOR(8), m->t_b2, 1, D, D, false, LIN, (int)D);
  rec(FH_GLOBAL_TENSOR(9), m->t_wp, 6 * D, D, D, true, LIN, (int)D);
  rec(FH_GLOBAL_TENSOR(10), m->t_bp, 1, 6 * D, 6 * D, false, LIN, (int)D);
  rec(FH_AUDIO_TENSOR(0), m->a_w1, AU_HID, AU_K0, AU_K0, true, LIN, AU_K0);
  rec(FH_AUDIO_TENSOR(1), m->a_b1, 1, AU_HID, AU_HID, false, LIN, AU_K0);
  rec(FH_AUDIO_TENSOR(2), m->a_w1v, AU_HID, AU_KV, AU_KV, true, LIN, AU_KV);
  rec(FH_AUDIO_TENSOR(3), m->a_b1v, 1, AU_HID, AU_HID, false, LIN, AU_KV);
  rec(FH_AUDIO_TENSOR(4), m->a_w2, AU_HID, AU_HID, AU_HID, true, LIN, AU_HID);
  rec(FH_AUDIO_TENSOR(5), m->a_b2, 1, AU_HID, AU_HID, false, LIN, AU_HID);
  rec(FH_AUDIO_TENSOR(6), m->a_w3, 32 * D, AU_HID, AU_HID, true, LIN, AU_HID);
  rec(FH_AUDIO_TENSOR(7), m->a_b3, 1, 32 * D, 32 * D, false, LIN, AU_HID);
  rec(FH_AUDIO_TENSOR(8), m->a_nw, 1, D, D, false, GAIN, 1);
  rec(FH_AUDIO_TENSOR(9), m->a_nb, 1, D, D, false, LNB, 1);

  // ---- generate
  int rc = FH_OK;
  auto genfail = [&](cudaError_t er) {
    rc = fail(FH_ERR_CUDA, "weight generation: %s", cudaGetErrorString(er));
  };
  for (const TensorRec& r : m->recs) {
    cudaError_t er;
    if (r.mat && m->bf16)
      er = gen_tensor<bf16>((bf16*)r.ptr, r.rows, r.cols, r.ld, seed, r.tid, r.kind, r.fan, false, st);
    else
      er = gen_tensor<float>((float*)r.ptr, r.rows, r.cols, r.ld, seed, r.tid, r.kind, r.fan, m->bf16, st);
    if (er != cudaSuccess) {
      genfail(er);
      break;
    }
  }
  // gains of the unnormalised (value) columns are 1
  for (long k = 0; rc == FH_OK && k < NB; ++k) {
    cudaError_t e1 = fill_f32(m->blk[k].gqkv + 2 * D, D, 1.f, st);
    cudaError_t e2 = fill_f32(m->gckv + k * 2 * D + D, D, 1.f, st);
    if (e1 != cudaSuccess || e2 != cudaSuccess) genfail(e1 != cudaSuccess ? e1 : e2);
  }
  if (rc == FH_OK) {
    cudaError_t er = rope_table(m->rope, m->F, c.lat_h, c.lat_w, c.rope_split[0] / 2, c.rope_split[1] / 2,
                                c.rope_split[2] / 2, c.rope_theta, st);
    if (er != cudaSuccess) genfail(er);
  }
  if (rc == FH_OK && cudaStreamSynchronize(st) != cudaSuccess) rc = fail(FH_ERR_CUDA, "weight generation sync");

  // ---- weight tensor maps
  if (rc == FH_OK && m->bf16) {
    bool ok = true;
    for (long k = 0; k < NB && ok; ++k) {
      BlockW& b = m->blk[k];
      auto box = [](long n, long kk) { return (uint32_t)tile_cfg((int)n, (int)kk).wbox; };
      ok = make_map(&b.m_qkv, b.wqkv, 3 * D, D, box(3 * D, D)) && make_map(&b.m_o, b.wo, D, D, box(D, D)) &&
           make_map(&b.m_cq, b.wcq, D, D, box(D, D)) && make_map(&b.m_co, b.wco, D, D, box(D, D)) &&
           make_map(&b.m_1, b.w1, FF, D, box(FF, D)) && make_map(&b.m_2, b.w2, D, FF, box(D, FF)) &&
           make_map(&b.m_ckv, (uint8_t*)m->wckv + (size_t)k * 2 * D * D * e, 2 * D, D, box(2 * D, D));
    }
    auto box = [](long n, long kk) { return (uint32_t)tile_cfg((int)n, (int)kk).wbox; };
    ok = ok && make_map(&m->m_ckv_all, m->wckv, NB * 2 * D, D, box(NB * 2 * D, D)) &&
         make_map(&m->m_patch, m->patch_w, D, 2 * C, box(D, 2 * C)) && make_map(&m->m_head, m->head_w, C, D, box(C, D));
    if (!ok) rc = fail(FH_ERR_CUDA, "weight tensor map encoding failed");
  }
  if (rc == FH_OK) {
    if (cudaHostAlloc((void**)&m->err_host, sizeof(unsigned), cudaHostAllocMapped) != cudaSuccess ||
        cudaHostGetDevicePointer((void**)&m->err_dev, m->err_host, 0) != cudaSuccess)
      rc = fail(FH_ERR_CUDA, "error word allocation failed");
    else
      *m->err_host = 0;
  }
  if (rc == FH_OK && cudaStreamCreateWithFlags(&m->cap, cudaStreamNonBlocking) != cudaSuccess)
    rc = fail(FH_ERR_CUDA, "capture stream creation failed");
  if (rc != FH_OK) {
    fh_dit_destroy(m);
    return rc;
  }
  *out = m;
  return FH_OK;
}

int fh_dit_destroy(fh_dit* m) {
  if (!m) return FH_OK;
  cudaSetDevice(m->device);
  for (auto& g : m->graphs) cudaGraphExecDestroy(g.exec);
  for (auto ev : m->events) cudaEventDestroy(ev);
  if (m->cap) cudaStreamDestroy(m->cap);
  if (m->err_host) cudaFreeHost(m->err_host);
  if (m->arena) cudaFree(m->arena);
  delete m;
  return FH_OK;
}

size_t fh_dit_workspace_bytes(const fh_dit* m, int batch) {
  if (!m || batch < 1 || batch > m->cfg.max_batch) return 0;
  return layout(m, batch).total;
}

int fh_dit_block_forward(fh_dit* m, int block, const float* x_in, float* x_out, const void* audio, const float* t,
                         int batch, void* ws, void* stream) {
  RUN(common_checks(m, batch, ws));
  if (block < 0 || block >= m->NB) return fail(FH_ERR_ARG, "block %d outside [0, %d)", block, m->NB);
  if (!x_in || !x_out || !audio || !t || !aligned16(x_in) || !aligned16(x_out) || !aligned16(audio))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  m->launches = 0;
  const size_t M = (size_t)batch * m->L;
  CK(cudaMemcpyAsync(at<void>(ws, P->lay.audio), audio, (size_t)batch * m->F * m->A * m->D * elt(m),
                     cudaMemcpyDeviceToDevice, st));
  if (x_out != x_in) CK(cudaMemcpyAsync(x_out, x_in, M * m->D * 4, cudaMemcpyDeviceToDevice, st));
  TVals tv;
  for (int b = 0; b < 8; ++b) tv.t[b] = t[b < batch ? b : 0];
  RUN(run_cross_kv(m, *P, block, 1, st));
  RUN(run_time_cond(m, *P, tv, st));
  if (m->bf16)
    RUN(run_block<bf16>(m, *P, block, x_out, st));
  else
    RUN(run_block<float>(m, *P, block, x_out, st));
  m->last_launches = m->launches;
  return FH_OK;
}

int fh_dit_predict_flow(fh_dit* m, const float* x_noisy, const float* ref, const void* audio, float sigma,
                        float* v_out, int batch, void* ws, void* stream) {
  RUN(common_checks(m, batch, ws));
  if (!x_noisy || !ref || !audio || !v_out || !aligned16(x_noisy) || !aligned16(ref) || !aligned16(audio) ||
      !aligned16(v_out))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  m->launches = 0;
  const WsLayout& w = P->lay;
  CK(cudaMemcpyAsync(at<void>(ws, w.audio), audio, (size_t)batch * m->F * m->A * m->D * elt(m),
                     cudaMemcpyDeviceToDevice, st));
  TVals tv;
  for (int b = 0; b < 8; ++b) tv.t[b] = sigma;
  if (m->bf16)
    LAUNCH(prep_tokens<bf16>(x_noisy, ref, nullptr, 0, nullptr, at<bf16>(ws, w.tok), batch, m->C, m->L, m->HW, st));
  else
    LAUNCH(prep_tokens<float>(x_noisy, ref, nullptr, 0, nullptr, at<float>(ws, w.tok), batch, m->C, m->L, m->HW, st));
  RUN(run_cross_kv(m, *P, 0, m->NB, st));
  RUN(run_time_cond(m, *P, tv, st));
  if (m->bf16)
    RUN(run_network<bf16>(m, *P, st));
  else
    RUN(run_network<float>(m, *P, st));
  LAUNCH(tokens_to_latent(at<float>(ws, w.v), v_out, batch, m->C, m->L, st));
  m->last_launches = m->launches;
  return FH_OK;
}

static int sample_impl(fh_dit* m, const float* noise, const float* ref, const float* motion, const float* sigmas,
                       int nsteps, const float* eps, float* x_out, int batch, void* ws, cudaStream_t st) {
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  const WsLayout& w = P->lay;
  m->launches = 0;
  if (m->bf16)
    LAUNCH(prep_tokens<bf16>(noise, ref, motion, 2, at<float>(ws, w.lat), at<bf16>(ws, w.tok), batch, m->C, m->L,
                             m->HW, st));
  else
    LAUNCH(prep_tokens<float>(noise, ref, motion, 2, at<float>(ws, w.lat), at<float>(ws, w.tok), batch, m->C, m->L,
                              m->HW, st));
  const int outside = m->launches;
  // find or record the graph of the step loop
  GraphEntry* g = nullptr;
  for (auto& e : m->graphs)
    if (e.ws == ws && e.eps == eps && e.batch == batch && e.nsteps == nsteps && e.timing == m->timing &&
        memcmp(e.sigmas.data(), sigmas, sizeof(float) * (nsteps + 1)) == 0)
      g = &e;
  if (!g) {
    if (m->graphs.size() >= 8) {
      cudaGraphExecDestroy(m->graphs.front().exec);
      m->graphs.erase(m->graphs.begin());
    }
    CK(cudaStreamBeginCapture(m->cap, cudaStreamCaptureModeRelaxed));
    m->capturing = true;
    m->launches = 0;
    m->ev_used = 0;
    m->last_pairs.clear();
    int rc = m->bf16 ? run_sampler_steps<bf16>(m, *P, sigmas, nsteps, eps, m->cap)
                     : run_sampler_steps<float>(m, *P, sigmas, nsteps, eps, m->cap);
    m->capturing = false;
    cudaGraph_t graph = nullptr;
    cudaError_t ce = cudaStreamEndCapture(m->cap, &graph);
    if (rc != FH_OK) {
      if (graph) cudaGraphDestroy(graph);
      return rc;
    }
    if (ce != cudaSuccess) return fail(FH_ERR_CUDA, "stream capture failed: %s", cudaGetErrorString(ce));
    cudaGraphExec_t exec = nullptr;
    ce = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ce != cudaSuccess) return fail(FH_ERR_CUDA, "graph instantiation failed: %s", cudaGetErrorString(ce));
    GraphEntry ge;
    ge.ws = ws;
    ge.eps = eps;
    ge.batch = batch;
    ge.nsteps = nsteps;
    ge.timing = m->timing;
    ge.sigmas.assign(sigmas, sigmas + nsteps + 1);
    ge.exec = exec;
    ge.launches = m->launches;
    ge.ev_pairs = m->last_pairs;
    m->graphs.push_back(ge);
    g = &m->graphs.back();
  }
  CK(cudaGraphLaunch(g->exec, st));
  m->last_pairs = g->ev_pairs;
  m->launches = outside + g->launches;
  LAUNCH(tokens_to_latent(at<float>(ws, w.lat), x_out, batch, m->C, m->L, st));
  m->last_launches = m->launches;
  return FH_OK;
}

static int check_sigmas(const float* sigmas, int nsteps) {
  if (!sigmas || nsteps < 1 || nsteps > 64) return fail(FH_ERR_ARG, "sigmas null or nsteps %d outside [1, 64]", nsteps);
  return FH_OK;
}

int fh_sample_slice(fh_dit* m, const float* noise, const float* ref, const float* motion, const void* audio,
                    const float* sigmas, int nsteps, float* x_out, int batch, void* ws, void* stream) {
  RUN(common_checks(m, batch, ws));
  RUN(check_sigmas(sigmas, nsteps));
  if (!noise || !ref || !motion || !audio || !x_out || !aligned16(noise) || !aligned16(ref) || !aligned16(motion) ||
      !aligned16(audio) || !aligned16(x_out))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  CK(cudaMemcpyAsync(at<void>(ws, P->lay.audio), audio, (size_t)batch * m->F * m->A * m->D * elt(m),
                     cudaMemcpyDeviceToDevice, st));
  return sample_impl(m, noise, ref, motion, sigmas, nsteps, nullptr, x_out, batch, ws, st);
}

int fh_sample_slice_renoise(fh_dit* m, const float* noise, const float* ref, const float* motion, const void* audio,
                            const float* sigmas, int nsteps, const float* eps, float* x_out, int batch, void* ws,
                            void* stream) {
  RUN(common_checks(m, batch, ws));
  RUN(check_sigmas(sigmas, nsteps));
  if (!noise || !ref || !motion || !audio || !eps || !x_out || !aligned16(noise) || !aligned16(ref) ||
      !aligned16(motion) || !aligned16(audio) || !aligned16(eps) || !aligned16(x_out))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  CK(cudaMemcpyAsync(at<void>(ws, P->lay.audio), audio, (size_t)batch * m->F * m->A * m->D * elt(m),
                     cudaMemcpyDeviceToDevice, st));
  return sample_impl(m, noise, ref, motion, sigmas, nsteps, eps, x_out, batch, ws, st);
}

int fh_sample_slice_host(fh_dit* m, const float* noise_host, const float* ref_host, const float* motion_host,
                         const void* audio_host, const float* sigmas, int nsteps, float* x_out_host, int batch,
                         void* ws, void* stream) {
  RUN(common_checks(m, batch, ws));
  RUN(check_sigmas(sigmas, nsteps));
  if (!noise_host || !ref_host || !motion_host || !audio_host || !x_out_host)
    return fail(FH_ERR_ARG, "null host pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  const WsLayout& w = P->lay;
  const size_t lat = (size_t)batch * m->C * m->L * 4;
  CK(cudaMemcpyAsync(at<void>(ws, w.in_noise), noise_host, lat, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(at<void>(ws, w.in_ref), ref_host, lat, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(at<void>(ws, w.in_motion), motion_host, (size_t)batch * m->C * 2 * m->HW * 4,
                     cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(at<void>(ws, w.audio), audio_host, (size_t)batch * m->F * m->A * m->D * elt(m),
                     cudaMemcpyHostToDevice, st));
  RUN(sample_impl(m, at<float>(ws, w.in_noise), at<float>(ws, w.in_ref), at<float>(ws, w.in_motion), sigmas, nsteps, nullptr,
                  at<float>(ws, w.out), batch, ws, st));
  CK(cudaMemcpyAsync(x_out_host, at<void>(ws, w.out), lat, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  return check_err_word(m);
}

int fh_audio_project(fh_dit* m, const float* states, void* tokens, int batch, void* ws, void* stream) {
  RUN(common_checks(m, batch, ws));
  if (!states || !tokens || !aligned16(states) || !aligned16(tokens)) return fail(FH_ERR_ARG, "null or unaligned pointer");
  const int nv = 1 + AU_STRIDE * (m->F - 1);
  if (nv > AU_STATES || m->A != 32) return fail(FH_ERR_SHAPE, "%d latent frames need %d video frames of states", m->F, nv);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Plan* P;
  RUN(get_plan(m, ws, batch, &P));
  const WsLayout& w = P->lay;
  m->launches = 0;
  const int B = batch, F = m->F, R = B * F, D = m->D;
  float *win0 = at<float>(ws, w.au_win0), *winv = at<float>(ws, w.au_winv), *part = at<float>(ws, w.au_part),
        *h1 = at<float>(ws, w.au_h1), *h2 = at<float>(ws, w.au_h2), *tk = at<float>(ws, w.au_tok);
  LAUNCH(audio_windows(states, win0, winv, B, AU_STATES, AU_PER_STATE, F, AU_STATES - nv, AU_WIN, AU_STRIDE, AU_GROUP,
                       st));
  cudaError_t e;
  if (m->bf16) {
    e = audio_linear<bf16>((const bf16*)m->a_w1, win0, m->a_b1, part, h1, AU_HID, AU_K0, B, 1, 1, F, 0, st);
    if (e == cudaSuccess)
      e = audio_linear<bf16>((const bf16*)m->a_w1v, winv, m->a_b1v, part, h1, AU_HID, AU_KV, B * (F - 1), 1, F - 1, F,
                             1, st);
    if (e == cudaSuccess)
      e = audio_linear<bf16>((const bf16*)m->a_w2, h1, m->a_b2, part, h2, AU_HID, AU_HID, R, 1, R, 0, 0, st);
    if (e == cudaSuccess)
      e = audio_linear<bf16>((const bf16*)m->a_w3, h2, m->a_b3, part, tk, 32 * D, AU_HID, R, 0, R, 0, 0, st);
    if (e == cudaSuccess)
      e = norm_rows<bf16>(tk, (bf16*)tokens, R * 32, D, R * 32, 1, nullptr, nullptr, 0, m->a_nw, m->a_nb, m->cfg.eps,
                          st);
  } else {
    e = audio_linear<float>((const float*)m->a_w1, win0, m->a_b1, part, h1, AU_HID, AU_K0, B, 1, 1, F, 0, st);
    if (e == cudaSuccess)
      e = audio_linear<float>((const float*)m->a_w1v, winv, m->a_b1v, part, h1, AU_HID, AU_KV, B * (F - 1), 1, F - 1,
                              F, 1, st);
    if (e == cudaSuccess)
      e = audio_linear<float>((const float*)m->a_w2, h1, m->a_b2, part, h2, AU_HID, AU_HID, R, 1, R, 0, 0, st);
    if (e == cudaSuccess)
      e = audio_linear<float>((const float*)m->a_w3, h2, m->a_b3, part, tk, 32 * D, AU_HID, R, 0, R, 0, 0, st);
    if (e == cudaSuccess)
      e = norm_rows<float>(tk, (float*)tokens, R * 32, D, R * 32, 1, nullptr, nullptr, 0, m->a_nw, m->a_nb, m->cfg.eps,
                           st);
  }
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "audio projection launch: %s", cudaGetErrorString(e));
  m->launches += 9;  // four split-K products with their reductions, and the norm
  m->last_launches = m->launches;
  return FH_OK;
}

int fh_dit_get_weight(const fh_dit* m, int tensor_id, void* host_dst, size_t bytes) {
  if (!m || !host_dst) return fail(FH_ERR_ARG, "null argument");
  for (const TensorRec& r : m->recs) {
    if (r.tid != tensor_id) continue;
    const size_t n = (size_t)r.rows * r.cols;
    if (bytes != n * 4) return fail(FH_ERR_ARG, "tensor %d needs %zu bytes, got %zu", tensor_id, n * 4, bytes);
    if (cudaSetDevice(m->device) != cudaSuccess) return fail(FH_ERR_CUDA, "cudaSetDevice");
    float* dst = reinterpret_cast<float*>(host_dst);
    if (r.mat && m->bf16) {
      std::vector<uint16_t> tmp(n);
      CK(cudaMemcpy2D(tmp.data(), r.cols * 2, r.ptr, r.ld * 2, r.cols * 2, r.rows, cudaMemcpyDeviceToHost));
      for (size_t i = 0; i < n; ++i) {
        uint32_t u = (uint32_t)tmp[i] << 16;
        memcpy(&dst[i], &u, 4);
      }
    } else {
      CK(cudaMemcpy2D(dst, r.cols * 4, r.ptr, r.ld * 4, r.cols * 4, r.rows, cudaMemcpyDeviceToHost));
    }
    return FH_OK;
  }
  return fail(FH_ERR_ARG, "unknown tensor id %d", tensor_id);
}

int fh_dit_sync(fh_dit* m, void* stream) {
  if (!m) return fail(FH_ERR_ARG, "null model");
  cudaSetDevice(m->device);
  CK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  return check_err_word(m);
}

int fh_dit_last_launch_count(const fh_dit* m) { return m ? m->last_launches : 0; }

int fh_dit_set_timing(fh_dit* m, int kernel_class) {
  if (!m || kernel_class < 0 || kernel_class > 7) return fail(FH_ERR_ARG, "bad timing class");
  cudaSetDevice(m->device);
  if (kernel_class && m->events.empty()) {
    m->events.resize(2048);
    for (auto& ev : m->events) CK(cudaEventCreate(&ev));
  }
  m->timing = kernel_class;
  return FH_OK;
}

int fh_dit_get_timing(fh_dit* m, double* mean_us, int* launches) {
  if (!m || !mean_us || !launches) return fail(FH_ERR_ARG, "null argument");
  cudaSetDevice(m->device);
  double tot = 0;
  int n = 0;
  for (int i : m->last_pairs) {
    float ms = 0;
    CK(cudaEventSynchronize(m->events[i + 1]));
    CK(cudaEventElapsedTime(&ms, m->events[i], m->events[i + 1]));
    tot += ms * 1000.0;
    ++n;
  }
  *mean_us = n ? tot / n : 0.0;
  *launches = n;
  return FH_OK;
}

int fh_dit_probe_wait_timeout(fh_dit* m, void* stream) {
  if (!m) return fail(FH_ERR_ARG, "null model");
  if (cudaSetDevice(m->device) != cudaSuccess) return fail(FH_ERR_CUDA, "cudaSetDevice failed");
  CK(wait_probe(m->err_dev, reinterpret_cast<cudaStream_t>(stream)));
  return FH_OK;
}

// ------------------------------------------------------------ operator entry points
int fh_op_linear(const void* A, const void* W, const float* bias, float* out, int M, int N, int K, int dtype,
                 void* stream) {
  if (!A || !W || !bias || !out || !aligned16(A) || !aligned16(W) || !aligned16(bias) || !aligned16(out))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  if (M < 1 || N < 128 || N % 128 || K < 32) return fail(FH_ERR_SHAPE, "bad GEMM shape %d x %d x %d", M, N, K);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  EpiParams ep = epi0(1 << 30);
  ep.bias = bias;
  ep.out = out;
  ep.ldo = N;
  cudaError_t e;
  if (dtype == FH_BF16) {
    if (K % 64) return fail(FH_ERR_SHAPE, "K %% 64 != 0");
    if (!load_encode()) return fail(FH_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled unavailable");
    const TileCfg tc = tile_cfg(N, K);
    CUtensorMap ma, mb, mc;
    if (!make_map(&ma, A, M, K, 128) || !make_map(&mb, W, N, K, tc.wbox) ||
        !make_out_map(&mc, out, M, N, N, true))
      return fail(FH_ERR_CUDA, "tensor map encoding");
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    RUN(prepare_device(dev));
    e = gemm_tc(ma, mb, &mc, M, N, K, tc.bn, EPI_STORE, false, ep, nullptr, sms, st, tc.pair);
  } else if (dtype == FH_F32) {
    if (K % 32) return fail(FH_ERR_SHAPE, "K %% 32 != 0");
    e = gemm_simt((const float*)A, K, (const float*)W, K, M, N, K, EPI_STORE, ep, st);
  } else {
    return fail(FH_ERR_ARG, "bad dtype");
  }
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "linear launch: %s", cudaGetErrorString(e));
  return FH_OK;
}

int fh_op_cross_attention(const void* q, const float* ssq_q, const void* kv, const float* ssq_k, void* out, int batch,
                          int heads, int frames, int hw, int audio_tokens, float eps, int dtype, void* stream) {
  if (!q || !ssq_q || !kv || !ssq_k || !out || !aligned16(q) || !aligned16(kv) || !aligned16(out))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  if (batch < 1 || heads < 1 || heads > 64 || frames < 1 || hw < 1 || audio_tokens != 32)
    return fail(FH_ERR_SHAPE, "bad cross-attention shape (audio_tokens must be 32)");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int D = heads * 128, L = frames * hw;
  cudaError_t e;
  if (dtype == FH_BF16) {
    if (!load_encode()) return fail(FH_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled unavailable");
    const uint64_t nf = (uint64_t)batch * frames;
    CUtensorMap mq, mkv, mo;
    if (!make_map_3d(&mq, q, D, hw, nf, 64, 128) || !make_map_3d(&mo, out, D, hw, nf, 64, 32) ||
        !make_map(&mkv, kv, nf * audio_tokens, 2 * (uint64_t)D, 32))
      return fail(FH_ERR_CUDA, "tensor map encoding");
    int dev = 0;
    cudaGetDevice(&dev);
    RUN(prepare_device(dev));
    e = xattn_tc(mq, mkv, mo, ssq_q, ssq_k, heads, 0, 0, D, batch, heads, L, frames, audio_tokens, eps, nullptr, st);
  } else if (dtype == FH_F32) {
    int dev = 0;
    cudaGetDevice(&dev);
    RUN(prepare_device(dev));
    e = cross_attn<float>((const float*)q, ssq_q, (const float*)kv, 2L * D, 0, D, ssq_k, heads, 0, batch, heads, L,
                          frames, audio_tokens, eps, (float*)out, st);
  } else {
    return fail(FH_ERR_ARG, "bad dtype");
  }
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "cross-attention launch: %s", cudaGetErrorString(e));
  return FH_OK;
}

int fh_op_row_norm(const float* x, void* out, int M, int D, int mode, const float* a, const float* c, long bstride,
                   int rows_per_batch, float eps, int dtype, void* stream) {
  if (!x || !out || !a || !c || !aligned16(x) || !aligned16(out) || !aligned16(a) || !aligned16(c))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  if (M < 1 || rows_per_batch < 1 || mode < 0 || mode > 2 || bstride < 0)
    return fail(FH_ERR_SHAPE, "bad row-norm arguments");
  const int nv = D / 128;
  if (D % 128 || !(nv == 1 || nv == 2 || nv == 3 || nv == 4 || nv == 6 || nv == 8 || nv == 12 || nv == 16))
    return fail(FH_ERR_SHAPE, "row width %d not supported", D);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // norm_rows takes (shift, scale) for the modulated modes and (weight, bias) for mode 1
  cudaError_t e;
  if (dtype == FH_BF16)
    e = mode == 1 ? norm_rows<bf16>(x, (bf16*)out, M, D, rows_per_batch, 1, nullptr, nullptr, 0, a, c, eps, st)
                  : norm_rows<bf16>(x, (bf16*)out, M, D, rows_per_batch, mode, c, a, bstride, nullptr, nullptr, eps, st);
  else if (dtype == FH_F32)
    e = mode == 1 ? norm_rows<float>(x, (float*)out, M, D, rows_per_batch, 1, nullptr, nullptr, 0, a, c, eps, st)
                  : norm_rows<float>(x, (float*)out, M, D, rows_per_batch, mode, c, a, bstride, nullptr, nullptr, eps,
                                     st);
  else
    return fail(FH_ERR_ARG, "bad dtype");
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "row-norm launch: %s", cudaGetErrorString(e));
  return FH_OK;
}

int fh_op_attention(const void* q, const void* k, const void* v, const float* ssq, void* out, int batch, int heads,
                    int L, float eps, int dtype, void* stream) {
  if (!q || !k || !v || !ssq || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(FH_ERR_ARG, "null or unaligned pointer");
  if (batch < 1 || heads < 1 || L < 1) return fail(FH_ERR_SHAPE, "bad attention shape");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == FH_BF16) {
    if (!load_encode()) return fail(FH_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled unavailable");
    const uint64_t rows = (uint64_t)batch * heads * L;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, rows, 128, 128) || !make_map(&mk, k, rows, 128, 128) || !make_map(&mv, v, rows, 128, 128))
      return fail(FH_ERR_CUDA, "tensor map encoding");
    int dev = 0;
    cudaGetDevice(&dev);
    RUN(prepare_device(dev));
    e = attn_tc(mq, mk, mv, ssq, 2 * heads, batch, heads, L, eps, (bf16*)out, nullptr, st);
  } else if (dtype == FH_F32) {
    e = attn_simt<float>((const float*)q, (const float*)k, (const float*)v, ssq, 2 * heads, batch, heads, L, eps,
                         (float*)out, st);
  } else {
    return fail(FH_ERR_ARG, "bad dtype");
  }
  if (e != cudaSuccess) return fail(FH_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
  return FH_OK;
}

}  // extern "C"

// ------------------------------------------------------------ internal helpers for other files
namespace fh {
int set_error(int code, const char* msg) { return fail(code, "%s", msg); }
int model_device(const fh_dit* m) { return m ? m->device : -1; }
}  // namespace fh
