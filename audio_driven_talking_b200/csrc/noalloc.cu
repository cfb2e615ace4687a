// noalloc.cu - a block forward that allocates nothing, for callers that cannot allocate.
//
// fh_dit_block_forward needs a caller-allocated workspace. Some callers cannot call
// cudaMalloc at the point where they run a block: plugins that run inside a host
// framework that owns all device memory, and real-time threads that must not take the
// allocator's locks. For them this file provides
// fh_dit_block_forward_noalloc, which runs the same kernels on a scratch buffer that
// the library itself holds as a file-scope __device__ array (FH_STATIC_SCRATCH_BYTES;
// every GPU that loads this library keeps it until the process exits).
#include <cstdio>
#include <mutex>

#include <cuda_runtime.h>

#include "fh.h"

namespace fh {
int set_error(int code, const char* msg);
int model_device(const fh_dit* m);
}  // namespace fh

static __device__ __align__(256) unsigned char fh_static_scratch[FH_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};  // device address of fh_static_scratch, per device ordinal

// In host code `fh_static_scratch` names a host-side stand-in, not device memory: the
// device address is looked up once per device, with that device current.
int scratch_for_device(int dev, void** out) {
  if (dev < 0 || dev >= 64) return fh::set_error(FH_ERR_ARG, "device ordinal outside [0, 64)");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, fh_static_scratch);
    if (e != cudaSuccess) {
      char buf[256];
      snprintf(buf, sizeof buf, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      return fh::set_error(FH_ERR_CUDA, buf);
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FH_OK;
}
}  // namespace

extern "C" int fh_dit_block_forward_noalloc(fh_dit* m, int block, const float* x_in, float* x_out,
                                            const void* audio, const float* t, int batch, void* stream) {
  if (!m) return fh::set_error(FH_ERR_ARG, "null model");
  const size_t need = fh_dit_workspace_bytes(m, batch);
  if (need == 0) return fh::set_error(FH_ERR_SHAPE, "batch outside [1, max_batch]");
  if (need > FH_STATIC_SCRATCH_BYTES) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "this model and batch need %zu bytes of scratch; the static scratch holds %u bytes "
             "(use fh_dit_block_forward with a caller-allocated workspace)",
             need, FH_STATIC_SCRATCH_BYTES);
    return fh::set_error(FH_ERR_SHAPE, buf);
  }
  const int dev = fh::model_device(m);
  if (cudaSetDevice(dev) != cudaSuccess) return fh::set_error(FH_ERR_CUDA, "cudaSetDevice failed");
  void* scratch = nullptr;
  int rc = scratch_for_device(dev, &scratch);
  if (rc != FH_OK) return rc;
  // every buffer the block reads from the scratch is written earlier in the same call,
  // so nothing has to start at zero
  return fh_dit_block_forward(m, block, x_in, x_out, audio, t, batch, scratch, stream);
}
