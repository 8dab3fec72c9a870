// Allocation-free variant of mla_decode_absorbed.
//
// Some callers cannot allocate device memory at the point where they decode:
// a host framework that owns every device allocation through its own pool, a
// plugin that is handed only input and output tensors, or a serving loop that
// forbids allocation on its latency path.  For them this entry point keeps its
// scratch in one fixed array that the library itself declares in device
// memory, so the caller passes only inputs and outputs.  The array is part of
// the library's device image: every GPU that loads the library holds
// MLA_DECODE_NOALLOC_SCRATCH_BYTES of it until the process exits.
#include <cstdio>
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" {

mla_status mla_decode_absorbed_noalloc(const mla_config* cfg, const void* q_nope, const void* q_pe,
                                       const void* w_kv_b, const void* latent_cache,
                                       const int32_t* cu_ctx, int32_t B, int32_t max_ctx,
                                       const void* w_o, void* out, void* stream) {
  if (!cfg) {
    mla::set_error_detail("cfg is NULL");
    return MLA_ERR_NULL;
  }
  if (mla_decode_workspace_size(cfg, B, max_ctx, nullptr) == 0) {
    mla::set_error_detail("invalid configuration, B or max_ctx");
    return MLA_ERR_SHAPE;
  }
  // the array may hold fewer partial slots than the full layout: the decode
  // then runs on fewer SM pairs
  const size_t need = mla::decode_min_workspace(*cfg, B, max_ctx);
  if (need > (size_t)MLA_DECODE_NOALLOC_SCRATCH_BYTES) {
    char msg[160];
    snprintf(msg, sizeof(msg), "decode needs %zu scratch bytes; the static array holds %zu",
             need, (size_t)MLA_DECODE_NOALLOC_SCRATCH_BYTES);
    mla::set_error_detail(msg);
    return MLA_ERR_WORKSPACE;
  }
  int dev = 0;
  const cudaError_t ed = cudaGetDevice(&dev);
  if (ed != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();   // leave no sticky runtime error behind
    char msg[160];
    snprintf(msg, sizeof(msg), "cudaGetDevice: %s (device %d, at most %d devices)",
             cudaGetErrorString(ed), dev, kMaxDevices);
    mla::set_error_detail(msg);
    return MLA_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    // Once per device, with that device current: the host-side name of the
    // array is not a device address, so ask the runtime for this device's copy.
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      const cudaError_t es = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (es != cudaSuccess || !p) {
        cudaGetLastError();
        char msg[160];
        snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the scratch array on device %d: %s",
                 dev, cudaGetErrorString(es));
        mla::set_error_detail(msg);
        return MLA_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  // The existing entry point clears the status word at the start of the
  // array and fully writes every other scratch buffer it uses.
  return mla_decode_absorbed(cfg, q_nope, q_pe, w_kv_b, latent_cache, cu_ctx, B, max_ctx, w_o,
                             out, scratch, (size_t)MLA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
