// Ring-buffer decode for callers that cannot provide scratch memory.
//
// sinkattn_decode needs a caller-provided workspace for its per-split partial
// results.  Some callers cannot allocate one: a serving loop that reserves all
// device memory up front and forbids allocation while requests are in flight
// (cudaMalloc can block on the device and can fail under memory pressure),
// or a plain C host program that only owns its input and output buffers.
// This entry point serves them from a fixed scratch array that lives in the
// library's device image: every GPU that loads the library holds it until the
// process exits.
#include <mutex>

#include "internal.h"

namespace {

// Maximum scratch: B * Hq * num_splits * (D + 2) floats (rounded up to 256
// bytes).  4 MiB per device.
constexpr size_t kScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_decode_noalloc_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Host code must
// not pass the array's name itself to a kernel: on the host it is only a
// stand-in symbol, not device memory.  Looked up once per device.
float* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch[dev] = static_cast<float*>(p);
  }
  return g_scratch[dev];
}

}  // namespace

extern "C" int sinkattn_decode_noalloc(sinkattn_dtype dt, int B, int Hq, int Hkv, int D,
                                       float scale, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* cache_seqlens,
                                       int n_sink, int window, const float* learnable_sink,
                                       void* out, float* lse_new, float* sink_s, int num_splits,
                                       sinkattn_stream_t stream) {
  if (B < 1 || Hq < 1 || (D != 64 && D != 128) || n_sink < 0 || window < 0 ||
      n_sink + window < 1)
    return SINKATTN_ERR_INVALID_ARG;
  const size_t capacity = sizeof(float) * kScratchFloats;
  if (num_splits <= 0) {
    // automatic choice, reduced until the partials fit the fixed scratch
    num_splits = sinkattn_decode_num_splits(B, Hq, Hkv, D, n_sink, window);
    while (num_splits > 1 && sinkattn_decode_workspace_bytes(B, Hq, D, num_splits) > capacity)
      --num_splits;
  }
  // the same clamp sinkattn_decode applies, before the capacity check: an
  // explicit count beyond it gives the same result with fewer slots
  num_splits = sk::decode_clamp_splits(num_splits, n_sink, window);
  if (sinkattn_decode_workspace_bytes(B, Hq, D, num_splits) > capacity)
    return SINKATTN_ERR_WORKSPACE;  // the problem needs more than the built-in scratch
  float* scratch = scratch_on_current_device();
  if (!scratch) return SINKATTN_ERR_CUDA;
  // The merge reads only the partial slots this call's streaming kernel
  // writes, so nothing needs clearing between calls.  After a call whose
  // device status is SINKATTN_ERR_TIMEOUT some slots were not written and the
  // outputs are undefined.
  return sinkattn_decode(dt, B, Hq, Hkv, D, scale, q, k_cache, v_cache, cache_seqlens, n_sink,
                         window, learnable_sink, out, lse_new, sink_s, num_splits, scratch,
                         capacity, stream);
}
