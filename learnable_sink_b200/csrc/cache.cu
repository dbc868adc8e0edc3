// StreamingLLM ring-cache maintenance (page "Attention Sink / StreamingLLM",
// the core-idea section): the cache keeps the first n_sink tokens of a
// sequence in fixed slots and its most recent `window` tokens in a circular
// segment, each new token overwriting the oldest non-sink one.  Slot rule
// (shared with the decode): position p < n_sink -> slot p, otherwise
// n_sink + (p - n_sink) % window.  Both kernels are plain 16-byte copies.
#include <cuda_fp8.h>

#include "internal.h"

namespace sk {

namespace {

__device__ __forceinline__ int ring_slot(long long p, int n_sink, int window) {
  if (p < n_sink) return (int)p;
  if (window <= 0) return -1;  // no window: only the sink slots exist
  return n_sink + (int)((p - n_sink) % window);
}

// One CTA per sequence: the appended token (Hkv rows of D elements) goes to
// its slot in both caches.
__global__ void cache_append_kernel(const uint4* k_new, const uint4* v_new, const int32_t* seqlens,
                                    uint4* k_cache, uint4* v_cache, int S, int n_sink, int window,
                                    int row16) {
  const int b = blockIdx.x;
  const long long p = (long long)seqlens[b] - 1;
  if (p < 0) return;
  const int slot = ring_slot(p, n_sink, window);
  if (slot < 0) return;
  const long long dst = ((long long)b * S + slot) * row16, src = (long long)b * row16;
  for (int i = threadIdx.x; i < row16; i += blockDim.x) {
    k_cache[dst + i] = k_new[src + i];
    v_cache[dst + i] = v_new[src + i];
  }
}

// One warp per prefill token: a token that survives in the ring (one of the
// first n_sink, or one of the last `window` past them) is copied to its slot.
__global__ void cache_fill_kernel(const uint4* k, const uint4* v, const int32_t* cu, int n_seq,
                                  int T_tot, uint4* k_cache, uint4* v_cache, int32_t* lens_out,
                                  int S, int n_sink, int window, int row16) {
  if (blockIdx.x == 0 && lens_out)
    for (int s = threadIdx.x; s < n_seq; s += blockDim.x) lens_out[s] = cu[s + 1] - cu[s];
  const long long t = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T_tot) return;
  int lo = 0, hi = n_seq - 1;  // sequence holding token t: last s with cu[s] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const long long p = t - cu[lo], L = cu[lo + 1] - cu[lo];
  if (p >= L) return;
  const bool keep = p < n_sink || (window > 0 && p >= L - window);
  if (!keep) return;
  const int slot = ring_slot(p, n_sink, window);
  const long long dst = ((long long)lo * S + slot) * row16, src = t * row16;
  for (int i = lane; i < row16; i += 32) {
    k_cache[dst + i] = k[src + i];
    v_cache[dst + i] = v[src + i];
  }
}

// Mixed-precision cache (bf16 sink slots, FP8 E4M3 window rows with a scale
// per KV head): one CTA per sequence, one thread per 8 elements of the
// token's Hkv x D values.  A sink position copies its 16 bytes; a window
// position stores the E4M3 codes of value / scale (IEEE division, round to
// nearest even, saturating at +-448, NaN kept), 8 bytes per thread.
__global__ void cache_append_fp8_kernel(const uint4* k_new, const uint4* v_new,
                                        const int32_t* seqlens, uint4* k_sink, uint4* v_sink,
                                        uint2* k_win, uint2* v_win, const float* k_scale,
                                        const float* v_scale, int Hkv, int D, int n_sink,
                                        int window) {
  const int b = blockIdx.x;
  const long long p = (long long)seqlens[b] - 1;
  if (p < 0) return;
  const int row8 = Hkv * D / 8;  // 8-element chunks of the token
  if (p < n_sink) {
    const long long dst = ((long long)b * n_sink + p) * row8, src = (long long)b * row8;
    for (int i = threadIdx.x; i < row8; i += blockDim.x) {
      k_sink[dst + i] = k_new[src + i];
      v_sink[dst + i] = v_new[src + i];
    }
    return;
  }
  if (window <= 0) return;
  const long long r = (p - n_sink) % window;
  const long long dst = ((long long)b * window + r) * row8, src = (long long)b * row8;
  for (int i = threadIdx.x; i < row8; i += blockDim.x) {
    const int h = (i * 8) / D;
    const float ks = k_scale[h], vs = v_scale[h];
    const uint4 kk = k_new[src + i], vv = v_new[src + i];
    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kk);
    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vv);
    uint32_t kc[2], vc[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      uint32_t kb = 0, vb = 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float2 kf = __bfloat1622float2(k2[2 * w + u]);
        const float2 vf = __bfloat1622float2(v2[2 * w + u]);
        const uint32_t kq = __nv_cvt_float2_to_fp8x2(
            make_float2(__fdiv_rn(kf.x, ks), __fdiv_rn(kf.y, ks)), __NV_SATFINITE, __NV_E4M3);
        const uint32_t vq = __nv_cvt_float2_to_fp8x2(
            make_float2(__fdiv_rn(vf.x, vs), __fdiv_rn(vf.y, vs)), __NV_SATFINITE, __NV_E4M3);
        kb |= (kq & 0xffffu) << (16 * u);
        vb |= (vq & 0xffffu) << (16 * u);
      }
      kc[w] = kb;
      vc[w] = vb;
    }
    k_win[dst + i] = make_uint2(kc[0], kc[1]);
    v_win[dst + i] = make_uint2(vc[0], vc[1]);
  }
}

bool cache_args_ok(sinkattn_dtype dt, int Hkv, int D, int n_sink, int window) {
  return (dt == SINKATTN_BF16 || dt == SINKATTN_FP16 || dt == SINKATTN_FP32) && Hkv >= 1 && (D == 64 || D == 128) &&
         n_sink >= 0 && window >= 0 && n_sink + window >= 1;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

}  // namespace sk

using namespace sk;

extern "C" int sinkattn_cache_append(sinkattn_dtype dt, int B, int Hkv, int D, int n_sink,
                                     int window, const void* k_new, const void* v_new,
                                     const int32_t* cache_seqlens, void* k_cache, void* v_cache,
                                     sinkattn_stream_t stream) {
  if (!cache_args_ok(dt, Hkv, D, n_sink, window) || B < 1) return SINKATTN_ERR_INVALID_ARG;
  if (!k_new || !v_new || !cache_seqlens || !k_cache || !v_cache) return SINKATTN_ERR_INVALID_ARG;
  if (!a16(k_new) || !a16(v_new) || !a16(k_cache) || !a16(v_cache)) return SINKATTN_ERR_INVALID_ARG;
  const int row16 = Hkv * D * (dt == SINKATTN_FP32 ? 4 : 2) / 16;
  cache_append_kernel<<<B, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), cache_seqlens,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), n_sink + window, n_sink, window,
      row16);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

extern "C" int sinkattn_cache_fill(sinkattn_dtype dt, int n_seq, int T_tot, int Hkv, int D,
                                   int n_sink, int window, const int32_t* cu_seqlens,
                                   const void* k, const void* v, void* k_cache, void* v_cache,
                                   int32_t* cache_seqlens_out, sinkattn_stream_t stream) {
  if (!cache_args_ok(dt, Hkv, D, n_sink, window) || n_seq < 1 || T_tot < 0)
    return SINKATTN_ERR_INVALID_ARG;
  if (!cu_seqlens || !k_cache || !v_cache || (T_tot > 0 && (!k || !v)))
    return SINKATTN_ERR_INVALID_ARG;
  if (!a16(k_cache) || !a16(v_cache) || (k && !a16(k)) || (v && !a16(v)))
    return SINKATTN_ERR_INVALID_ARG;
  const int row16 = Hkv * D * (dt == SINKATTN_FP32 ? 4 : 2) / 16;
  const long long warps = T_tot > 0 ? T_tot : 1;
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  cache_fill_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), cu_seqlens, n_seq, T_tot,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), cache_seqlens_out,
      n_sink + window, n_sink, window, row16);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

extern "C" int sinkattn_cache_append_fp8(int B, int Hkv, int D, int n_sink, int window,
                                         const void* k_new, const void* v_new,
                                         const int32_t* cache_seqlens, void* k_sink,
                                         void* v_sink, void* k_win, void* v_win,
                                         const float* k_scale, const float* v_scale,
                                         sinkattn_stream_t stream) {
  if (!cache_args_ok(SINKATTN_BF16, Hkv, D, n_sink, window) || B < 1)
    return SINKATTN_ERR_INVALID_ARG;
  if (!k_new || !v_new || !cache_seqlens || !a16(k_new) || !a16(v_new))
    return SINKATTN_ERR_INVALID_ARG;
  if (n_sink > 0 && (!k_sink || !v_sink || !a16(k_sink) || !a16(v_sink)))
    return SINKATTN_ERR_INVALID_ARG;
  if (window > 0 && (!k_win || !v_win || !k_scale || !v_scale || !a16(k_win) || !a16(v_win)))
    return SINKATTN_ERR_INVALID_ARG;
  cache_append_fp8_kernel<<<B, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), cache_seqlens,
      static_cast<uint4*>(k_sink), static_cast<uint4*>(v_sink), static_cast<uint2*>(k_win),
      static_cast<uint2*>(v_win), k_scale, v_scale, Hkv, D, n_sink, window);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}
