// Split-KV decode over a StreamingLLM ring-buffer KV cache (page
// "Attention Sink / StreamingLLM" interview notes: the cache is a fixed
// segment of initial sink tokens plus a sliding window of recent tokens).
// Slot s of sequence b holds a valid token iff s < min(cache_seqlens[b], S):
// the n_sink sink slots fill first, then the window slots, and once the
// window has wrapped every slot is valid.  No positional encoding is applied
// here, so the ring head's position does not matter.
//
// Stage 1 (one CTA per (split, KV head, sequence)): stream the split's K and
// V rows once with 16-byte coalesced loads; the G = Hq/Hkv query heads of the
// KV head share every loaded row.  Each CTA writes (m, l, acc[D]) per head.
// Stage 2: merge the splits with the sink column (page "Attention Sink,
// Learnable Sink and dsink", section 4: e^{a_h} joins the denominator, the
// sink value is zero) and write O, LSE_new and sink_s.
#include "internal.h"

namespace sk {

namespace {

constexpr int kDecThreads = 256;

template <int D>
struct DecGeom {
  static constexpr int LPR = D / 8;          // lanes per K/V row (8 bf16 = 16 B each)
  static constexpr int NGRP = kDecThreads / LPR;  // rows in flight per pass
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]) {
  if constexpr (sizeof(T) == 2) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    bf16x8_to_f32(u, f);
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}

// smem: scores/probabilities [G][chunk], group accumulators [NGRP][G][D]
template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(DecodeProblem p, int chunk) {
  using Geo = DecGeom<D>;
  constexpr int LPR = Geo::LPR, NGRP = Geo::NGRP;
  extern __shared__ float dsm[];
  float* sc = dsm;                       // [G][chunk]
  float* red = dsm + G * chunk;          // [NGRP][G][D]
  __shared__ float m_s[G], l_s[G];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int S = p.n_sink + p.window;
  const int n_valid = min(max(p.cache_seqlens[b], 0), S);
  const int s0 = split * chunk;
  const int s1 = min(s0 + chunk, n_valid);
  const int n = max(s1 - s0, 0);
  const int tid = threadIdx.x, grp = tid / LPR, gl = tid % LPR;
  const int c0 = gl * 8;  // this lane's 8 columns
  const float scale_log2 = p.scale * kLog2e;

  const T* qb = static_cast<const T*>(p.q) + ((long long)b * p.Hq + kvh * G) * D;
  float qv[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    load8<T>(qb + h * D + c0, qv[h]);
#pragma unroll
    for (int c = 0; c < 8; ++c) qv[h][c] *= scale_log2;
  }
  const long long row_stride = (long long)p.Hkv * D;
  const T* kbase = static_cast<const T*>(p.k_cache) + ((long long)b * S * p.Hkv + kvh) * D + c0;
  const T* vbase = static_cast<const T*>(p.v_cache) + ((long long)b * S * p.Hkv + kvh) * D + c0;

  // stage A: scores for this split's slots
  // every lane runs the same number of passes (the shuffles below use the
  // full warp mask); lanes past the split's last slot compute but store nothing
  constexpr int U = 4;
  for (int pass = 0; pass * NGRP * U < n; ++pass) {
    const int base = pass * NGRP * U + grp;
    float kf[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int sl = base + u * NGRP;
      if (sl < n) load8<T>(kbase + (long long)(s0 + sl) * row_stride, kf[u]);
      else
#pragma unroll
        for (int c = 0; c < 8; ++c) kf[u][c] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int sl = base + u * NGRP;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) s += qv[h][c] * kf[u][c];
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (gl == 0 && sl < n) sc[h * chunk + sl] = s;
      }
    }
  }
  __syncthreads();
  // stage B: per-head max and exponentials (warp h handles head h)
  const int warp = tid >> 5, lane = tid & 31;
  for (int h = warp; h < G; h += kDecThreads / 32) {
    float m = -INFINITY;
    for (int i = lane; i < n; i += 32) m = fmaxf(m, sc[h * chunk + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float e = exp2f(sc[h * chunk + i] - m);
      sc[h * chunk + i] = e;
      l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) { m_s[h] = m; l_s[h] = l; }
  }
  __syncthreads();
  // stage C: probability-weighted V rows
  float acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[h][c] = 0.f;
  for (int pass = 0; pass * NGRP * U < n; ++pass) {
    const int base = pass * NGRP * U + grp;
    float vf[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int sl = base + u * NGRP;
      if (sl < n) load8<T>(vbase + (long long)(s0 + sl) * row_stride, vf[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int sl = base + u * NGRP;
      if (sl < n) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr = sc[h * chunk + sl];
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[h][c] += pr * vf[u][c];
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < 8; ++c) red[((long long)grp * G + h) * D + c0 + c] = acc[h][c];
  __syncthreads();
  // reduce over groups (fixed order) and write the split's partial
  float* part = p.part + (((long long)b * p.Hq + kvh * G) * gridDim.x + split) * (D + 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int h = i / D, d = i % D;
    float s = 0.f;
    for (int g = 0; g < NGRP; ++g) s += red[((long long)g * G + h) * D + d];
    part[(long long)h * gridDim.x * (D + 2) + d] = s;
  }
  if (tid < G) {
    float* ph = part + (long long)tid * gridDim.x * (D + 2);
    ph[D] = n > 0 ? m_s[tid] : -INFINITY;
    ph[D + 1] = n > 0 ? l_s[tid] : 0.f;
  }
}

// bf16 variant of the split kernel: the split's K and V rows are fetched
// into shared memory by TMA bulk tensor copies (every byte requested at once,
// no per-thread load latency), then scored and accumulated from shared memory
// exactly as above.  A split longer than kChunkRows is processed in pieces
// with an online rescale.
constexpr int kChunkRows = 128;

template <int D, int G>
struct TmaDecGeom {
  static constexpr int DH = D / 64;
  static constexpr int ROWS_BYTES = kChunkRows * 128;         // one 64-column half
  static constexpr int KV_BYTES = DH * ROWS_BYTES;            // K (or V) piece
  static constexpr int OFF_K = 0, OFF_V = KV_BYTES, OFF_SC = 2 * KV_BYTES;
  static constexpr int OFF_RED = OFF_SC + G * kChunkRows * 4;
  static constexpr int LPR = D / 8, NGRP = kDecThreads / LPR;
  static constexpr int OFF_BAR = OFF_RED + NGRP * G * D * 4;
  static constexpr int SMEM = OFF_BAR + 64 + 128;
};

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_tma_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    DecodeProblem p, int chunk) {
  using Geo = TmaDecGeom<D, G>;
  constexpr int LPR = Geo::LPR, NGRP = Geo::NGRP, DH = Geo::DH;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) & ~uintptr_t(127));
  float* sc = reinterpret_cast<float*>(sm + Geo::OFF_SC);    // [G][kChunkRows]
  float* red = reinterpret_cast<float*>(sm + Geo::OFF_RED);  // [NGRP][G][D]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Geo::OFF_BAR);
  __shared__ float m_s[G], l_s[G], f_s[G];
  __shared__ int abort_s;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int S = p.n_sink + p.window;
  const int n_valid = min(max(p.cache_seqlens[b], 0), S);
  const int s0 = split * chunk;
  const int n = max(min(s0 + chunk, n_valid) - s0, 0);
  const int tid = threadIdx.x, grp = tid / LPR, gl = tid % LPR;
  const int c0 = gl * 8, hf = c0 / 64, cin = c0 % 64;
  const int warp = tid >> 5, lane = tid & 31;
  const float scale_log2 = p.scale * kLog2e;

  if (tid == 0) {
    mbar_init(bar, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (tid < G) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
  __syncthreads();

  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) + ((long long)b * p.Hq + kvh * G) * D;
  float qv[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    load8<__nv_bfloat16>(qb + h * D + c0, qv[h]);
#pragma unroll
    for (int c = 0; c < 8; ++c) qv[h][c] *= scale_log2;
  }
  float acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[h][c] = 0.f;

  const int n_pieces = (n + kChunkRows - 1) / kChunkRows;
  for (int pc = 0; pc < n_pieces; ++pc) {
    const int base = pc * kChunkRows;
    const int rows = min(kChunkRows, n - base);
    if (tid == 0) {
      mbar_expect_tx(bar, 2 * Geo::KV_BYTES);
      const int row0 = b * S + s0 + base;  // rows past the split are read but unused
      for (int h = 0; h < DH; ++h) {
        tma_load_3d(sm + Geo::OFF_K + h * Geo::ROWS_BYTES, &tmap_k, bar, h * 64, kvh, row0);
        tma_load_3d(sm + Geo::OFF_V + h * Geo::ROWS_BYTES, &tmap_v, bar, h * 64, kvh, row0);
      }
    }
    if (!mbar_wait(bar, pc & 1, &abort_s, p.status)) break;
    // scores of this piece
    for (int r = grp; r < kChunkRows; r += NGRP) {
      float kf[8];
      const uint4 u = *reinterpret_cast<const uint4*>(sm + Geo::OFF_K + hf * Geo::ROWS_BYTES + r * 128 + cin * 2);
      bf16x8_to_f32(u, kf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) s += qv[h][c] * kf[c];
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (gl == 0 && r < rows) sc[h * kChunkRows + r] = s;
      }
    }
    __syncthreads();
    // running max / sum per head (warp h handles head h)
    for (int h = warp; h < G; h += kDecThreads / 32) {
      float m = -INFINITY;
      for (int i = lane; i < rows; i += 32) m = fmaxf(m, sc[h * kChunkRows + i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float mo = m_s[h];
      const float mn = fmaxf(mo, m);
      float l = 0.f;
      for (int i = lane; i < rows; i += 32) {
        const float e = exp2f(sc[h * kChunkRows + i] - mn);
        sc[h * kChunkRows + i] = e;
        l += e;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) {
        const float f = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
        f_s[h] = f;
        l_s[h] = l_s[h] * f + l;
        m_s[h] = mn;
      }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float f = f_s[h];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[h][c] *= f;
    }
    for (int r = grp; r < rows; r += NGRP) {
      float vf[8];
      const uint4 u = *reinterpret_cast<const uint4*>(sm + Geo::OFF_V + hf * Geo::ROWS_BYTES + r * 128 + cin * 2);
      bf16x8_to_f32(u, vf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pr = sc[h * kChunkRows + r];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[h][c] += pr * vf[c];
      }
    }
    __syncthreads();  // the piece's buffers may be refilled
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < 8; ++c) red[((long long)grp * G + h) * D + c0 + c] = acc[h][c];
  __syncthreads();
  float* part = p.part + (((long long)b * p.Hq + kvh * G) * gridDim.x + split) * (D + 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int h = i / D, d = i % D;
    float s = 0.f;
    for (int g = 0; g < NGRP; ++g) s += red[((long long)g * G + h) * D + d];
    part[(long long)h * gridDim.x * (D + 2) + d] = s;
  }
  if (tid < G) {
    float* ph = part + (long long)tid * gridDim.x * (D + 2);
    ph[D] = n > 0 ? m_s[tid] : -INFINITY;
    ph[D + 1] = n > 0 ? l_s[tid] : 0.f;
  }
}

// Merge splits + sink.  One CTA per (head, sequence), D threads.
template <typename T, int D>
__global__ void decode_combine_kernel(DecodeProblem p, int n_splits) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const float* part = p.part + ((long long)b * p.Hq + h) * n_splits * (D + 2);
  const float a2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
  float mt = a2;
  for (int i = 0; i < n_splits; ++i) mt = fmaxf(mt, part[i * (D + 2) + D]);
  float l = 0.f, o = 0.f;
  if (mt != -INFINITY) {
    for (int i = 0; i < n_splits; ++i) {
      const float mi = part[i * (D + 2) + D];
      if (mi == -INFINITY) continue;
      const float w = exp2f(mi - mt);
      l += part[i * (D + 2) + D + 1] * w;
      o += part[i * (D + 2) + d] * w;
    }
  }
  const float den = l + (p.sink && mt != -INFINITY ? exp2f(a2 - mt) : 0.f);
  const long long row = (long long)b * p.Hq + h;
  const float ov = den > 0.f ? o / den : 0.f;
  if constexpr (sizeof(T) == 2)
    static_cast<__nv_bfloat16*>(p.out)[row * D + d] = __float2bfloat16_rn(ov);
  else
    static_cast<float*>(p.out)[row * D + d] = ov;
  if (d == 0) {
    p.lse[row] = den > 0.f ? (mt + log2f(den)) * kLn2 : -INFINITY;
    if (p.sink_s) p.sink_s[row] = den > 0.f ? l / den : 0.f;
  }
}

template <int D, int G>
int launch_tma(const DecodeProblem& p, int chunk, cudaStream_t stream) {
  using Geo = TmaDecGeom<D, G>;
  const int S = p.n_sink + p.window;
  CUtensorMap mk, mv;
  if (!make_tmap_3d_plain(&mk, p.k_cache, p.B * S, p.Hkv, D, 1, kChunkRows) ||
      !make_tmap_3d_plain(&mv, p.v_cache, p.B * S, p.Hkv, D, 1, kChunkRows))
    return SINKATTN_ERR_CUDA;
  auto kern = decode_tma_kernel<D, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  dim3 grid(p.num_splits, p.Hkv, p.B);
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, kDecThreads, Geo::SMEM, stream>>>(mk, mv, p, chunk);
  record_stop(SINKATTN_KERNEL_DECODE, stream);
  dim3 g2(p.Hq, p.B);
  decode_combine_kernel<__nv_bfloat16, D><<<g2, D, 0, stream>>>(p, p.num_splits);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

template <typename T, int D, int G>
int launch_split(const DecodeProblem& p, int chunk, cudaStream_t stream) {
  if constexpr (sizeof(T) == 2) return launch_tma<D, G>(p, chunk, stream);
  using Geo = DecGeom<D>;
  const size_t smem = sizeof(float) * ((size_t)G * chunk + (size_t)Geo::NGRP * G * D);
  auto kern = decode_split_kernel<T, D, G>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  dim3 grid(p.num_splits, p.Hkv, p.B);
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, kDecThreads, smem, stream>>>(p, chunk);
  record_stop(SINKATTN_KERNEL_DECODE, stream);
  dim3 g2(p.Hq, p.B);
  decode_combine_kernel<T, D><<<g2, D, 0, stream>>>(p, p.num_splits);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

template <typename T, int D>
int dispatch_g(const DecodeProblem& p, int chunk, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return launch_split<T, D, 1>(p, chunk, stream);
    case 2: return launch_split<T, D, 2>(p, chunk, stream);
    case 4: return launch_split<T, D, 4>(p, chunk, stream);
    case 8: return launch_split<T, D, 8>(p, chunk, stream);
    default: return SINKATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_decode(const DecodeProblem& p, cudaStream_t stream) {
  const int S = p.n_sink + p.window;
  const int chunk = (S + p.num_splits - 1) / p.num_splits;
  if (p.dt == SINKATTN_BF16)
    return p.D == 64 ? dispatch_g<__nv_bfloat16, 64>(p, chunk, stream)
                     : dispatch_g<__nv_bfloat16, 128>(p, chunk, stream);
  return p.D == 64 ? dispatch_g<float, 64>(p, chunk, stream)
                   : dispatch_g<float, 128>(p, chunk, stream);
}

}  // namespace sk
