// Backward preprocess and dsink (page "Attention Sink, Learnable Sink and
// dsink", section 7 and section 10):
//   Delta_ih = sum_d dO_ihd * O_ihd                 (fp32, from the sink-scaled O)
//   p_sink   = exp(a_h - L_new,ih)                  (section 10: avoids 1 - sink_s)
//   dsink_h  = -sum_i Delta_ih * p_sink,ih          (every query counted once)
// Delta and LSE_new * log2(e) are written head-major ([Hq][T_tot]) so the
// backward kernels read a query tile's values with coalesced loads; a row
// with LSE = -inf (it sees no key and has no sink) gets +inf there, which
// makes every recomputed probability of the row exactly 0.
// Each CTA owns a fixed range of tokens and writes one partial per head; a
// second kernel sums the partials in a fixed order, so dsink is bitwise
// deterministic.  HBM-bound: it streams O and dO once.
#include "internal.h"

namespace sk {

namespace {

constexpr int kPreThreads = 256;
constexpr int kPreTokens = 64;  // tokens per CTA
constexpr int kMaxHeads = 256;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T, int D>
__device__ __forceinline__ float row_dot(const T* a, const T* b, int lane) {
  float s = 0.f;
  if constexpr (sizeof(T) == 2) {
    // D/32 bf16 per lane, loaded as one 4- or 8-byte vector
    constexpr int E = D / 32;
    const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(a) + lane * E;
    const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(b) + lane * E;
    if constexpr (E == 4) {
      const uint2 ua = *reinterpret_cast<const uint2*>(pa);
      const uint2 ub = *reinterpret_cast<const uint2*>(pb);
      const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&ua);
      const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&ub);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 fx = __bfloat1622float2(x[e]), fy = __bfloat1622float2(y[e]);
        s += fx.x * fy.x + fx.y * fy.y;
      }
    } else {
      const uint32_t ua = *reinterpret_cast<const uint32_t*>(pa);
      const uint32_t ub = *reinterpret_cast<const uint32_t*>(pb);
      const float2 fx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ua));
      const float2 fy = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ub));
      s = fx.x * fy.x + fx.y * fy.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) s += a[lane + 32 * e] * b[lane + 32 * e];
  }
  return warp_sum(s);
}

template <typename T, int D>
__global__ void __launch_bounds__(kPreThreads) preprocess_kernel(
    const T* out, const T* dout, const float* lse, const float* sink, float* delta,
    float* lse2, float* part, int T_tot, int Hq) {
  __shared__ float wpart[kPreThreads / 32][kMaxHeads];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = kPreThreads / 32;
  for (int hh = threadIdx.x; hh < NW * kMaxHeads; hh += kPreThreads)
    (&wpart[0][0])[hh] = 0.f;
  __syncthreads();
  const int t0 = blockIdx.x * kPreTokens;
  const int t1 = min(t0 + kPreTokens, T_tot);
  const long long r0 = (long long)t0 * Hq, r1 = (long long)t1 * Hq;
  // warp w handles rows r0 + w, r0 + w + NW, ... in order (deterministic)
  for (long long r = r0 + warp; r < r1; r += NW) {
    const float d = row_dot<T, D>(out + r * D, dout + r * D, lane);
    if (lane == 0) {
      const int h = (int)(r % Hq);
      const long long t = r / Hq;
      const float l = lse[r];
      delta[(long long)h * T_tot + t] = d;
      lse2[(long long)h * T_tot + t] = (l == -INFINITY) ? INFINITY : l * kLog2e;
      if (sink) {
        const float ps = __expf(sink[h] - lse[r]);
        wpart[warp][h] -= d * ps;
      }
    }
  }
  __syncthreads();
  if (sink) {
    for (int h = threadIdx.x; h < Hq; h += kPreThreads) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) s += wpart[w][h];
      part[(long long)blockIdx.x * Hq + h] = s;
    }
  }
}

__global__ void dsink_reduce_kernel(const float* part, int n_blocks, int Hq, float* dsink) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= Hq) return;
  float s = 0.f;
  for (int b = 0; b < n_blocks; ++b) s += part[(long long)b * Hq + h];
  dsink[h] = s;
}

}  // namespace

int preprocess_blocks(int T_tot) { return (T_tot + kPreTokens - 1) / kPreTokens; }

int launch_bwd_preprocess(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  if (p.Hq > kMaxHeads) return SINKATTN_ERR_UNSUPPORTED;
  const int nb = preprocess_blocks(p.T_tot);
  if (p.dt == SINKATTN_BF16) {
    const auto* o = static_cast<const __nv_bfloat16*>(b.out);
    const auto* d = static_cast<const __nv_bfloat16*>(b.dout);
    if (p.D == 64)
      preprocess_kernel<__nv_bfloat16, 64><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
    else
      preprocess_kernel<__nv_bfloat16, 128><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
  } else {
    const auto* o = static_cast<const float*>(b.out);
    const auto* d = static_cast<const float*>(b.dout);
    if (p.D == 64)
      preprocess_kernel<float, 64><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
    else
      preprocess_kernel<float, 128><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
  }
  if (p.sink && b.dsink)
    dsink_reduce_kernel<<<(p.Hq + 127) / 128, 128, 0, stream>>>(b.dsink_part, nb, p.Hq, b.dsink);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk
