// Backward preprocess and dsink (page "Attention Sink, Learnable Sink and
// dsink", section 7 and section 10):
//   Delta_ih = sum_d dO_ihd * O_ihd                 (fp32, from the sink-scaled O)
//   p_sink   = exp(a_h - L_new,ih)                  (section 10: avoids 1 - sink_s)
//   dsink_h  = -sum_i Delta_ih * p_sink,ih          (every query counted once)
// Delta and LSE_new * log2(e) are written head-major ([Hq][T_tot]) so the
// backward kernels read a query tile's values with coalesced loads; a row
// with LSE = -inf (it sees no key and has no sink) gets +inf there, which
// makes every recomputed probability of the row exactly 0.
// An upstream gradient g_ih = dL/d sink_s,ih (page "Attention Sink and the
// native MoE in attention layers", lvdousha26.github.io, sections 4-5: the
// head-importance statistic and the auxiliary balance loss are functions of
// the gate sink_s) adds g to dL/dPhat_j of every real key, since
// sink_s = sum_j Phat_j.  The softmax backward then needs
//   mu_ih    = Delta_ih + g_ih * sink_s,ih
//   dx_j     = Phat_j (<dO, V_j> + g - mu) = Phat_j (<dO, V_j> - Delta'),
//   Delta'   = Delta - g * p_sink                   (1 - sink_s = p_sink)
//   dsink_h  = -sum_i p_sink (Delta + g * (1 - p_sink))
// so the key-tile kernels are unchanged: they read Delta' in place of Delta.
// Each CTA owns a fixed range of tokens and writes one partial per head; a
// second kernel sums the partials in a fixed order, so dsink is bitwise
// deterministic.  HBM-bound: it streams O and dO once.
#include "internal.h"

namespace sk {

namespace {

constexpr int kPreThreads = 256;
constexpr int kPreTokens = 16;   // tokens per CTA
constexpr int kRows = 8;         // rows in flight per warp
constexpr int kMaxHeads = 256;

// D/32 elements of one row held by a lane, converted to fp32.
template <typename T, int D>
struct RowFrag {
  static constexpr int E = D / 32;
  float v[E];
  __device__ __forceinline__ void load(const T* row, int lane) {
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(row) + lane * E;
      if constexpr (E == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
      } else {
        const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(p));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        v[0] = a.x; v[1] = a.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = __ldg(row + lane * E + e);
    }
  }
};

// One warp owns one head of the CTA's tokens, kRows rows at a time: all loads
// of a group are issued before any reduction, so each lane keeps 2 kRows loads
// in flight.  Delta and LSE2 of consecutive tokens land in consecutive words
// of the head-major arrays; the warp also writes the CTA's dsink partial for
// its head (fixed order, so dsink is bitwise deterministic).
template <typename T, int D>
__global__ void __launch_bounds__(kPreThreads) preprocess_kernel(
    const T* out, const T* dout, const float* lse, const float* sink, const float* dss,
    float* delta, float* lse2, float* part, int T_tot, int Hq) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kPreTokens;
  for (int h = warp; h < Hq; h += kPreThreads / 32) {
    const float a = sink ? __ldg(sink + h) : 0.f;
    float dsum = 0.f;
#pragma unroll
    for (int g = 0; g < kPreTokens; g += kRows) {
      RowFrag<T, D> o[kRows], d[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int t = min(t0 + g + r, T_tot - 1);
        const long long row = ((long long)t * Hq + h) * D;
        o[r].load(out + row, lane);
        d[r].load(dout + row, lane);
      }
      float acc[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        acc[r] = 0.f;
#pragma unroll
        for (int e = 0; e < RowFrag<T, D>::E; ++e) acc[r] += o[r].v[e] * d[r].v[e];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int r = 0; r < kRows; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
      // lane r (< kRows) writes token t0 + g + r
      float mine = 0.f;
#pragma unroll
      for (int r = 0; r < kRows; ++r) mine = (lane == r) ? acc[r] : mine;
      const int t = t0 + g + lane;
      float contrib = 0.f;
      if (lane < kRows && t < T_tot) {
        const float l = __ldg(lse + (long long)t * Hq + h);
        float dl = mine;
        if (sink) {
          const float ps = __expf(a - l);  // p_sink
          if (dss) {
            const float g = __ldg(dss + (long long)t * Hq + h);
            contrib = -ps * (mine + g * (1.f - ps));
            dl = mine - g * ps;
          } else {
            contrib = -mine * ps;  // -Delta * p_sink
          }
        }
        delta[(long long)h * T_tot + t] = dl;
        lse2[(long long)h * T_tot + t] = (l == -INFINITY) ? INFINITY : l * kLog2e;
      }
      dsum += contrib;
    }
    if (sink) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      if (lane == 0) part[(long long)blockIdx.x * Hq + h] = dsum;
    }
  }
}

// dsink[h] = sum of the per-CTA partials: one warp per head, lanes stride
// over the partials in a fixed order, then a fixed butterfly.
__global__ void dsink_reduce_kernel(const float* part, int n_blocks, int Hq, float* dsink) {
  const int h = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= Hq) return;
  float s = 0.f;
  for (int b = lane; b < n_blocks; b += 32) s += part[(long long)b * Hq + h];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) dsink[h] = s;
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
      preprocess_kernel<__nv_bfloat16, 64><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
    else
      preprocess_kernel<__nv_bfloat16, 128><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
  } else {
    const auto* o = static_cast<const float*>(b.out);
    const auto* d = static_cast<const float*>(b.dout);
    if (p.D == 64)
      preprocess_kernel<float, 64><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
    else
      preprocess_kernel<float, 128><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
  }
  if (p.sink && b.dsink)
    dsink_reduce_kernel<<<(p.Hq + 3) / 4, 128, 0, stream>>>(b.dsink_part, nb, p.Hq, b.dsink);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk
