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
#include <type_traits>

#include "internal.h"

namespace sk {

namespace {

constexpr int kPreThreads = 256;
constexpr int kPreTokens = 4;    // tokens per CTA
constexpr int kPreSlots = 8;     // rows per lane group in flight (each of O and dO)
constexpr int kMaxHeads = 256;
constexpr int kRedThreads = 256;

// <a, b> over one 16-byte chunk of each row.
template <typename T>
__device__ __forceinline__ float chunk_dot(const uint4& a, const uint4& b) {
  if constexpr (sizeof(T) == 2) {
    using E = std::conditional_t<std::is_same_v<T, __half>, ElemF16, ElemBf16>;
    const uint32_t* x = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* y = reinterpret_cast<const uint32_t*>(&b);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 u = E::widen(x[i]), v = E::widen(y[i]);
      s = fmaf(u.x, v.x, s);
      s = fmaf(u.y, v.y, s);
    }
    return s;
  } else {
    float s = __uint_as_float(a.x) * __uint_as_float(b.x);
    s = fmaf(__uint_as_float(a.y), __uint_as_float(b.y), s);
    s = fmaf(__uint_as_float(a.z), __uint_as_float(b.z), s);
    return fmaf(__uint_as_float(a.w), __uint_as_float(b.w), s);
  }
}

// The CTA's rows (token, head) are contiguous in memory: row r of the CTA is
// token t0 + r / Hq, head r % Hq.  A row is L = D sizeof(T) / 16 chunks of 16
// bytes, so one warp load instruction covers 32 / L rows (one chunk a lane);
// a warp phase issues kPreSlots such loads of O and of dO before any
// arithmetic (8 KB in flight per warp), reduces each row over its L lanes,
// and lane (row group, i < kPreSlots) finishes the row of slot i, whose LSE
// (and upstream gate gradient) it loaded beside the chunks.
template <typename T, int D>
__global__ void __launch_bounds__(kPreThreads) preprocess_kernel(
    const T* out, const T* dout, const float* lse, const float* sink, const float* dss,
    float* delta, float* lse2, float* part, int T_tot, int Hq) {
  constexpr int L = D * (int)sizeof(T) / 16;  // 8, 16 or 32
  static_assert(L >= kPreSlots && L <= 32, "row layout");
  constexpr int RPI = 32 / L;                 // rows per load instruction
  constexpr int RPP = RPI * kPreSlots;        // rows per warp phase
  __shared__ float contrib_s[kPreTokens * kMaxHeads];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / L, li = lane % L;
  const int t0 = blockIdx.x * kPreTokens;
  const int nt = min(kPreTokens, T_tot - t0);
  const int R = nt * Hq;
  const long long row0 = (long long)t0 * Hq;
  const uint4* O = reinterpret_cast<const uint4*>(out) + row0 * L;
  const uint4* dO = reinterpret_cast<const uint4*>(dout) + row0 * L;
  for (int ph = warp * RPP; ph < R; ph += (kPreThreads / 32) * RPP) {
    uint4 o[kPreSlots], d[kPreSlots];
#pragma unroll
    for (int s = 0; s < kPreSlots; ++s) {
      const int r = min(ph + s * RPI + sub, R - 1);
      o[s] = __ldg(O + (long long)r * L + li);
      d[s] = __ldg(dO + (long long)r * L + li);
    }
    // the row this lane finishes: slot li of its row group
    const int my_r = ph + li * RPI + sub;
    const bool mine_ok = li < kPreSlots && my_r < R;
    const int rr = min(my_r, R - 1);
    const float l = __ldg(lse + row0 + rr);
    const float g = dss ? __ldg(dss + row0 + rr) : 0.f;
    float acc[kPreSlots];
#pragma unroll
    for (int s = 0; s < kPreSlots; ++s) acc[s] = chunk_dot<T>(o[s], d[s]);
#pragma unroll
    for (int off = L / 2; off > 0; off >>= 1)
#pragma unroll
      for (int s = 0; s < kPreSlots; ++s) acc[s] += __shfl_xor_sync(0xffffffffu, acc[s], off);
    float dot = 0.f;
#pragma unroll
    for (int s = 0; s < kPreSlots; ++s) dot = (li == s) ? acc[s] : dot;
    if (mine_ok) {
      const int t = t0 + my_r / Hq, h = my_r % Hq;
      float dl = dot, contrib = 0.f;
      if (sink) {
        const float ps = __expf(__ldg(sink + h) - l);  // p_sink
        if (dss) {
          contrib = -ps * (dot + g * (1.f - ps));
          dl = dot - g * ps;
        } else {
          contrib = -dot * ps;  // -Delta * p_sink
        }
      }
      delta[(long long)h * T_tot + t] = dl;
      lse2[(long long)h * T_tot + t] = (l == -INFINITY) ? INFINITY : l * kLog2e;
      contrib_s[my_r] = contrib;
    }
  }
  if (!sink) return;  // uniform over the CTA
  __syncthreads();
  // the CTA's partial of head h: its tokens in order; head-major partials
  for (int h = threadIdx.x; h < Hq; h += kPreThreads) {
    float s = 0.f;
    for (int tt = 0; tt < nt; ++tt) s += contrib_s[tt * Hq + h];
    part[(long long)h * gridDim.x + blockIdx.x] = s;
  }
}

// dsink[h] = sum of head h's partials [n_blocks]: one CTA per head, each
// thread sums a fixed strided subset in order, then a fixed tree.
__global__ void __launch_bounds__(kRedThreads) dsink_reduce_kernel(const float* part, int n_blocks,
                                                                  float* dsink) {
  __shared__ float red[kRedThreads];
  const int h = blockIdx.x;
  const float* p = part + (long long)h * n_blocks;
  float s = 0.f;
  for (int b = threadIdx.x; b < n_blocks; b += kRedThreads) s += __ldg(p + b);
  red[threadIdx.x] = s;
  __syncthreads();
#pragma unroll
  for (int w = kRedThreads / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) dsink[h] = red[0];
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
  } else if (p.dt == SINKATTN_FP16) {
    const auto* o = static_cast<const __half*>(b.out);
    const auto* d = static_cast<const __half*>(b.dout);
    if (p.D == 64)
      preprocess_kernel<__half, 64><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
    else
      preprocess_kernel<__half, 128><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
  } else {
    const auto* o = static_cast<const float*>(b.out);
    const auto* d = static_cast<const float*>(b.dout);
    if (p.D == 64)
      preprocess_kernel<float, 64><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
    else
      preprocess_kernel<float, 128><<<nb, kPreThreads, 0, stream>>>(o, d, b.lse, p.sink, b.dss, b.delta, b.lse2, b.dsink_part, p.T_tot, p.Hq);
  }
  if (p.sink && b.dsink)
    dsink_reduce_kernel<<<p.Hq, kRedThreads, 0, stream>>>(b.dsink_part, nb, b.dsink);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk
