// Head importance from the gate (page "Attention Sink and the native MoE in
// attention layers", lvdousha26.github.io, section 4): the gate of query
// token t and head h is the mass on real tokens, G = sigma(LSE - sink) =
// sink_s, and a head's importance is its mean gate over the token set,
//   Imp_h = (1 / T_tot) * sum_t sink_s[t, h].
// Section 5's auxiliary balance loss is a function of these Hq numbers; its
// gradient reaches the attention through d sink_s = dL/dImp_h / T_tot, which
// sinkattn_bwd_ex takes.
//
// Two deterministic passes: each CTA of the first owns a fixed token range
// and writes a float64 partial per head (coalesced row reads: thread i reads
// head i % Hq of rows i / Hq, i / Hq + R, ...); the second sums the partials
// per head in a fixed order.  The partition depends only on (T_tot, Hq), so
// the result is bitwise reproducible.  HBM-bound: sink_s is read once.
#include <type_traits>

#include "internal.h"

namespace sk {

namespace {

constexpr int kGateMaxHeads = 256;
constexpr int kGateMaxBlocks = 1024;
constexpr int kGateMinRows = 32;   // tokens per CTA at least
constexpr int kGateThreads = 256;

int gate_blocks(int T_tot) {
  const int b = (T_tot + kGateMinRows - 1) / kGateMinRows;
  return b < kGateMaxBlocks ? b : kGateMaxBlocks;
}

// blockDim = R * Hq with R = 256 / Hq rows in flight; thread (r, h).
__global__ void __launch_bounds__(kGateThreads) gate_partial_kernel(
    const float* __restrict__ sink_s, int T_tot, int Hq, int rows_per_blk, double* part) {
  __shared__ double red[kGateThreads];
  const int R = blockDim.x / Hq;
  const int r = threadIdx.x / Hq, h = threadIdx.x % Hq;
  const int t0 = blockIdx.x * rows_per_blk;
  const int t1 = min(T_tot, t0 + rows_per_blk);
  double acc = 0.0;
  int t = t0 + r;
  // four independent loads in flight per thread
  for (; t + 3 * R < t1; t += 4 * R) {
    const float a = __ldg(sink_s + (long long)t * Hq + h);
    const float b = __ldg(sink_s + (long long)(t + R) * Hq + h);
    const float c = __ldg(sink_s + (long long)(t + 2 * R) * Hq + h);
    const float d = __ldg(sink_s + (long long)(t + 3 * R) * Hq + h);
    acc += ((double)a + (double)b) + ((double)c + (double)d);
  }
  for (; t < t1; t += R) acc += (double)__ldg(sink_s + (long long)t * Hq + h);
  red[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < Hq) {
    double s = 0.0;
    for (int i = 0; i < R; ++i) s += red[i * Hq + threadIdx.x];
    part[(long long)blockIdx.x * Hq + threadIdx.x] = s;
  }
}

// Imp_h = (sum of the partials of head h) / T_tot; one warp per head, lanes
// stride over the partials, then a fixed butterfly.
__global__ void gate_reduce_kernel(const double* part, int n_blocks, int Hq, int T_tot,
                                   float* imp) {
  const int h = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= Hq) return;
  double s = 0.0;
  for (int b = lane; b < n_blocks; b += 32) s += part[(long long)b * Hq + h];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) imp[h] = (float)(s / (double)T_tot);
}

// Gate of a sink-free model whose attention sink is the first token k_0 of
// each sequence (same page, section 5): G = sigma(LSE_not0 - x_0), x_0 =
// scale <q, k_0>.  With L = the sink-free forward's LSE over the visible set,
// L = logaddexp(LSE_not0, x_0), so G = 1 - e^(x_0 - L) = -expm1(x_0 - L): one
// dot product per (token, head) and the LSE the forward already wrote.  A row
// that does not see k_0 gets 1, a row that sees no key (L = -inf) gets 0.
// HBM-bound (reads Q once).  A warp streams one token's contiguous Q row
// [Hq, D] as 16-byte chunks, kGvInFlight per lane in flight; the CPH chunks
// of a head row sit in CPH adjacent lanes.  Their partial dot products are
// summed by a shuffle reduce-scatter, after which every lane holds whole
// dot products of max(1, kGvInFlight / CPH) heads (each head once per warp,
// or twice when CPH = 32) and finishes those heads alone: one expm1 per head,
// not one per lane and chunk.  CTA = kGvRows tokens of one sequence; the
// sequence's k_0 rows [Hkv, D] are staged once in shared memory when they fit
// kGvK0Smem bytes (else read through L1), so the loop's only global loads
// are Q's and the LSE.
constexpr int kGvRows = 16;
constexpr int kGvInFlight = 16;
constexpr int kGvK0Smem = 32 * 1024;

template <typename T>
__device__ __forceinline__ float dot16(const uint4& a, const uint4& b) {
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
    return __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
           __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
  }
}

// Reduce-scatter over lane masks M, M/2, ..., 1 of N values a lane: while
// N > 1 a step sends one half of the values to the partner lane (lane ^ M),
// keeps the other half and adds what arrives; once N = 1 a step is a plain
// butterfly add.  Afterwards v[0 .. N_end) are sums over the lane group of
// the values u0 .. u0 + N_end - 1, where u0 adds H for every halving step
// whose mask bit is set in the lane.
template <int M, int N>
struct ReduceScatter {
  template <int U>
  __device__ __forceinline__ static void run(float (&v)[U], int lane) {
    if constexpr (M >= 1) {
      if constexpr (N > 1) {
        constexpr int H = N / 2;
        const bool up = (lane & M) != 0;
#pragma unroll
        for (int k = 0; k < H; ++k) {
          const float send = up ? v[k] : v[k + H];
          const float keep = up ? v[k + H] : v[k];
          v[k] = keep + __shfl_xor_sync(0xffffffffu, send, M);
        }
        ReduceScatter<M / 2, H>::run(v, lane);
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
        ReduceScatter<M / 2, 1>::run(v, lane);
      }
    }
  }
  __device__ __forceinline__ static int first(int lane) {
    if constexpr (M >= 1 && N > 1)
      return ((lane & M) ? N / 2 : 0) + ReduceScatter<M / 2, N / 2>::first(lane);
    else
      return 0;
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(256, 2) gate_vanilla_kernel(GateVanillaArgs a) {
  constexpr int CPH = D * (int)sizeof(T) / 16;  // 16-byte chunks per head row: 8, 16 or 32
  constexpr int U = kGvInFlight;
  constexpr int NV = U / CPH > 0 ? U / CPH : 1;   // heads a lane finishes per batch
  constexpr int DUP = CPH / U > 0 ? CPH / U : 1;  // lanes holding the same head
  using RS = ReduceScatter<CPH / 2, U>;
  const int s = blockIdx.y;
  const int start = __ldg(a.cu + s), len = __ldg(a.cu + s + 1) - start;
  const int i0 = blockIdx.x * kGvRows;
  if (i0 >= len) return;  // uniform over the CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // block-sparse lists are indexed by query blocks numbered over all
  // sequences: count the blocks of the sequences before s
  __shared__ int red[8];
  int qb_base = 0;
  if (a.bi) {
    int acc = 0;
    for (int j = threadIdx.x; j < s; j += blockDim.x) {
      const int l = __ldg(a.cu + j + 1) - __ldg(a.cu + j);
      acc += (l + a.block_q - 1) / a.block_q;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 8; ++w) qb_base += red[w];
  }
  const int G = a.Hq / a.Hkv;
  const int n16 = a.Hq * CPH;  // chunks per token row
  const uint4* k0 = reinterpret_cast<const uint4*>(static_cast<const T*>(a.k) +
                                                   (long long)start * a.Hkv * D);
  extern __shared__ uint4 k0s[];
  const bool k0_in_smem = a.Hkv * CPH * 16 <= kGvK0Smem;
  if (k0_in_smem) {
    for (int j = threadIdx.x; j < a.Hkv * CPH; j += blockDim.x) k0s[j] = __ldg(k0 + j);
    __syncthreads();
  }
  // this lane's heads after the reduce-scatter: values u0 .. u0 + NV - 1 of
  // lane group g; the lane writes them when it is the group's first copy
  const int u0 = RS::first(lane), g = lane / CPH;
  const bool writer = (lane % DUP) == 0;
  for (int i = i0 + warp; i < min(len, i0 + kGvRows); i += 8) {
    const long long t = start + i;
    const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) + t * a.Hq * D);
    // is k_0 visible to query i (sequence-local)?  causal: always (0 <= i)
    const bool vis_band = a.window == 0 || a.n_sink > 0 || i < a.window;
    for (int c0 = 0; c0 < n16; c0 += 32 * U) {
      float lse_v[NV];
      int hv[NV];
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        hv[k] = (c0 + (u0 + k) * 32) / CPH + g;
        lse_v[k] = __ldg(a.lse + t * a.Hq + min(hv[k], a.Hq - 1));
      }
      float dot[U];
      {
        uint4 qv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) qv[u] = __ldg(qrow + min(c0 + u * 32 + lane, n16 - 1));
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = min(c0 + u * 32 + lane, n16 - 1);
          const int h = c / CPH;
          const int kc = (h / G) * CPH + (c - h * CPH);
          dot[u] = dot16<T>(qv[u], k0_in_smem ? k0s[kc] : __ldg(k0 + kc));
        }
      }
      RS::run(dot, lane);
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int h = hv[k];
        if (!writer || h >= a.Hq) continue;
        bool vis = vis_band;
        if (a.bi && vis) {
          const int qb = qb_base + i / a.block_q;
          vis = false;
          if (qb < a.n_qblk) {
            const int32_t* lst = a.bi + ((long long)(h / G) * a.n_qblk + qb) * a.max_blocks;
            for (int e = 0; e < a.max_blocks; ++e) vis |= __ldg(lst + e) == 0;
          }
        }
        const float l = lse_v[k];
        float gv;
        if (l == -INFINITY) gv = 0.f;
        else if (!vis) gv = 1.f;
        else gv = fmaxf(0.f, -expm1f(dot[k] * a.scale - l));
        a.gate[t * a.Hq + h] = gv;
      }
    }
  }
}

}  // namespace

int launch_gate_vanilla(const GateVanillaArgs& a, int dt, int D, int max_seqlen,
                        cudaStream_t stream) {
  const dim3 grid((max_seqlen + kGvRows - 1) / kGvRows, a.n_seq);
  const size_t k0_bytes = (size_t)a.Hkv * D * (dt == SINKATTN_FP32 ? 4 : 2);
  const size_t smem = k0_bytes <= (size_t)kGvK0Smem ? k0_bytes : 0;
  record_start(SINKATTN_KERNEL_GATE, stream);
  if (dt == SINKATTN_BF16) {
    if (D == 64) gate_vanilla_kernel<__nv_bfloat16, 64><<<grid, 256, smem, stream>>>(a);
    else gate_vanilla_kernel<__nv_bfloat16, 128><<<grid, 256, smem, stream>>>(a);
  } else if (dt == SINKATTN_FP16) {
    if (D == 64) gate_vanilla_kernel<__half, 64><<<grid, 256, smem, stream>>>(a);
    else gate_vanilla_kernel<__half, 128><<<grid, 256, smem, stream>>>(a);
  } else {
    if (D == 64) gate_vanilla_kernel<float, 64><<<grid, 256, smem, stream>>>(a);
    else gate_vanilla_kernel<float, 128><<<grid, 256, smem, stream>>>(a);
  }
  record_stop(SINKATTN_KERNEL_GATE, stream);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk

using namespace sk;

extern "C" size_t sinkattn_gate_importance_workspace_bytes(int T_tot, int Hq) {
  if (T_tot < 1 || Hq < 1 || Hq > kGateMaxHeads) return 0;
  return (size_t)gate_blocks(T_tot) * (size_t)Hq * sizeof(double);
}

extern "C" int sinkattn_gate_importance(int T_tot, int Hq, const float* sink_s, float* imp,
                                        void* workspace, size_t workspace_bytes,
                                        sinkattn_stream_t stream) {
  if (T_tot < 1 || Hq < 1) return SINKATTN_ERR_INVALID_ARG;
  if (Hq > kGateMaxHeads) return SINKATTN_ERR_UNSUPPORTED;
  if (!sink_s || !imp || !workspace) return SINKATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(sink_s) | reinterpret_cast<uintptr_t>(imp) |
       reinterpret_cast<uintptr_t>(workspace)) & 15)
    return SINKATTN_ERR_INVALID_ARG;
  if (workspace_bytes < sinkattn_gate_importance_workspace_bytes(T_tot, Hq))
    return SINKATTN_ERR_WORKSPACE;
  const int nb = gate_blocks(T_tot);
  const int rows_per_blk = (T_tot + nb - 1) / nb;
  const int threads = (kGateThreads / Hq) * Hq;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(workspace);
  gate_partial_kernel<<<nb, threads, 0, s>>>(sink_s, T_tot, Hq, rows_per_blk, part);
  gate_reduce_kernel<<<(Hq + 3) / 4, 128, 0, s>>>(part, nb, Hq, T_tot, imp);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}
