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

}  // namespace

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
