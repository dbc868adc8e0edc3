// fp32 backward on the CUDA cores (the fp32 forward runs on the tensor cores
// with the 3xTF32 split, fwd_tf32.cu).  One warp owns one (row, head) for dQ
// and one (key, KV head) for dK/dV; lanes split the head dimension.  dQ per
// row and dK/dV per key from P = exp(x - L_new) and Delta (page "Attention
// Sink, Learnable Sink and dsink", sections 7-8), visiting only the tiles the
// plan lists.
#include "internal.h"

namespace sk {

namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

struct SimtArgs {
  const float* q;
  const float* k;
  const float* v;
  const float* sink;
  const int* plan;
  int Hq, Hkv, causal, n_sink, window, tile, T_tot;
  float scale_log2;  // alpha * log2(e)
  int* status;
  float* lse_orig;   // or nullptr
};

template <int D>
__global__ void __launch_bounds__(kWarps * 32) dq_simt_kernel(SimtArgs a, const float* dout,
                                                              const float* lse,
                                                              const float* delta, float* dq) {
  constexpr int E = D / 32;
  const PlanHdr* h = reinterpret_cast<const PlanHdr*>(a.plan);
  const int G = a.Hq / a.Hkv;
  const int heads_per_item = h->kh_slots == 1 ? a.Hq : G;
  const int rank = blockIdx.x / heads_per_item, hh = blockIdx.x % heads_per_item;
  if (rank >= h->n_fwd_items) return;
  const int idx = a.plan[h->off_fwd_order + rank];
  const TileItem it = reinterpret_cast<const TileItem*>(a.plan + h->off_fwd_items)[idx];
  const int head = it.kvh < 0 ? hh : it.kvh * G + hh;
  const int kvh = head / G;
  const int* ent = a.plan + h->off_fwd_entries + it.entry_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < it.tile_len; r += kWarps) {
    const int qi = it.tile_start + r;
    const long long row = (long long)(it.seq_start + qi) * a.Hq + head;
    const float lse2 = lse[row] * kLog2e;
    const float dl = delta[(long long)head * a.T_tot + it.seq_start + qi];
    float qv[E], dov[E], acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qv[e] = a.q[row * D + lane + 32 * e] * a.scale_log2;
      dov[e] = dout[row * D + lane + 32 * e];
      acc[e] = 0.f;
    }
    for (int t = 0; t < it.entry_len; ++t) {
      const int kt = ent[t] >> 1, partial = ent[t] & 1;
      const int k0 = kt * a.tile;
      const int kend = min(k0 + a.tile, it.seq_len);
      for (int kj = k0; kj < kend; ++kj) {
        if (partial && !visible_elem(qi, kj, it.seq_len, a.causal, a.n_sink, a.window)) continue;
        const long long krow = (long long)(it.seq_start + kj) * a.Hkv + kvh;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s += qv[e] * a.k[krow * D + lane + 32 * e];
          dp += dov[e] * a.v[krow * D + lane + 32 * e];
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const float p = exp2f(s - lse2);
        const float ds = p * (dp - dl);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += ds * a.k[krow * D + lane + 32 * e];
      }
    }
    const float alpha = a.scale_log2 / kLog2e;
#pragma unroll
    for (int e = 0; e < E; ++e) dq[row * D + lane + 32 * e] = acc[e] * alpha;
  }
}

// dK/dV: one warp per key row of a key tile (reverse lists), summing over
// every visible query row of the listed query tiles and the G heads.
template <int D>
__global__ void __launch_bounds__(kWarps * 32) dkdv_simt_kernel(SimtArgs a, const float* dout,
                                                                const float* lse,
                                                                const float* delta, float* dk,
                                                                float* dv) {
  constexpr int E = D / 32;
  const PlanHdr* h = reinterpret_cast<const PlanHdr*>(a.plan);
  const int G = a.Hq / a.Hkv;
  const int kv_per_item = h->kh_slots == 1 ? a.Hkv : 1;
  const int rank = blockIdx.x / kv_per_item, kk = blockIdx.x % kv_per_item;
  if (rank >= h->n_bwd_items) return;
  const int idx = a.plan[h->off_bwd_order + rank];
  const TileItem it = reinterpret_cast<const TileItem*>(a.plan + h->off_bwd_items)[idx];
  const int kvh = it.kvh < 0 ? kk : it.kvh;
  const int* ent = a.plan + h->off_bwd_entries + it.entry_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float alpha = a.scale_log2 / kLog2e;
  for (int r = warp; r < it.tile_len; r += kWarps) {
    const int kj = it.tile_start + r;
    const long long krow = (long long)(it.seq_start + kj) * a.Hkv + kvh;
    float kv[E], vv[E], dka[E], dva[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kv[e] = a.k[krow * D + lane + 32 * e];
      vv[e] = a.v[krow * D + lane + 32 * e];
      dka[e] = 0.f;
      dva[e] = 0.f;
    }
    for (int t = 0; t < it.entry_len; ++t) {
      const int qt = ent[t] >> 1, partial = ent[t] & 1;
      const int q0 = qt * a.tile;
      const int qend = min(q0 + a.tile, it.seq_len);
      for (int qi = q0; qi < qend; ++qi) {
        if (partial && !visible_elem(qi, kj, it.seq_len, a.causal, a.n_sink, a.window)) continue;
        for (int head = kvh * G; head < (kvh + 1) * G; ++head) {
          const long long row = (long long)(it.seq_start + qi) * a.Hq + head;
          float s = 0.f, dp = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            s += a.q[row * D + lane + 32 * e] * kv[e];
            dp += dout[row * D + lane + 32 * e] * vv[e];
          }
          s = warp_sum(s) * a.scale_log2;
          dp = warp_sum(dp);
          const float p = exp2f(s - lse[row] * kLog2e);
          const float ds = p * (dp - delta[(long long)head * a.T_tot + it.seq_start + qi]);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            dka[e] += ds * a.q[row * D + lane + 32 * e];
            dva[e] += p * dout[row * D + lane + 32 * e];
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dk[krow * D + lane + 32 * e] = dka[e] * alpha;
      dv[krow * D + lane + 32 * e] = dva[e];
    }
  }
}

SimtArgs make_args(const AttnProblem& p) {
  SimtArgs a{};
  a.q = static_cast<const float*>(p.q);
  a.k = static_cast<const float*>(p.k);
  a.v = static_cast<const float*>(p.v);
  a.sink = p.sink;
  a.plan = p.plan;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.causal = p.causal;
  a.n_sink = p.n_sink;
  a.window = p.window;
  a.tile = p.ps.tile;
  a.T_tot = p.T_tot;
  a.scale_log2 = p.scale * kLog2e;
  a.status = p.status;
  a.lse_orig = p.lse_orig;
  return a;
}

}  // namespace

int launch_bwd_simt(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  const SimtArgs a = make_args(p);
  const int G = p.Hq / p.Hkv;
  const long long grid_q = (long long)p.ps.cap_items * (p.ps.kh_slots == 1 ? p.Hq : G);
  const long long grid_k = (long long)p.ps.cap_items * (p.ps.kh_slots == 1 ? p.Hkv : 1);
  if (grid_q > 0x7fffffffLL || grid_k > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  const float* dout = static_cast<const float*>(b.dout);
  if (p.D == 64) {
    dq_simt_kernel<64><<<(unsigned)grid_q, kWarps * 32, 0, stream>>>(a, dout, b.lse, b.delta, static_cast<float*>(b.dq));
    dkdv_simt_kernel<64><<<(unsigned)grid_k, kWarps * 32, 0, stream>>>(a, dout, b.lse, b.delta, static_cast<float*>(b.dk), static_cast<float*>(b.dv));
  } else {
    dq_simt_kernel<128><<<(unsigned)grid_q, kWarps * 32, 0, stream>>>(a, dout, b.lse, b.delta, static_cast<float*>(b.dq));
    dkdv_simt_kernel<128><<<(unsigned)grid_k, kWarps * 32, 0, stream>>>(a, dout, b.lse, b.delta, static_cast<float*>(b.dk), static_cast<float*>(b.dv));
  }
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk
