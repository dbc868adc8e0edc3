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

// bf16 -> fp32 is exact and needs only the 16 bits moved up: integer ops,
// no conversion unit.  Pair i holds elements 2i (low half) and 2i + 1.
__device__ __forceinline__ void bf16x8_to_f32x2(const uint4& u, float2 (&f)[4]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}

// The streaming decode moves its running maximum only past this margin
// (log2 units): probabilities stay below 2^8, far from fp32 overflow.
constexpr float kLazyLog2 = 8.f;

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

// Persistent streaming variant (bf16): one CTA per SM loops over work items
// (sequence, KV head, split).  The last warp streams 64-row pieces of K and V
// with TMA through a kStreamStages-deep ring that runs ahead across item
// boundaries, so HBM stays busy while the consumer warps compute.  A group of D/8
// lanes holds one row's 8-element slices; each group takes PR rows of every
// piece and keeps its own online-softmax state per head (running max, sum and
// output slice), so groups never wait for each other inside an item; they
// merge, max-rescaled, once per item.  Dot products of a group's PR x G
// (row, head) pairs are reduced by a butterfly that splits the values across
// the group's lanes.  The loop is kept short because the consumers, not HBM,
// set the pace: bf16 is widened with integer ops, products use the packed
// fp32x2 FMA, and the running maximum moves only when a score exceeds it by
// more than 2^8 (so the output rescale is rare; the final O = acc / l does not
// depend on which reference maximum was used).
constexpr int kPieceRows = 64;
constexpr int kStreamStages = 4;
// consumer threads: 8 warps; with the producer warp the CTA has 9 warps, and
// registers are handed out per group of four warps, so a thread may use
// 65536 / (12 x 32) = 170 -> 168 registers (17 warps would leave 96)
template <int G>
constexpr int consumer_threads() { return 256; }
template <int G>
constexpr int stream_regs() { return 65536 / ((consumer_threads<G>() + 32 + 127) / 128 * 128) / 8 * 8; }

template <int D, int G>
struct StreamGeom {
  static constexpr int kConsumerThreads = consumer_threads<G>();
  static constexpr int kConsumerWarps = kConsumerThreads / 32;
  static constexpr int DH = D / 64;
  static constexpr int LPR = D / 8;                          // lanes per row
  static constexpr int NGRP = kConsumerThreads / LPR;        // row groups
  static constexpr int PR = kPieceRows / NGRP;               // rows per group per piece
  static constexpr int V = PR * G;                           // values per lane before reduce
  static constexpr int HALF_BYTES = kPieceRows * 128;        // one 64-column half of a piece
  static constexpr int PIECE_BYTES = DH * HALF_BYTES;        // K or V piece
  static constexpr int STAGE_BYTES = 2 * PIECE_BYTES;
  static constexpr int OFF_SC = kStreamStages * STAGE_BYTES; // float [2][NGRP][V] scores, probabilities
  static constexpr int OFF_RED = OFF_SC + 2 * NGRP * V * 4;  // float [warps][G][D]
  static constexpr int OFF_ML = OFF_RED + kConsumerWarps * G * D * 4;  // float [warps][G][2]
  static constexpr int OFF_BAR = OFF_ML + kConsumerWarps * G * 2 * 4;
  // + 1024: the kernel rounds the dynamic shared-memory base up to 1024 bytes
  static constexpr int SMEM = OFF_BAR + 2 * kStreamStages * 8 + 1024;
  static constexpr int LOG_LPR = LPR == 16 ? 4 : 3;
  static constexpr int LOG_V = V >= 32 ? 5 : V >= 16 ? 4 : V >= 8 ? 3 : V >= 4 ? 2 : V >= 2 ? 1 : 0;
  static constexpr int KS = LOG_V < LOG_LPR ? LOG_V : LOG_LPR;  // splitting steps
  static constexpr int KEEP = V >> KS;                        // values a lane ends with
  static_assert(PR >= 1 && (1 << LOG_V) == V, "power-of-two rows x heads");
};

// Sum each of the V values over the LPR lanes of a group; afterwards lane gl
// holds KEEP totals, value index decode_value_index(gl, j).
template <int V, int LPR>
__device__ __forceinline__ void butterfly_reduce(float (&v)[V], int gl) {
  int c = V;
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) {
    if (c > 1) {
      const int half = c / 2;
      const bool upper = (gl & o) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      c = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

template <int LOG_V, int LOG_LPR, int KS>
__device__ __forceinline__ int decode_value_index(int gl, int j) {
  int idx = 0;
#pragma unroll
  for (int k = 0; k < KS; ++k)
    idx |= ((gl >> (LOG_LPR - 1 - k)) & 1) << (LOG_V - 1 - k);
  return idx | j;
}

template <int D, int G>
__global__ void __maxnreg__(stream_regs<G>()) decode_stream_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    DecodeProblem p, int chunk, int n_items) {
  using Geo = StreamGeom<D, G>;
  constexpr int LPR = Geo::LPR, PR = Geo::PR, V = Geo::V, DH = Geo::DH;
  constexpr int kConsumerThreads = Geo::kConsumerThreads, kConsumerWarps = Geo::kConsumerWarps;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(sm + Geo::OFF_RED);
  float* ml = reinterpret_cast<float*>(sm + Geo::OFF_ML);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Geo::OFF_BAR);
  uint64_t* empty = full + kStreamStages;
  __shared__ int abort_s;
  const int S = p.n_sink + p.window;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kStreamStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kConsumerWarps);  // one arrival per consumer warp
    }
    abort_s = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto item_rows = [&](int item, int& b, int& kvh, int& split, int& n) {
    split = item % p.num_splits;
    kvh = (item / p.num_splits) % p.Hkv;
    b = item / (p.num_splits * p.Hkv);
    const int n_valid = min(max(p.cache_seqlens[b], 0), S);
    n = max(min(split * chunk + chunk, n_valid) - split * chunk, 0);
  };

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int pc = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        int b, kvh, split, n;
        item_rows(item, b, kvh, split, n);
        for (int r0 = 0; r0 < n; r0 += kPieceRows, ++pc) {
          const int st = pc % kStreamStages;
          if (!mbar_wait(empty + st, ((pc / kStreamStages) & 1) ^ 1, &abort_s, p.status)) return;
          mbar_expect_tx(full + st, Geo::STAGE_BYTES);
          const int row0 = b * S + split * chunk + r0;  // rows past the split are unused
          uint8_t* base = sm + st * Geo::STAGE_BYTES;
          for (int h = 0; h < DH; ++h) {
            tma_load_3d(base + h * Geo::HALF_BYTES, &tmap_k, full + st, h * 64, kvh, row0);
            tma_load_3d(base + Geo::PIECE_BYTES + h * Geo::HALF_BYTES, &tmap_v, full + st, h * 64,
                        kvh, row0);
          }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int grp = tid / LPR, gl = tid % LPR;
  const int c0 = gl * 8, hf = c0 / 64, cin = c0 % 64;
  float* sc_s = reinterpret_cast<float*>(sm + Geo::OFF_SC) + grp * V;               // scores
  float* sc_p = reinterpret_cast<float*>(sm + Geo::OFF_SC) + (Geo::NGRP + grp) * V;  // probabilities
  const float scale_log2 = p.scale * kLog2e;
  int pc = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int b, kvh, split, n;
    item_rows(item, b, kvh, split, n);
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) + ((long long)b * p.Hq + kvh * G) * D;
    float2 qv[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float2 t[4];
      bf16x8_to_f32x2(__ldg(reinterpret_cast<const uint4*>(qb + h * D + c0)), t);
#pragma unroll
      for (int i = 0; i < 4; ++i) qv[h][i] = make_float2(t[i].x * scale_log2, t[i].y * scale_log2);
    }
    float2 acc[G][4];
    float m_run[G], l_run[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_run[h] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][i] = make_float2(0.f, 0.f);
    }
    for (int r0 = 0; r0 < n; r0 += kPieceRows, ++pc) {
      const int st = pc % kStreamStages;
      const int rows = min(kPieceRows, n - r0);
      if (!mbar_wait(full + st, (pc / kStreamStages) & 1, &abort_s, p.status)) return;
      const uint8_t* kbuf = sm + st * Geo::STAGE_BYTES;
      const uint8_t* vbuf = kbuf + Geo::PIECE_BYTES;
      // scores of this group's PR rows for all G heads
      float v[V];
#pragma unroll
      for (int rr = 0; rr < PR; ++rr) {
        const int r = grp * PR + rr;
        float2 kf[4];
        bf16x8_to_f32x2(*reinterpret_cast<const uint4*>(kbuf + hf * Geo::HALF_BYTES + r * 128 + cin * 2), kf);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float2 a = __fmul2_rn(qv[h][0], kf[0]);
#pragma unroll
          for (int i = 1; i < 4; ++i) a = __ffma2_rn(qv[h][i], kf[i], a);
          v[rr * G + h] = a.x + a.y;
        }
      }
      butterfly_reduce<V, LPR>(v, gl);
#pragma unroll
      for (int j = 0; j < Geo::KEEP; ++j) {
        const int idx = decode_value_index<Geo::LOG_V, Geo::LOG_LPR, Geo::KS>(gl, j);
        sc_s[idx] = (grp * PR + idx / G < rows) ? v[j] : -INFINITY;
      }
      __syncwarp();
      // Running maximum per head over the group's rows; it moves (and the
      // group's sum and output are rescaled) only when a score exceeds it by
      // more than 2^kLazyLog2.  From -inf any finite score moves it; an
      // all-masked piece leaves it alone.
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float mx = -INFINITY;
#pragma unroll
        for (int rr = 0; rr < PR; ++rr) mx = fmaxf(mx, sc_s[rr * G + h]);
        if (mx > m_run[h] + kLazyLog2) {
          const float corr = fast_exp2(m_run[h] - mx);  // 0 when m_run was -inf
          l_run[h] *= corr;
          const float2 c2 = make_float2(corr, corr);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[h][i] = __fmul2_rn(acc[h][i], c2);
          m_run[h] = mx;
        }
      }
#pragma unroll
      for (int j = 0; j < Geo::KEEP; ++j) {
        const int idx = decode_value_index<Geo::LOG_V, Geo::LOG_LPR, Geo::KS>(gl, j);
        const int hj = idx % G;
        float mh = m_run[0];
#pragma unroll
        for (int h = 1; h < G; ++h) mh = hj == h ? m_run[h] : mh;
        sc_p[idx] = (grp * PR + idx / G < rows) ? fast_exp2(v[j] - mh) : 0.f;
      }
      __syncwarp();
      // P V over the group's rows (rows past the valid range may hold any
      // bits, so they are skipped rather than weighted by zero)
#pragma unroll
      for (int rr = 0; rr < PR; ++rr) {
        const int r = grp * PR + rr;
        if (r < rows) {
          float2 vf[4];
          bf16x8_to_f32x2(*reinterpret_cast<const uint4*>(vbuf + hf * Geo::HALF_BYTES + r * 128 + cin * 2), vf);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pr = sc_p[rr * G + h];
            l_run[h] += pr;
            const float2 p2 = make_float2(pr, pr);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[h][i] = __ffma2_rn(p2, vf[i], acc[h][i]);
          }
        }
      }
      __syncwarp();  // every lane of the warp is done with the stage and the scratch
      if (lane == 0) mbar_arrive(empty + st);
    }
    // merge the groups of a warp (lanes gl and gl + LPR, ...) with max rescaling
#pragma unroll
    for (int o = 16; o >= LPR; o >>= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mo = __shfl_xor_sync(0xffffffffu, m_run[h], o);
        const float lo = __shfl_xor_sync(0xffffffffu, l_run[h], o);
        const float mm = fmaxf(m_run[h], mo);
        const float fa = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - mm);
        const float fb = (mo == -INFINITY) ? 0.f : exp2f(mo - mm);
        l_run[h] = l_run[h] * fa + lo * fb;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float ax = __shfl_xor_sync(0xffffffffu, acc[h][i].x, o);
          const float ay = __shfl_xor_sync(0xffffffffu, acc[h][i].y, o);
          acc[h][i] = make_float2(acc[h][i].x * fa + ax * fb, acc[h][i].y * fa + ay * fb);
        }
        m_run[h] = mm;
      }
    }
    if (lane < LPR) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          red[(warp * G + h) * D + c0 + 2 * i] = acc[h][i].x;
          red[(warp * G + h) * D + c0 + 2 * i + 1] = acc[h][i].y;
        }
        if (gl == 0) {
          ml[(warp * G + h) * 2] = m_run[h];
          ml[(warp * G + h) * 2 + 1] = l_run[h];
        }
      }
    }
    named_bar_sync(1, kConsumerThreads);
    // merge the warps (fixed order) and write the split's partial
    float* part = p.part + (((long long)b * p.Hq + kvh * G) * p.num_splits + split) * (D + 2);
    for (int i = tid; i < G * D; i += kConsumerThreads) {
      const int h = i / D, d = i % D;
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mm = fmaxf(mm, ml[(w * G + h) * 2]);
      float sacc = 0.f, sl = 0.f;
      if (mm != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float mw = ml[(w * G + h) * 2];
          if (mw == -INFINITY) continue;
          const float f = exp2f(mw - mm);
          sacc += red[(w * G + h) * D + d] * f;
          sl += ml[(w * G + h) * 2 + 1] * f;
        }
      }
      part[(long long)h * p.num_splits * (D + 2) + d] = sacc;
      if (d == 0) {
        part[(long long)h * p.num_splits * (D + 2) + D] = n > 0 ? mm : -INFINITY;
        part[(long long)h * p.num_splits * (D + 2) + D + 1] = n > 0 ? sl : 0.f;
      }
    }
    named_bar_sync(1, kConsumerThreads);  // red / ml reused by the next item
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
  using Geo = StreamGeom<D, G>;
  const int S = p.n_sink + p.window;
  CUtensorMap mk, mv;
  if (!make_tmap_3d_plain(&mk, p.k_cache, p.B * S, p.Hkv, D, 1, kPieceRows) ||
      !make_tmap_3d_plain(&mv, p.v_cache, p.B * S, p.Hkv, D, 1, kPieceRows))
    return SINKATTN_ERR_CUDA;
  auto kern = decode_stream_kernel<D, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = p.B * p.Hkv * p.num_splits;
  const int grid = n_items < sms ? n_items : sms;
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, Geo::kConsumerThreads + 32, Geo::SMEM, stream>>>(mk, mv, p, chunk, n_items);
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
