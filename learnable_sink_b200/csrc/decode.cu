// Split-KV decode over a StreamingLLM ring-buffer KV cache (page
// "Attention Sink / StreamingLLM" interview notes: the cache is a fixed
// segment of initial sink tokens plus a sliding window of recent tokens).
// Slot s of sequence b holds a valid token iff s < min(cache_seqlens[b], S):
// the n_sink sink slots fill first, then the window slots, and once the
// window has wrapped every slot is valid.  No positional encoding is applied
// here, so the ring head's position does not matter.
//
// Stage 1 streams each (sequence, KV head, split)'s K and V rows once; the
// G = Hq/Hkv query heads of the KV head share every loaded row, and each split
// writes (m, l, acc[D]) per query head.  bf16 runs the warp-streaming kernel
// below (TMA rings, warp-level MMAs); fp32 runs one CTA per split with 16-byte
// coalesced loads on the CUDA cores.
// Stage 2: merge the splits with the sink column (page "Attention Sink,
// Learnable Sink and dsink", section 4: e^{a_h} joins the denominator, the
// sink value is zero) and write O, LSE_new and sink_s.
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <type_traits>

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

// Warp-streaming variant (bf16).  Static, balanced schedule: every
// (sequence b, KV head) pair owns np_max pieces of R = 16 cache rows (its
// capacity, whether the rows are filled or not); the pairs' pieces are laid
// end to end (pair = b Hkv + kvh) and warp w streams the flattened range
// [w ppw, (w + 1) ppw).  A warp's range is cut at pair boundaries into
// segments; each segment ends with one partial (m, l, acc) per query head,
// stored in the pair's partial slot w - floor(pair np_max / ppw).  With full
// caches every warp moves the same number of bytes (to within one piece), and
// nothing is shared between warps: no work counter, no atomics, no memset.
// Each warp streams K and V rows with TMA through a private ring of RS stages
// (the loads for the next pieces, and for the first pieces of its next
// segment, are in flight while it computes).
//
// The kernel is bound by HBM, so its arithmetic only has to stay off the
// critical path; it runs on the warp-level tensor-core MMA (m16n8k16, bf16
// in, fp32 accumulate), which spends a few instructions where CUDA-core
// dot products spend hundreds.  The G query heads of the KV head are the 16
// M rows (zero-padded; G <= 8, so rows 8-15 are always padding):
//   S^T-free form   S[h][r] = Q[h] . K[r]  : A = Q (registers, once per segment),
//                                            B = K rows via ldmatrix
//                   O[h][:] += P[h][r] V[r] : A = P (the S accumulators,
//                                            rounded to bf16), B = V via
//                                            ldmatrix.trans
// A lane quad (lane / 4 = head) holds four scores of a 16-row piece, so the
// online softmax needs two shuffles per piece.  K and V land in 64-column
// (128-byte) TMA boxes with the 128-byte swizzle, which keeps the ldmatrix
// row reads free of bank conflicts.  The running maximum moves only when a
// score exceeds it by more than 2^8 (the output rescale is rare; O = acc / l
// does not depend on which reference maximum was used); l is summed from the
// fp32 probabilities.
constexpr int kDecWarps = 8;      // warps per CTA (one CTA per SM)
constexpr int kDecStages = 3;     // ring stages per warp
// per-block shared-memory limit, less room for the kernel's static shared memory
constexpr int kDecSmemMax = 232448 - 256;

template <int D, int G>
struct WarpGeom {
  static constexpr int R = kDecodeRows;                      // rows per piece
  static constexpr int HALVES = D / 64;                      // 64-column TMA boxes per row
  static constexpr int HALF_BYTES = R * 128;                 // one box: R rows x 128 bytes
  static constexpr int PIECE_BYTES = HALVES * HALF_BYTES;    // K or V piece [R][D]
  static constexpr int STAGE_BYTES = 2 * PIECE_BYTES;
  static constexpr int KSTEPS = D / 16;                      // MMA k-steps of Q K^T
  static constexpr int NT = D / 8;                           // MMA n-tiles of P V
  static constexpr int Q_BYTES = G * D * 2;                  // a segment's query heads (bf16)
  static constexpr int OFF_Q = kDecStages * STAGE_BYTES;     // 2 q slots (this segment, next)
  // stages start on 1024-byte boundaries (the swizzle pattern's period)
  static constexpr int WARP_BYTES = (OFF_Q + 2 * Q_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = kDecWarps * WARP_BYTES;
  static constexpr int OFF_LEN = OFF_BAR + kDecWarps * kDecStages * 8;
  // cache lengths staged in shared memory (sequences past this read global)
  static constexpr int LEN_FIT = (kDecSmemMax - 1024 - OFF_LEN) / 4;
  static constexpr int LEN_SLOTS = LEN_FIT < 1024 ? LEN_FIT : 1024;
  // + 1024: the kernel rounds the dynamic shared-memory base up to 1024 bytes
  static constexpr int SMEM = OFF_LEN + LEN_SLOTS * 4 + 1024;
  static_assert(G >= 1 && G <= 8, "query heads per KV head");
  static_assert(D % 64 == 0 && HALF_BYTES % 1024 == 0, "swizzled boxes");
  static_assert(LEN_SLOTS >= 64 && SMEM <= kDecSmemMax, "shared memory");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// (c0, c1) += A B for one m16n8k16 tile whose A rows 8-15 are zero: a_lo / a_hi
// hold row lane/4 at k = 2(lane%4) + {0, 1} and + 8; c0, c1 are that row's
// outputs at n = 2(lane%4) + {0, 1}.  The accumulators of rows 8-15 are dropped.
__device__ __forceinline__ void mma_top_rows(float& c0, float& c1, uint32_t a_lo, uint32_t a_hi,
                                             uint32_t b0, uint32_t b1) {
  float x2, x3;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %10, %10};"
      : "+f"(c0), "+f"(c1), "=f"(x2), "=f"(x3)
      : "r"(a_lo), "r"(0u), "r"(a_hi), "r"(0u), "r"(b0), "r"(b1), "f"(0.f));
}

// The same with f16 operands.
__device__ __forceinline__ void mma_top_rows_h(float& c0, float& c1, uint32_t a_lo, uint32_t a_hi,
                                               uint32_t b0, uint32_t b1) {
  float x2, x3;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %10, %10};"
      : "+f"(c0), "+f"(c1), "=f"(x2), "=f"(x3)
      : "r"(a_lo), "r"(0u), "r"(a_hi), "r"(0u), "r"(b0), "r"(b1), "f"(0.f));
}
template <class E>
__device__ __forceinline__ void mma_top_rows_e(float& c0, float& c1, uint32_t a_lo, uint32_t a_hi,
                                               uint32_t b0, uint32_t b1) {
  if constexpr (E::kFmt == 0) mma_top_rows_h(c0, c1, a_lo, a_hi, b0, b1);
  else mma_top_rows(c0, c1, a_lo, a_hi, b0, b1);
}

// Where the partial results of one (sequence, KV head) pair are.  A pair
// owns np_max units of cache rows; its units are numbered from F = pair
// np_max in a space split into runs of ppw units, and the run of global unit
// u writes partial slot u / ppw - F / ppw.  A pair's filled units come first,
// units past its filled rows write nothing, so the valid slots are
// [0, n_slots).  Units: `rows` cache rows each (mixed = 0), or, for the
// mixed-precision cache (mixed = 1), the sink slots in units of 16 rows
// followed by the window slots in units of 32.
struct DecSched {
  int rows;    // cache rows per unit (mixed = 0)
  int np_max;  // units per pair
  int ppw;     // units per run (warp)
  int mixed;
};
constexpr int kFp8SinkRows = 16, kFp8WinRows = 32;
__device__ __forceinline__ int filled_units(const DecSched& s, int n_valid, int n_sink) {
  if (!s.mixed) return (n_valid + s.rows - 1) / s.rows;
  const int vs = min(n_valid, n_sink), vw = max(n_valid - n_sink, 0);
  return (vs + kFp8SinkRows - 1) / kFp8SinkRows + (vw + kFp8WinRows - 1) / kFp8WinRows;
}
__device__ __forceinline__ int pair_slots(const DecSched& s, long long pair, int np) {
  if (np <= 0) return 0;
  const long long F = pair * s.np_max;
  return int((F + np - 1) / s.ppw - F / s.ppw) + 1;
}

// Merge the partial slots of query head h of sequence b with the sink column
// (page "Attention Sink, Learnable Sink and dsink", section 4: e^{a_h} joins
// the denominator, the sink value is zero) and write O, LSE_new and sink_s.
// One warp; lane l owns output columns [l D/32, (l + 1) D/32).  Every slot's
// (m, l) is loaded at once (slot i in lane i % 32), then eight slots' output
// columns per step, so the merge costs a few L2 round trips, not one per slot.
template <typename T, int D>
__device__ __forceinline__ void combine_head(const DecodeProblem& p, const DecSched& sc, int b,
                                             int h, int lane) {
  constexpr int DPL = D / 32;
  const int S = p.n_sink + p.window;
  const int n_valid = min(max(__ldg(p.cache_seqlens + b), 0), S);
  const int G = p.Hq / p.Hkv;
  const int ns = min(pair_slots(sc, (long long)b * p.Hkv + h / G,
                               filled_units(sc, n_valid, p.n_sink)), p.num_splits);
  const float* part = p.part + ((long long)b * p.Hq + h) * p.num_splits * (D + 2);
  const float a2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
  // slot i's (m, l) in lane i % 32 (all loads in flight at once)
  constexpr int MAXR = 4;  // up to 128 slots
  float mi[MAXR], li[MAXR];
  float mt = a2;
#pragma unroll
  for (int r = 0; r < MAXR; ++r) {
    const int i = r * 32 + lane;
    mi[r] = i < ns ? __ldcg(part + i * (D + 2) + D) : -INFINITY;
    li[r] = i < ns ? __ldcg(part + i * (D + 2) + D + 1) : 0.f;
    mt = fmaxf(mt, mi[r]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
  float l = 0.f, o[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) o[k] = 0.f;
  if (mt != -INFINITY) {
    float wi[MAXR];
#pragma unroll
    for (int r = 0; r < MAXR; ++r) {
      wi[r] = mi[r] == -INFINITY ? 0.f : exp2f(mi[r] - mt);
      l += li[r] * wi[r];
    }
#pragma unroll
    for (int o2 = 16; o2 >= 1; o2 >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o2);
    // output columns: eight slots' loads in flight per step
    for (int i0 = 0; i0 < ns; i0 += 8) {
      float2 x[8][DPL / 2];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int k = 0; k < DPL; k += 2)
          x[u][k / 2] = i0 + u < ns
              ? __ldcg(reinterpret_cast<const float2*>(part + (i0 + u) * (D + 2) + lane * DPL + k))
              : make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u;
        float w = 0.f;
#pragma unroll
        for (int r = 0; r < MAXR; ++r) {
          const float wr = __shfl_sync(0xffffffffu, wi[r], i & 31);
          w = (i >> 5) == r ? wr : w;
        }
#pragma unroll
        for (int k = 0; k < DPL; k += 2) {
          o[k] += x[u][k / 2].x * w;
          o[k + 1] += x[u][k / 2].y * w;
        }
      }
    }
  }
  const float den = l + (p.sink && mt != -INFINITY ? exp2f(a2 - mt) : 0.f);
  const long long row = (long long)b * p.Hq + h;
#pragma unroll
  for (int k = 0; k < DPL; k += 2) {
    const float o0 = den > 0.f ? o[k] / den : 0.f, o1 = den > 0.f ? o[k + 1] / den : 0.f;
    if constexpr (std::is_same_v<T, __half>)
      *reinterpret_cast<uint32_t*>(static_cast<__half*>(p.out) + row * D + lane * DPL + k) =
          pack_f16x2(o0, o1);
    else if constexpr (sizeof(T) == 2)
      *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(p.out) + row * D + lane * DPL + k) =
          pack_bf16x2(o0, o1);
    else
      *reinterpret_cast<float2*>(static_cast<float*>(p.out) + row * D + lane * DPL + k) =
          make_float2(o0, o1);
  }
  if (lane == 0) {
    p.lse[row] = den > 0.f ? (mt + log2f(den)) * kLn2 : -INFINITY;
    if (p.sink_s) p.sink_s[row] = den > 0.f ? l / den : 0.f;
  }
}

// Let the grid launched after this one (the split merge, launched as a
// programmatic dependent) be scheduled now; it still waits for this grid to
// finish before it reads anything.
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the grids this one depends on have finished and their writes
// are visible.
__device__ __forceinline__ void wait_prerequisite_grids() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D, int G, class E = ElemBf16>
__global__ void __launch_bounds__(kDecWarps * 32, 1) decode_warp_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    DecodeProblem p, DecSched sc, int n_warps) {
  using Geo = WarpGeom<D, G>;
  constexpr int R = Geo::R, RS = kDecStages;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int abort_s;
  const int S = p.n_sink + p.window;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wsm = sm + warp * Geo::WARP_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Geo::OFF_BAR) + warp * RS;
  // cache_seqlens of every sequence, staged once per CTA when they fit
  int* s_len = reinterpret_cast<int*>(sm + Geo::OFF_LEN);
  const bool len_in_smem = p.B <= Geo::LEN_SLOTS;
  if (len_in_smem)
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) s_len[i] = __ldg(p.cache_seqlens + i);
  if (threadIdx.x == 0) abort_s = 0;
  if (lane == 0) {
    for (int i = 0; i < RS; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
  }
  __syncthreads();
  allow_dependent_launch();

  // This warp's run of pieces, cut into segments at pair boundaries.
  const int gw = blockIdx.x * kDecWarps + warp;
  const long long total = (long long)p.B * p.Hkv * sc.np_max;
  long long f_next = gw < n_warps ? (long long)gw * sc.ppw : total;
  const long long f_end = min(f_next + sc.ppw, total);
  struct Seg {
    bool valid;
    int n, row0, kvh, b, slot;  // n = filled rows, row0 = first cache row
  };
  // next segment with at least one filled row (pieces past a pair's filled
  // rows are skipped without a load)
  auto next_seg = [&]() {
    Seg s{false, 0, 0, 0, 0, 0};
    while (f_next < f_end) {
      const long long pair = f_next / sc.np_max;
      const int piece0 = int(f_next - pair * sc.np_max);
      const long long seg_end = min(f_end, (pair + 1) * sc.np_max);
      const int piece1 = int(seg_end - pair * sc.np_max);
      f_next = seg_end;
      const int b = int(pair / p.Hkv);
      const int cs = len_in_smem ? s_len[b] : __ldg(p.cache_seqlens + b);
      const int n_valid = min(max(cs, 0), S);
      const int r0 = piece0 * R, r1 = min(piece1 * R, n_valid);
      if (r0 >= r1) continue;
      s.valid = true;
      s.n = r1 - r0;
      s.row0 = b * S + r0;
      s.b = b;
      s.kvh = int(pair % p.Hkv);
      s.slot = int(gw - (pair * sc.np_max) / sc.ppw);
      break;
    }
    return s;
  };
  Seg cur = next_seg();
  Seg nxt{false, 0, 0, 0, 0, 0};
  bool nxt_ready = !cur.valid;
  auto ensure_next = [&]() {
    if (!nxt_ready) {
      nxt = next_seg();
      nxt_ready = true;
    }
  };
  int kc = 0;  // segments started by this warp (q slot parity)

  // producer side (lane 0 issues): up to RS pieces ahead, at most one segment ahead
  int p_sel = 0, p_r0 = 0;        // issuing from cur (0) or nxt (1), next row
  int pc_issue = 0, pc_cons = 0;  // pieces issued / consumed
  auto issue = [&]() {
    while (pc_issue - pc_cons < RS) {
      if (p_sel == 1) ensure_next();
      const Seg& I = p_sel == 0 ? cur : nxt;
      if (!I.valid) break;
      if (p_r0 >= I.n) {
        if (p_sel == 0) { p_sel = 1; p_r0 = 0; continue; }
        break;
      }
      if (lane == 0) {
        const int st = pc_issue % RS;
        uint8_t* base = wsm + st * Geo::STAGE_BYTES;
        // The warp's reads of this stage and of the q slot completed before
        // the __syncwarp that preceded this call (their values are in
        // registers), so the asynchronous writes may reuse the space.
        mbar_expect_tx(full + st, Geo::STAGE_BYTES + (p_r0 == 0 ? Geo::Q_BYTES : 0));
        if (p_r0 == 0)  // the segment's G query rows (contiguous) ride with its first piece
          bulk_load(wsm + Geo::OFF_Q + ((kc + p_sel) & 1) * Geo::Q_BYTES,
                    static_cast<const __nv_bfloat16*>(p.q) + ((long long)I.b * p.Hq + I.kvh * G) * D,
                    Geo::Q_BYTES, full + st);
        const int row0 = I.row0 + p_r0;  // rows past the segment are unused
#pragma unroll
        for (int hf = 0; hf < Geo::HALVES; ++hf) {
          tma_load_3d(base + hf * Geo::HALF_BYTES, &tmap_k, full + st, hf * 64, I.kvh, row0);
          tma_load_3d(base + Geo::PIECE_BYTES + hf * Geo::HALF_BYTES, &tmap_v, full + st, hf * 64,
                      I.kvh, row0);
        }
      }
      p_r0 += R;
      ++pc_issue;
    }
  };

  const int g = lane >> 2, t = lane & 3;  // fragment row (query head) and column pair
  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const float scale_log2 = p.scale * kLog2e;
  bool ok = true;
  while (cur.valid && ok) {
    const int kvh = cur.kvh, b = cur.b, n_cur = cur.n;
    uint32_t qa[Geo::KSTEPS][2];  // A fragments of Q (row g; zero for padding heads)
    float oc[Geo::NT][2];         // O[g][8 j + 2 t + {0, 1}]
#pragma unroll
    for (int j = 0; j < Geo::NT; ++j) oc[j][0] = oc[j][1] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // head g; l_run sums this lane's probabilities
    issue();
    for (int r0 = 0; r0 < n_cur; r0 += R) {
      const int st = pc_cons % RS;
      ok = __all_sync(0xffffffffu, mbar_wait(full + st, (pc_cons / RS) & 1, &abort_s, p.status));
      if (!ok) break;
      const int rows = min(R, n_cur - r0);
      if (r0 == 0) {
        // padding heads read head 0's row (inside the slot) and drop it
        const uint8_t* qs =
            wsm + Geo::OFF_Q + (kc & 1) * Geo::Q_BYTES + (g < G ? g : 0) * D * 2 + t * 4;
#pragma unroll
        for (int kk = 0; kk < Geo::KSTEPS; ++kk) {
          const uint32_t lo = *reinterpret_cast<const uint32_t*>(qs + kk * 32);
          const uint32_t hi = *reinterpret_cast<const uint32_t*>(qs + kk * 32 + 16);
          qa[kk][0] = g < G ? lo : 0u;
          qa[kk][1] = g < G ? hi : 0u;
        }
      }
      uint8_t* kbuf = wsm + st * Geo::STAGE_BYTES;
      uint8_t* vbuf = kbuf + Geo::PIECE_BYTES;
      // Rows past the valid range hold whatever the cache holds there; their
      // scores are masked below, and their V rows are zeroed so that a stale
      // NaN cannot reach the P V products (only a segment's last piece).
      if (rows < R) {
        const int nz = Geo::HALVES * (R - rows) * 8;  // 16-byte chunks
        for (int i = lane; i < nz; i += 32) {
          const int hf = i / ((R - rows) * 8), rem = i % ((R - rows) * 8);
          *reinterpret_cast<uint4*>(vbuf + hf * Geo::HALF_BYTES + (rows + rem / 8) * 128 +
                                    (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        // order these generic writes before the stage's next asynchronous refill
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      // S = Q K^T for rows 0-7 (sa) and 8-15 (sb) of the piece
      const uint32_t kb = smem_u32(kbuf), vb = smem_u32(vbuf);
      float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
#pragma unroll
      for (int kk = 0; kk < Geo::KSTEPS; ++kk) {
        // matrices: rows (mi >> 1) * 8 + mr, columns 16 kk + (mi & 1) * 8
        const int row = (mi >> 1) * 8 + mr, chunk = ((2 * kk) & 7) + (mi & 1);
        uint32_t r[4];
        ldsm_x4(kb + (kk >> 2) * Geo::HALF_BYTES + row * 128 + ((chunk ^ mr) << 4), r);
        mma_top_rows_e<E>(sa0, sa1, qa[kk][0], qa[kk][1], r[0], r[1]);
        mma_top_rows_e<E>(sb0, sb1, qa[kk][0], qa[kk][1], r[2], r[3]);
      }
      // scores of head g at rows 2t, 2t + 1, 8 + 2t, 9 + 2t (log2 units)
      const int ra = 2 * t;
      const float x0 = ra < rows ? sa0 * scale_log2 : -INFINITY;
      const float x1 = ra + 1 < rows ? sa1 * scale_log2 : -INFINITY;
      const float x2 = ra + 8 < rows ? sb0 * scale_log2 : -INFINITY;
      const float x3 = ra + 9 < rows ? sb1 * scale_log2 : -INFINITY;
      float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      // From -inf any finite score moves the maximum; an all-masked piece
      // leaves it alone.
      if (mx > m_run + kLazyLog2) {
        const float corr = fast_exp2(m_run - mx);  // 0 when m_run was -inf
        l_run *= corr;
#pragma unroll
        for (int j = 0; j < Geo::NT; ++j) {
          oc[j][0] *= corr;
          oc[j][1] *= corr;
        }
        m_run = mx;
      }
      const float p0 = x0 == -INFINITY ? 0.f : fast_exp2(x0 - m_run);
      const float p1 = x1 == -INFINITY ? 0.f : fast_exp2(x1 - m_run);
      const float p2 = x2 == -INFINITY ? 0.f : fast_exp2(x2 - m_run);
      const float p3 = x3 == -INFINITY ? 0.f : fast_exp2(x3 - m_run);
      l_run += (p0 + p1) + (p2 + p3);
      const uint32_t pa_lo = E::pack(p0, p1), pa_hi = E::pack(p2, p3);
      // O += P V, two n-tiles (16 columns) per ldmatrix
#pragma unroll
      for (int jp = 0; jp < Geo::NT / 2; ++jp) {
        // matrices: rows (mi & 1) * 8 + mr, columns 16 jp + (mi >> 1) * 8
        const int row = (mi & 1) * 8 + mr, chunk = ((2 * jp) & 7) + (mi >> 1);
        uint32_t r[4];
        ldsm_x4_trans(vb + (jp >> 2) * Geo::HALF_BYTES + row * 128 + ((chunk ^ mr) << 4), r);
        mma_top_rows_e<E>(oc[2 * jp][0], oc[2 * jp][1], pa_lo, pa_hi, r[0], r[1]);
        mma_top_rows_e<E>(oc[2 * jp + 1][0], oc[2 * jp + 1][1], pa_lo, pa_hi, r[2], r[3]);
      }
      __syncwarp();  // every lane is done with the stage
      ++pc_cons;
      issue();       // refill the freed stage
    }
    if (!ok) break;
    // l of head g: the quad's lanes hold disjoint rows
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    // the segment's partial of every query head: [b][kvh G + h][slot][D + 2]
    // (the host's schedule keeps slot < num_splits; checked, never written past)
    const bool slot_ok = cur.slot >= 0 && cur.slot < p.num_splits;
    if (!slot_ok && lane == 0) set_status(p.status, SINKATTN_ERR_BOUNDS);
    if (g < G && slot_ok) {
      // rows of D + 2 floats are only 8-byte aligned: float2 stores
      float* part = p.part + (((long long)b * p.Hq + kvh * G + g) * p.num_splits + cur.slot) * (D + 2);
#pragma unroll
      for (int j = 0; j < Geo::NT; ++j)
        *reinterpret_cast<float2*>(part + 8 * j + 2 * t) = make_float2(oc[j][0], oc[j][1]);
      if (t == 0) {
        part[D] = m_run;
        part[D + 1] = l_run;
      }
    }
    // next segment; the producer side may already be streaming it
    ensure_next();
    cur = nxt;
    ++kc;
    if (p_sel == 1) {
      p_sel = 0;
    } else {
      p_sel = 0;
      p_r0 = 0;
    }
    nxt_ready = !cur.valid;
  }
  // leave no copy in flight: wait for every issued piece
  if (!ok) {
    for (; pc_cons < pc_issue; ++pc_cons) {
      const long long t0 = clock64();
      while (!mbar_try_wait(full + pc_cons % RS, (pc_cons / RS) & 1))
        if (clock64() - t0 > kWaitBudgetCycles) break;
    }
  }
}

// Merge slots + sink: one warp per (sequence, query head).  Launched as a
// programmatic dependent of the streaming kernel: its blocks may start while
// the streaming kernel drains and wait here until its partials are visible.
template <typename T, int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeProblem p, DecSched sc) {
  wait_prerequisite_grids();
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= p.B * p.Hq) return;
  combine_head<T, D>(p, sc, w / p.Hq, w % p.Hq, threadIdx.x & 31);
}

template <typename T, int D>
int launch_combine(const DecodeProblem& p, const DecSched& sc, cudaStream_t stream) {
  const int warps = p.B * p.Hq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((warps + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_combine_kernel<T, D>, p, sc) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

template <class T, int D, int G>
int launch_tma(const DecodeProblem& p, cudaStream_t stream) {
  using E = std::conditional_t<std::is_same_v<T, __half>, ElemF16, ElemBf16>;
  using Geo = WarpGeom<D, G>;
  const int S = p.n_sink + p.window;
  CUtensorMap mk, mv;
  if (!make_tmap_3d(&mk, p.k_cache, p.B * S, p.Hkv, D, 1, Geo::R) ||
      !make_tmap_3d(&mv, p.v_cache, p.B * S, p.Hkv, D, 1, Geo::R))
    return SINKATTN_ERR_CUDA;
  auto kern = decode_warp_kernel<D, G, E>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static_assert(Geo::R == kDecodeRows, "piece size of the schedule");
  const DecSchedule ds = decode_schedule(p.B, p.Hkv, S, p.num_splits, (long long)sms * kDecWarps);
  if (ds.ppw > 0x7fffffffLL || ds.np_max > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  const DecSched sc{Geo::R, (int)ds.np_max, (int)ds.ppw, 0};
  const int grid = (ds.n_warps + kDecWarps - 1) / kDecWarps;
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, kDecWarps * 32, Geo::SMEM, stream>>>(mk, mv, p, sc, ds.n_warps);
  record_stop(SINKATTN_KERNEL_DECODE, stream);
  if (cudaGetLastError() != cudaSuccess) return SINKATTN_ERR_CUDA;
  return launch_combine<T, D>(p, sc, stream);
}

template <typename T, int D, int G>
int launch_split(const DecodeProblem& p, cudaStream_t stream) {
  if constexpr (sizeof(T) == 2) {
    return launch_tma<T, D, G>(p, stream);
  } else {
  using Geo = DecGeom<D>;
  const int S = p.n_sink + p.window;
  // fp32: one CTA per (split, KV head, sequence), splits of `chunk` slots
  // rounded up to 16 (trailing splits may then be empty and write m = -inf)
  const int chunk = ((S + p.num_splits - 1) / p.num_splits + 15) / 16 * 16;
  const size_t smem = sizeof(float) * ((size_t)G * chunk + (size_t)Geo::NGRP * G * D);
  auto kern = decode_split_kernel<T, D, G>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  dim3 grid(p.num_splits, p.Hkv, p.B);
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, kDecThreads, smem, stream>>>(p, chunk);
  record_stop(SINKATTN_KERNEL_DECODE, stream);
  if (cudaGetLastError() != cudaSuccess) return SINKATTN_ERR_CUDA;
  // split i of a pair is unit i of a run of one unit
  return launch_combine<T, D>(p, DecSched{chunk, p.num_splits, 1, 0}, stream);
  }
}

// ---------------------------------------------------------------------------
// Mixed-precision ring cache (page "Attention Sink / StreamingLLM", on KV-cache
// quantisation: the first tokens carry much of the attention weight, so they
// stay in high precision while the rest are stored low).  The n_sink sink
// slots are bf16 ([B, n_sink, Hkv, D]); the window slots are FP8 E4M3 codes
// ([B, window, Hkv, D] bytes) whose value is code value x a per-KV-head scale.
//
// Same static schedule and streaming structure as decode_warp_kernel; a pair's
// units are its sink slots in 16-row pieces (bf16, 2D bytes per row) followed
// by its window slots in 32-row pieces (D bytes per row), so every piece fills
// the same ring stage.  A 32-row window piece runs as two 16-row sub-pieces on
// the f16 warp MMA (E4M3 codes convert to f16 exactly):
//   scores  S[h][r] = k_scale (Q[h] . code[r]): Q as f16, and since a dot
//           product does not depend on the order of its terms, each lane takes
//           the four consecutive codes one ldmatrix row read gives it
//           (k = 4t..4t+3 of a 16-code chunk) and Q's A fragment holds the
//           same four Q elements;
//   values  O[h][:] += v_scale (P[h][r] code[r][:]): ldmatrix.trans on the
//           byte rows gives a lane two adjacent columns of rows 2t and 2t+1;
//           a byte permute pairs the rows per column, so MMA n-tile (c, e)
//           holds columns 16 c + 2 n + e (a fixed column permutation, undone
//           when the partial is written).
// Sink pieces run on the bf16 MMA and accumulate into the same permuted
// accumulator (P divided by v_scale, which the partial's write multiplies
// back): the lane reads its two columns of the four rows it needs as 32-bit
// words and pairs the rows per column with byte permutes.
template <int D>
struct Fp8Geom {
  static constexpr int R = kFp8SinkRows;                    // sink rows per piece
  static constexpr int RW = kFp8WinRows;                    // window rows per piece
  static constexpr int HALVES = D / 64;
  static constexpr int HALF_BYTES = R * 128;                // bf16 box: 16 rows x 128 bytes
  static constexpr int PIECE_BYTES = HALVES * HALF_BYTES;   // K or V piece (either kind)
  static_assert(RW * D == PIECE_BYTES, "an FP8 window piece fills a bf16 piece's space");
  static constexpr int STAGE_BYTES = 2 * PIECE_BYTES;
  static constexpr int KSTEPS = D / 16;
  static constexpr int NT = D / 8;
  static constexpr int CHUNKS = D / 16;                     // 16-code chunks of a window row
};

__device__ __forceinline__ void mma_top_rows_f16(float& c0, float& c1, uint32_t a_lo, uint32_t a_hi,
                                                 uint32_t b0, uint32_t b1) {
  float x2, x3;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %10, %10};"
      : "+f"(c0), "+f"(c1), "=f"(x2), "=f"(x3)
      : "r"(a_lo), "r"(0u), "r"(a_hi), "r"(0u), "r"(b0), "r"(b1), "f"(0.f));
}
// two E4M3 codes (low byte first) -> f16x2 (exact)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
      static_cast<__nv_fp8x2_storage_t>(two_codes & 0xffffu), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.y) << 16);
}
// 16-byte chunk of a swizzled window row: 128-byte rows (D = 128) use the
// 128-byte swizzle (chunk ^ row % 8), 64-byte rows the 64-byte swizzle
// (chunk ^ (row / 2) % 4).
template <int D>
__device__ __forceinline__ uint32_t win_chunk_addr(uint32_t base, int row, int chunk) {
  if constexpr (D == 128) return base + row * 128 + ((chunk ^ (row & 7)) << 4);
  else return base + row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4);
}

struct Fp8Extra {
  const float* k_scale;  // [Hkv]
  const float* v_scale;  // [Hkv]
};

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32, 1) decode_fp8_kernel(
    const __grid_constant__ CUtensorMap tmap_ks, const __grid_constant__ CUtensorMap tmap_vs,
    const __grid_constant__ CUtensorMap tmap_kw, const __grid_constant__ CUtensorMap tmap_vw,
    DecodeProblem p, Fp8Extra x8, DecSched sc, int n_warps) {
  using Geo = WarpGeom<D, G>;  // shared-memory layout (stages, q slots, barriers)
  using F8 = Fp8Geom<D>;
  static_assert(Geo::STAGE_BYTES == F8::STAGE_BYTES, "stage size");
  constexpr int RS = kDecStages;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int abort_s;
  const int n_sink = p.n_sink, window = p.window;
  const int n_sp = (n_sink + F8::R - 1) / F8::R;  // sink pieces per pair
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wsm = sm + warp * Geo::WARP_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Geo::OFF_BAR) + warp * RS;
  int* s_len = reinterpret_cast<int*>(sm + Geo::OFF_LEN);
  const bool len_in_smem = p.B <= Geo::LEN_SLOTS;
  if (len_in_smem)
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) s_len[i] = __ldg(p.cache_seqlens + i);
  if (threadIdx.x == 0) abort_s = 0;
  if (lane == 0) {
    for (int i = 0; i < RS; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
  }
  __syncthreads();
  allow_dependent_launch();

  const int gw = blockIdx.x * kDecWarps + warp;
  const long long total = (long long)p.B * p.Hkv * sc.np_max;
  long long f_next = gw < n_warps ? (long long)gw * sc.ppw : total;
  const long long f_end = min(f_next + sc.ppw, total);
  struct Seg {
    bool valid;
    int p0, p1;   // filled pieces [p0, p1) of the pair
    int vs, vw;   // filled sink / window rows of the sequence
    int kvh, b, slot;
  };
  auto next_seg = [&]() {
    Seg s{false, 0, 0, 0, 0, 0, 0, 0};
    while (f_next < f_end) {
      const long long pair = f_next / sc.np_max;
      const int piece0 = int(f_next - pair * sc.np_max);
      const long long seg_end = min(f_end, (pair + 1) * sc.np_max);
      f_next = seg_end;
      const int b = int(pair / p.Hkv);
      const int cs = len_in_smem ? s_len[b] : __ldg(p.cache_seqlens + b);
      const int n_valid = min(max(cs, 0), n_sink + window);
      const int np = filled_units(sc, n_valid, n_sink);
      const int piece1 = min(int(seg_end - pair * sc.np_max), np);
      if (piece0 >= piece1) continue;
      s.valid = true;
      s.p0 = piece0;
      s.p1 = piece1;
      s.vs = min(n_valid, n_sink);
      s.vw = max(n_valid - n_sink, 0);
      s.b = b;
      s.kvh = int(pair % p.Hkv);
      s.slot = int(gw - (pair * sc.np_max) / sc.ppw);
      break;
    }
    return s;
  };
  Seg cur = next_seg();
  Seg nxt{false, 0, 0, 0, 0, 0, 0, 0};
  bool nxt_ready = !cur.valid;
  auto ensure_next = [&]() {
    if (!nxt_ready) {
      nxt = next_seg();
      nxt_ready = true;
    }
  };
  int kc = 0;
  int p_sel = 0, p_pc = -1;       // issuing from cur (0) or nxt (1); next piece (-1: start)
  int pc_issue = 0, pc_cons = 0;
  auto issue = [&]() {
    while (pc_issue - pc_cons < RS) {
      if (p_sel == 1) ensure_next();
      const Seg& I = p_sel == 0 ? cur : nxt;
      if (!I.valid) break;
      const int pc = p_pc < 0 ? I.p0 : p_pc;
      if (pc >= I.p1) {
        if (p_sel == 0) { p_sel = 1; p_pc = -1; continue; }
        break;
      }
      if (lane == 0) {
        const int st = pc_issue % RS;
        uint8_t* base = wsm + st * Geo::STAGE_BYTES;
        const bool first = (pc == I.p0);
        mbar_expect_tx(full + st, Geo::STAGE_BYTES + (first ? Geo::Q_BYTES : 0));
        if (first)
          bulk_load(wsm + Geo::OFF_Q + ((kc + p_sel) & 1) * Geo::Q_BYTES,
                    static_cast<const __nv_bfloat16*>(p.q) + ((long long)I.b * p.Hq + I.kvh * G) * D,
                    Geo::Q_BYTES, full + st);
        if (pc < n_sp) {  // bf16 sink piece: 16 rows as 64-column boxes
          const int row0 = I.b * n_sink + pc * F8::R;
#pragma unroll
          for (int hf = 0; hf < F8::HALVES; ++hf) {
            tma_load_3d(base + hf * F8::HALF_BYTES, &tmap_ks, full + st, hf * 64, I.kvh, row0);
            tma_load_3d(base + F8::PIECE_BYTES + hf * F8::HALF_BYTES, &tmap_vs, full + st,
                        hf * 64, I.kvh, row0);
          }
        } else {          // FP8 window piece: 32 rows of D bytes, one box each
          const int row0 = I.b * window + (pc - n_sp) * F8::RW;
          tma_load_3d(base, &tmap_kw, full + st, 0, I.kvh, row0);
          tma_load_3d(base + F8::PIECE_BYTES, &tmap_vw, full + st, 0, I.kvh, row0);
        }
      }
      p_pc = pc + 1;
      ++pc_issue;
    }
  };

  const int g = lane >> 2, t = lane & 3;
  const int mi = lane >> 3, mr = lane & 7;
  const float scale_log2 = p.scale * kLog2e;
  bool ok = true;
  while (cur.valid && ok) {
    const int kvh = cur.kvh, b = cur.b;
    const float ks_log2 = scale_log2 * __ldg(x8.k_scale + kvh);
    const float vsc = __ldg(x8.v_scale + kvh);
    const float inv_vsc = 1.f / vsc;
    // this segment's query rows (bf16, in shared memory for the whole segment)
    const uint8_t* qs = wsm + Geo::OFF_Q + (kc & 1) * Geo::Q_BYTES + (g < G ? g : 0) * D * 2;
    uint32_t qh[F8::CHUNKS][2];   // f16 Q fragments (window pieces), k = 4t..4t+3 per chunk
    // O / v_scale in the permuted column order: n-tile 2 c + e, lane (g, t)
    // holds columns 16 c + 4 t + e and 16 c + 4 t + 2 + e
    float ow[F8::NT][2];
#pragma unroll
    for (int j = 0; j < F8::NT; ++j) ow[j][0] = ow[j][1] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    issue();
    for (int pc = cur.p0; pc < cur.p1; ++pc) {
      const int st = pc_cons % RS;
      ok = __all_sync(0xffffffffu, mbar_wait(full + st, (pc_cons / RS) & 1, &abort_s, p.status));
      if (!ok) break;
      if (pc == cur.p0) {
#pragma unroll
        for (int c = 0; c < F8::CHUNKS; ++c) {
          const uint2 u = *reinterpret_cast<const uint2*>(qs + c * 32 + t * 8);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
          qh[c][0] = g < G ? pack_f16x2(f0.x, f0.y) : 0u;
          qh[c][1] = g < G ? pack_f16x2(f1.x, f1.y) : 0u;
        }
      }
      uint8_t* kbuf = wsm + st * Geo::STAGE_BYTES;
      uint8_t* vbuf = kbuf + F8::PIECE_BYTES;
      const uint32_t kb = smem_u32(kbuf), vb = smem_u32(vbuf);
      const bool sink_piece = pc < n_sp;
      const int rows_all = sink_piece ? min(F8::R, cur.vs - pc * F8::R)
                                      : min(F8::RW, cur.vw - (pc - n_sp) * F8::RW);
      const int cap = sink_piece ? F8::R : F8::RW;
      if (rows_all < cap) {  // zero the V rows past the filled ones (stale NaN guard)
        const int row_bytes = sink_piece ? 128 : D;           // bytes per row per box
        const int boxes = sink_piece ? F8::HALVES : 1;
        const int box_bytes = sink_piece ? F8::HALF_BYTES : F8::PIECE_BYTES;
        const int per_box = (cap - rows_all) * row_bytes / 16;  // 16-byte chunks
        for (int i = lane; i < boxes * per_box; i += 32) {
          const int bx = i / per_box, rem = i % per_box;
          *reinterpret_cast<uint4*>(vbuf + bx * box_bytes + rows_all * row_bytes + rem * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      const int n_sub = sink_piece ? 1 : 2;
      for (int sp = 0; sp < n_sub; ++sp) {
        const int rows = min(F8::R, rows_all - sp * F8::R);
        if (rows <= 0) break;
        float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
        if (sink_piece) {
          // bf16 scores, natural k order; the Q fragments come from shared
          // memory (sink pieces are a pair's first piece only)
#pragma unroll
          for (int kk = 0; kk < F8::KSTEPS; ++kk) {
            const uint32_t qlo = g < G ? *reinterpret_cast<const uint32_t*>(qs + t * 4 + kk * 32) : 0u;
            const uint32_t qhi = g < G ? *reinterpret_cast<const uint32_t*>(qs + t * 4 + kk * 32 + 16) : 0u;
            const int row = (mi >> 1) * 8 + mr, chunk = ((2 * kk) & 7) + (mi & 1);
            uint32_t r[4];
            ldsm_x4(kb + (kk >> 2) * F8::HALF_BYTES + row * 128 + ((chunk ^ mr) << 4), r);
            mma_top_rows(sa0, sa1, qlo, qhi, r[0], r[1]);
            mma_top_rows(sb0, sb1, qlo, qhi, r[2], r[3]);
          }
        } else {
#pragma unroll
          for (int c0 = 0; c0 < F8::CHUNKS; c0 += 2) {
            // matrices: rows 16 sp + (mi >> 1) * 8 + mr, 16-code chunk c0 + (mi & 1)
            const int row = sp * 16 + (mi >> 1) * 8 + mr;
            uint32_t r[4];
            ldsm_x4(win_chunk_addr<D>(kb, row, c0 + (mi & 1)), r);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const uint32_t a0 = e4m3x2_to_f16x2(r[u]), a1 = e4m3x2_to_f16x2(r[u] >> 16);
              const uint32_t b0 = e4m3x2_to_f16x2(r[2 + u]), b1 = e4m3x2_to_f16x2(r[2 + u] >> 16);
              mma_top_rows_f16(sa0, sa1, qh[c0 + u][0], qh[c0 + u][1], a0, a1);
              mma_top_rows_f16(sb0, sb1, qh[c0 + u][0], qh[c0 + u][1], b0, b1);
            }
          }
        }
        const float xs = sink_piece ? scale_log2 : ks_log2;
        const int ra = 2 * t;
        const float x0 = ra < rows ? sa0 * xs : -INFINITY;
        const float x1 = ra + 1 < rows ? sa1 * xs : -INFINITY;
        const float x2 = ra + 8 < rows ? sb0 * xs : -INFINITY;
        const float x3 = ra + 9 < rows ? sb1 * xs : -INFINITY;
        float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (mx > m_run + kLazyLog2) {
          const float corr = fast_exp2(m_run - mx);
          l_run *= corr;
#pragma unroll
          for (int j = 0; j < F8::NT; ++j) {
            ow[j][0] *= corr;
            ow[j][1] *= corr;
          }
          m_run = mx;
        }
        const float p0 = x0 == -INFINITY ? 0.f : fast_exp2(x0 - m_run);
        const float p1 = x1 == -INFINITY ? 0.f : fast_exp2(x1 - m_run);
        const float p2 = x2 == -INFINITY ? 0.f : fast_exp2(x2 - m_run);
        const float p3 = x3 == -INFINITY ? 0.f : fast_exp2(x3 - m_run);
        l_run += (p0 + p1) + (p2 + p3);
        if (sink_piece) {
          // bf16 values into the same permuted accumulator: the lane reads
          // columns 16 c + 2 g and + 1 of rows 2t, 2t + 1, 2t + 8, 2t + 9
          // (one 32-bit word per row) and pairs the rows per column; P is
          // divided by v_scale, which the partial's write multiplies back
          const uint32_t pa_lo = pack_bf16x2(p0 * inv_vsc, p1 * inv_vsc);
          const uint32_t pa_hi = pack_bf16x2(p2 * inv_vsc, p3 * inv_vsc);
#pragma unroll
          for (int cb = 0; cb < F8::CHUNKS; ++cb) {
            const int chunk = 2 * (cb & 3) + (g >> 2);  // 16-byte chunk of the 64-column half
            const uint32_t base = vb + (cb >> 2) * F8::HALF_BYTES + 4 * (g & 3);
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int row = 2 * t + (k & 1) + 8 * (k >> 1);
              asm volatile("ld.shared.b32 %0, [%1];"
                           : "=r"(w[k])
                           : "r"(base + row * 128 + ((chunk ^ (row & 7)) << 4)));
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint32_t sel = e ? 0x7632u : 0x5410u;
              mma_top_rows(ow[2 * cb + e][0], ow[2 * cb + e][1], pa_lo, pa_hi,
                           __byte_perm(w[0], w[1], sel), __byte_perm(w[2], w[3], sel));
            }
          }
        } else {
          const uint32_t pa_lo = pack_f16x2(p0, p1), pa_hi = pack_f16x2(p2, p3);
#pragma unroll
          for (int cb = 0; cb < F8::CHUNKS; cb += 2) {
            // matrices: rows 16 sp + (mi & 1) * 8 + mr, 16-column block cb + (mi >> 1)
            const int row = sp * 16 + (mi & 1) * 8 + mr;
            uint32_t r[4];
            ldsm_x4_trans(win_chunk_addr<D>(vb, row, cb + (mi >> 1)), r);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              // rows 2t / 2t + 1 (r[2u]) and 2t + 8 / 2t + 9 (r[2u + 1]) of
              // columns 2g, 2g + 1 of block cb + u, paired per column
              const uint32_t lo = __byte_perm(r[2 * u], 0u, 0x3120);
              const uint32_t hi = __byte_perm(r[2 * u + 1], 0u, 0x3120);
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int jj = 2 * (cb + u) + e;
                mma_top_rows_f16(ow[jj][0], ow[jj][1], pa_lo, pa_hi,
                                 e4m3x2_to_f16x2(lo >> (16 * e)), e4m3x2_to_f16x2(hi >> (16 * e)));
              }
            }
          }
        }
      }
      __syncwarp();
      ++pc_cons;
      issue();
    }
    if (!ok) break;
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    const bool slot_ok = cur.slot >= 0 && cur.slot < p.num_splits;
    if (!slot_ok && lane == 0) set_status(p.status, SINKATTN_ERR_BOUNDS);
    if (g < G && slot_ok) {
      float* part = p.part + (((long long)b * p.Hq + kvh * G + g) * p.num_splits + cur.slot) * (D + 2);
      // n-tile (c, e) holds columns 16 c + 4 t + e and + 2
#pragma unroll
      for (int jj = 0; jj < F8::NT; ++jj) {
        const int col = 16 * (jj >> 1) + 4 * t + (jj & 1);
        part[col] = ow[jj][0] * vsc;
        part[col + 2] = ow[jj][1] * vsc;
      }
      if (t == 0) {
        part[D] = m_run;
        part[D + 1] = l_run;
      }
    }
    ensure_next();
    cur = nxt;
    ++kc;
    if (p_sel == 1) {
      p_sel = 0;
    } else {
      p_sel = 0;
      p_pc = -1;
    }
    nxt_ready = !cur.valid;
  }
  if (!ok) {
    for (; pc_cons < pc_issue; ++pc_cons) {
      const long long t0 = clock64();
      while (!mbar_try_wait(full + pc_cons % RS, (pc_cons / RS) & 1))
        if (clock64() - t0 > kWaitBudgetCycles) break;
    }
  }
}

// uint8 [T, H, D] map of E4M3 codes, one box of box_t rows x D bytes; the
// 128-byte swizzle for 128-byte rows, the 64-byte swizzle for 64-byte rows.
bool make_tmap_codes(CUtensorMap* map, const void* base, int T, int H, int D, int box_t) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess || q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)H * D};
  cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)box_t};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G>
int launch_fp8_cfg(const DecodeFp8Problem& q, cudaStream_t stream) {
  using Geo = WarpGeom<D, G>;
  const DecodeProblem& p = q.base;
  CUtensorMap mks, mvs, mkw, mvw;
  // a problem without sink slots (or without window slots) never reads that
  // map; it is then built over the other kind's array, which is valid memory
  const void* ks = p.n_sink > 0 ? q.k_sink : q.k_win;
  const void* vs = p.n_sink > 0 ? q.v_sink : q.v_win;
  const void* kw = p.window > 0 ? q.k_win : q.k_sink;
  const void* vw = p.window > 0 ? q.v_win : q.v_sink;
  const int rows_s = p.B * (p.n_sink > 0 ? p.n_sink : 1);
  const int rows_w = p.B * (p.window > 0 ? p.window : 1);
  if (!make_tmap_3d(&mks, ks, rows_s, p.Hkv, D, 1, kFp8SinkRows) ||
      !make_tmap_3d(&mvs, vs, rows_s, p.Hkv, D, 1, kFp8SinkRows) ||
      !make_tmap_codes(&mkw, kw, rows_w, p.Hkv, D, kFp8WinRows) ||
      !make_tmap_codes(&mvw, vw, rows_w, p.Hkv, D, kFp8WinRows))
    return SINKATTN_ERR_CUDA;
  auto kern = decode_fp8_kernel<D, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const DecSchedule ds = decode_schedule_units(p.B, p.Hkv, fp8_pieces(p.n_sink, p.window),
                                               p.num_splits, (long long)sms * kDecWarps);
  if (ds.ppw > 0x7fffffffLL || ds.np_max > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  const DecSched sc{0, (int)ds.np_max, (int)ds.ppw, 1};
  const int grid = (int)((ds.n_warps + kDecWarps - 1) / kDecWarps);
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, kDecWarps * 32, Geo::SMEM, stream>>>(mks, mvs, mkw, mvw, p,
                                                    Fp8Extra{q.k_scale, q.v_scale}, sc,
                                                    (int)ds.n_warps);
  record_stop(SINKATTN_KERNEL_DECODE, stream);
  if (cudaGetLastError() != cudaSuccess) return SINKATTN_ERR_CUDA;
  return launch_combine<__nv_bfloat16, D>(p, sc, stream);
}

template <int D>
int dispatch_fp8(const DecodeFp8Problem& q, cudaStream_t stream) {
  switch (q.base.Hq / q.base.Hkv) {
    case 1: return launch_fp8_cfg<D, 1>(q, stream);
    case 2: return launch_fp8_cfg<D, 2>(q, stream);
    case 4: return launch_fp8_cfg<D, 4>(q, stream);
    case 8: return launch_fp8_cfg<D, 8>(q, stream);
    default: return SINKATTN_ERR_UNSUPPORTED;
  }
}

template <typename T, int D>
int dispatch_g(const DecodeProblem& p, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return launch_split<T, D, 1>(p, stream);
    case 2: return launch_split<T, D, 2>(p, stream);
    case 4: return launch_split<T, D, 4>(p, stream);
    case 8: return launch_split<T, D, 8>(p, stream);
    default: return SINKATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_decode_fp8(const DecodeFp8Problem& q, cudaStream_t stream) {
  return q.base.D == 64 ? dispatch_fp8<64>(q, stream) : dispatch_fp8<128>(q, stream);
}

int launch_decode(const DecodeProblem& p, cudaStream_t stream) {
  if (p.dt == SINKATTN_BF16)
    return p.D == 64 ? dispatch_g<__nv_bfloat16, 64>(p, stream)
                     : dispatch_g<__nv_bfloat16, 128>(p, stream);
  if (p.dt == SINKATTN_FP16)
    return p.D == 64 ? dispatch_g<__half, 64>(p, stream) : dispatch_g<__half, 128>(p, stream);
  return p.D == 64 ? dispatch_g<float, 64>(p, stream) : dispatch_g<float, 128>(p, stream);
}

}  // namespace sk
