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

// Warp-streaming variant (bf16).  Every warp works alone: it takes work
// items (sequence, KV head, split) from a global counter, streams its items'
// K and V rows with TMA through a private ring of RS stages (the loads for the
// next pieces, and for the first pieces of its next item, are in flight while
// it computes), and writes one partial (m, l, acc) per query head and item.
// No warp ever waits for another, so nothing couples the warps of an SM
// beyond sharing its load bandwidth.
//
// The kernel is bound by HBM, so its arithmetic only has to stay off the
// critical path; it runs on the warp-level tensor-core MMA (m16n8k16, bf16
// in, fp32 accumulate), which spends a few instructions where CUDA-core
// dot products spend hundreds.  The G query heads of the KV head are the 16
// M rows (zero-padded; G <= 8, so rows 8-15 are always padding):
//   S^T-free form   S[h][r] = Q[h] . K[r]  : A = Q (registers, once per item),
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
  static constexpr int R = 16;                               // rows per piece
  static constexpr int HALVES = D / 64;                      // 64-column TMA boxes per row
  static constexpr int HALF_BYTES = R * 128;                 // one box: R rows x 128 bytes
  static constexpr int PIECE_BYTES = HALVES * HALF_BYTES;    // K or V piece [R][D]
  static constexpr int STAGE_BYTES = 2 * PIECE_BYTES;
  static constexpr int KSTEPS = D / 16;                      // MMA k-steps of Q K^T
  static constexpr int NT = D / 8;                           // MMA n-tiles of P V
  static constexpr int Q_BYTES = G * D * 2;                  // an item's query heads (bf16)
  static constexpr int OFF_Q = kDecStages * STAGE_BYTES;     // 2 q slots (this item, next)
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

// Merge the splits of query head h of sequence b with the sink column (page
// "Attention Sink, Learnable Sink and dsink", section 4: e^{a_h} joins the
// denominator, the sink value is zero) and write O, LSE_new and sink_s.  One
// warp; lane l owns output columns [l D/32, (l + 1) D/32).  Every split's
// (m, l) is loaded at once (split i in lane i % 32), then eight splits' output
// columns per step, so the merge costs a few L2 round trips, not one per split.
template <typename T, int D>
__device__ __forceinline__ void combine_head(const DecodeProblem& p, int b, int h, int lane) {
  constexpr int DPL = D / 32;
  const int ns = p.num_splits;
  const float* part = p.part + ((long long)b * p.Hq + h) * ns * (D + 2);
  const float a2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
  // split i's (m, l) in lane i % 32 (all loads in flight at once)
  constexpr int MAXR = 4;  // up to 128 splits
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
    // output columns: eight splits' loads in flight per step
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
    if constexpr (sizeof(T) == 2)
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

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32, 1) decode_warp_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    DecodeProblem p, int chunk, int n_items) {
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

  // A work item, decoded once when the warp takes it.
  struct Item {
    int it, n, row0, kvh, b, split;  // n = valid rows, row0 = first cache row
  };
  auto decode_item = [&](int it) {
    Item I{it, 0, 0, 0, 0, 0};
    if (it < n_items) {
      I.split = it % p.num_splits;
      I.kvh = (it / p.num_splits) % p.Hkv;
      I.b = it / (p.num_splits * p.Hkv);
      const int cs = len_in_smem ? s_len[I.b] : __ldg(p.cache_seqlens + I.b);
      const int n_valid = min(max(cs, 0), S);
      I.n = max(min(I.split * chunk + chunk, n_valid) - I.split * chunk, 0);
      I.row0 = I.b * S + I.split * chunk;
    }
    return I;
  };
  // Items come from a global counter.  The atomic for the next item is issued
  // as soon as the current one starts; its result (held by lane 0) is only
  // read when the producer side or the next item needs it, so its latency
  // hides behind the current item's pieces.
  int raw_next = lane == 0 ? atomicAdd(p.counter, 1) : 0;
  Item cur = decode_item(__shfl_sync(0xffffffffu, raw_next, 0));
  if (lane == 0 && cur.it < n_items) raw_next = atomicAdd(p.counter, 1);
  Item nxt{n_items, 0, 0, 0, 0, 0};
  bool nxt_ready = cur.it >= n_items;
  auto ensure_next = [&]() {
    if (!nxt_ready) {
      nxt = decode_item(__shfl_sync(0xffffffffu, raw_next, 0));
      nxt_ready = true;
    }
  };
  int kc = 0;  // items started by this warp (q slot parity)

  // producer side (lane 0 issues): up to RS pieces ahead, at most one item ahead
  int p_sel = 0, p_r0 = 0;        // issuing from cur (0) or nxt (1), next row
  int pc_issue = 0, pc_cons = 0;  // pieces issued / consumed
  auto issue = [&]() {
    while (pc_issue - pc_cons < RS) {
      if (p_sel == 1) ensure_next();
      const Item& I = p_sel == 0 ? cur : nxt;
      if (I.it >= n_items) break;
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
        if (p_r0 == 0)  // the item's G query rows (contiguous) ride with its first piece
          bulk_load(wsm + Geo::OFF_Q + ((kc + p_sel) & 1) * Geo::Q_BYTES,
                    static_cast<const __nv_bfloat16*>(p.q) + ((long long)I.b * p.Hq + I.kvh * G) * D,
                    Geo::Q_BYTES, full + st);
        const int row0 = I.row0 + p_r0;  // rows past the split are unused
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
  while (cur.it < n_items && ok) {
    const int split = cur.split, kvh = cur.kvh, b = cur.b, n_cur = cur.n;
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
      // NaN cannot reach the P V products (only an item's last piece).
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
        mma_top_rows(sa0, sa1, qa[kk][0], qa[kk][1], r[0], r[1]);
        mma_top_rows(sb0, sb1, qa[kk][0], qa[kk][1], r[2], r[3]);
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
      const uint32_t pa_lo = pack_bf16x2(p0, p1), pa_hi = pack_bf16x2(p2, p3);
      // O += P V, two n-tiles (16 columns) per ldmatrix
#pragma unroll
      for (int jp = 0; jp < Geo::NT / 2; ++jp) {
        // matrices: rows (mi & 1) * 8 + mr, columns 16 jp + (mi >> 1) * 8
        const int row = (mi & 1) * 8 + mr, chunk = ((2 * jp) & 7) + (mi >> 1);
        uint32_t r[4];
        ldsm_x4_trans(vb + (jp >> 2) * Geo::HALF_BYTES + row * 128 + ((chunk ^ mr) << 4), r);
        mma_top_rows(oc[2 * jp][0], oc[2 * jp][1], pa_lo, pa_hi, r[0], r[1]);
        mma_top_rows(oc[2 * jp + 1][0], oc[2 * jp + 1][1], pa_lo, pa_hi, r[2], r[3]);
      }
      __syncwarp();  // every lane is done with the stage
      ++pc_cons;
      issue();       // refill the freed stage
    }
    if (!ok) break;
    // l of head g: the quad's lanes hold disjoint rows
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    // the split's partial of every query head: [b][kvh G + h][split][D + 2]
    if (g < G) {
      // rows of D + 2 floats are only 8-byte aligned: float2 stores
      float* part = p.part + (((long long)b * p.Hq + kvh * G + g) * p.num_splits + split) * (D + 2);
#pragma unroll
      for (int j = 0; j < Geo::NT; ++j)
        *reinterpret_cast<float2*>(part + 8 * j + 2 * t) = make_float2(oc[j][0], oc[j][1]);
      if (t == 0) {
        part[D] = n_cur > 0 ? m_run : -INFINITY;
        part[D + 1] = n_cur > 0 ? l_run : 0.f;
      }
    }
    // next item; the producer side may already be streaming it
    ensure_next();
    cur = nxt;
    ++kc;
    if (p_sel == 1) {
      p_sel = 0;
    } else {
      p_sel = 0;
      p_r0 = 0;
    }
    nxt_ready = cur.it >= n_items;
    if (lane == 0 && !nxt_ready) raw_next = atomicAdd(p.counter, 1);
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

// Merge splits + sink: one warp per (sequence, query head).
template <typename T, int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeProblem p) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= p.B * p.Hq) return;
  combine_head<T, D>(p, w / p.Hq, w % p.Hq, threadIdx.x & 31);
}

template <typename T, int D>
int launch_combine(const DecodeProblem& p, cudaStream_t stream) {
  const int warps = p.B * p.Hq;
  decode_combine_kernel<T, D><<<(warps + 7) / 8, 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

template <int D, int G>
int launch_tma(const DecodeProblem& p, int chunk, cudaStream_t stream) {
  using Geo = WarpGeom<D, G>;
  const int S = p.n_sink + p.window;
  CUtensorMap mk, mv;
  if (!make_tmap_3d(&mk, p.k_cache, p.B * S, p.Hkv, D, 1, Geo::R) ||
      !make_tmap_3d(&mv, p.v_cache, p.B * S, p.Hkv, D, 1, Geo::R))
    return SINKATTN_ERR_CUDA;
  auto kern = decode_warp_kernel<D, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = p.B * p.Hkv * p.num_splits;
  const int want = (n_items + kDecWarps - 1) / kDecWarps;
  const int grid = want < sms ? want : sms;
  if (cudaMemsetAsync(p.counter, 0, sizeof(int), stream) != cudaSuccess) return SINKATTN_ERR_CUDA;
  record_start(SINKATTN_KERNEL_DECODE, stream);
  kern<<<grid, kDecWarps * 32, Geo::SMEM, stream>>>(mk, mv, p, chunk, n_items);
  record_stop(SINKATTN_KERNEL_DECODE, stream);
  return launch_combine<__nv_bfloat16, D>(p, stream);
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
  if (cudaGetLastError() != cudaSuccess) return SINKATTN_ERR_CUDA;
  return launch_combine<T, D>(p, stream);
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
  // slots per split, rounded up to whole 16-row pieces (trailing splits may
  // then be empty; their partials carry m = -inf and drop out of the merge)
  const int chunk = ((S + p.num_splits - 1) / p.num_splits + 15) / 16 * 16;
  if (p.dt == SINKATTN_BF16)
    return p.D == 64 ? dispatch_g<__nv_bfloat16, 64>(p, chunk, stream)
                     : dispatch_g<__nv_bfloat16, 128>(p, chunk, stream);
  return p.D == 64 ? dispatch_g<float, 64>(p, chunk, stream)
                   : dispatch_g<float, 128>(p, chunk, stream);
}

}  // namespace sk
