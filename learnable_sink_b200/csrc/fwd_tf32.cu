// Forward pass for fp32 inputs on the tensor cores, with the 3xTF32 split.
//
// Same computation as the bf16 forward (page "Attention Sink, Learnable Sink
// and dsink": scores and GQA map, section 1; the sink logit in the softmax
// denominator with a zero value, section 4; LSE_new and sink_s, sections 4
// and 9).  Each fp32 operand x is written as hi + lo, hi = x with its low 13
// mantissa bits cleared (a TF32 value, exact on the tensor cores) and
// lo = x - hi (exact in fp32), and each product as lo*hi + hi*lo + hi*hi on
// kind::tf32 MMAs accumulating in fp32 (the lo*lo term lies below fp32
// rounding), so the result carries about 21 significant bits per product.
//
// V is transposed by the splitter into K-major tiles (keys contiguous per
// column of D): kind::tf32 reads its B operand K-major.
//
// One CTA = one query tile of 128 rows (128 tokens x 1 head, or 64 tokens x
// 2 heads for 64-key block tiles) and its list of key tiles, streamed in
// sub-tiles of KT = 32 keys.  Warps:
//   0-3  softmax, one thread per row (TMEM lane = row): splits its Q row
//        into tensor memory once, then per sub-tile the online softmax, P
//        split into hi / lo in tensor memory, lazy O rescale; the epilogue.
//   4-7  splitter: for each landed K/V stage writes K's hi in place and its
//        lo beside it (element by element on the swizzled bytes: both share
//        one layout), and V transposed into K-major hi / lo tiles.
//   8    TMA producer;  9  MMA issuer (one thread).
// The sub-tiles run one after another (S, softmax, P V): this path is for
// fp32 accuracy, not for throughput.
// Tensor memory: S, then P_hi over it [0, 32) | P_lo [32, 64) | O [64, 64 + D)
// | Q_hi | Q_lo (D columns each).
#include <cudaTypedefs.h>

#include "internal.h"

namespace sk {

namespace {

constexpr int kT32Keys = 32;  // keys per sub-tile
constexpr float kT32Rescale = 8.0f;

template <int D_>
struct T32Cfg {
  static constexpr int D = D_, KT = kT32Keys;
  static constexpr int ATOMS = D / 32;                 // 128-byte (32-float) column blocks
  static constexpr int TILE_BYTES = KT * D * 4;        // one K or V sub-tile
  // K (hi in place), K_lo, V as loaded, V^T hi, V^T lo
  static constexpr int STAGE_BYTES = 5 * TILE_BYTES;
  static constexpr int NS = D == 64 ? 4 : 2;
  static constexpr int THREADS = 10 * 32;
  static constexpr int SPLIT_WARP0 = 4, PRODUCER_WARP = 8, MMA_WARP = 9;
  static constexpr int S_COL = 0, PL_COL = KT, O_COL = 2 * KT, QH_COL = 2 * KT + D,
                       QL_COL = 2 * KT + 2 * D;
  static constexpr int TMEM_NEED = 2 * KT + 3 * D;
  static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int OFF_BAR = NS * STAGE_BYTES;
  // full, split, empty per stage; q, s, p, o, fin
  static constexpr int N_BARS = 3 * NS + 5;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(TMEM_NEED <= 512, "tensor memory");
};

// kind::tf32 instruction descriptor: TF32 x TF32 -> FP32 (format code 2 for
// A and B), dense; same field layout as the f16 kind.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N, int a_mn_major,
                                                      int b_mn_major) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(a_mn_major) << 15) |
         (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
// D[tmem] (+)= A[tmem] * B[smem] (kind::tf32)
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t tf32_hi_bits(uint32_t x) { return x & 0xFFFFE000u; }

struct T32Params {
  const int* plan;
  const float* q;
  const float* sink;
  float* out;
  float* lse;
  float* sink_s;
  float* lse_orig;
  int* status;
  int Hq, Hkv, G, causal, n_sink, window, per_item, chunks, hpt, ptile;
  float scale_log2;
};

__device__ __forceinline__ bool t32_wait_noabort(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudgetCycles) return false;
  return true;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fwd_tf32_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const T32Params p) {
  constexpr int D = C::D, KT = C::KT, NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_full = bars;            // TMA of stage s landed
  uint64_t* bar_split = bars + NS;      // hi / lo of stage s written
  uint64_t* bar_empty = bars + 2 * NS;  // stage s read by its last MMA
  uint64_t* bar_q = bars + 3 * NS;      // Q hi / lo in tensor memory
  uint64_t* bar_s = bar_q + 1;
  uint64_t* bar_p = bar_q + 2;
  uint64_t* bar_o = bar_q + 3;
  uint64_t* bar_fin = bar_q + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const PlanHdr* hdr = reinterpret_cast<const PlanHdr*>(p.plan);
  const int rank = blockIdx.x / p.per_item;
  if (rank >= hdr->n_fwd_items) return;
  const int rem = blockIdx.x % p.per_item;
  const int idx = p.plan[hdr->off_fwd_order + rank];
  const TileItem it = reinterpret_cast<const TileItem*>(p.plan + hdr->off_fwd_items)[idx];
  const int kvh = it.kvh >= 0 ? it.kvh : rem / p.chunks;
  const int head0 = kvh * p.G + (rem % p.chunks) * p.hpt;
  const int* ent = p.plan + hdr->off_fwd_entries + it.entry_off;
  const int sub = p.ptile / KT;           // sub-tiles per plan tile
  const int n = it.entry_len * sub;       // sub-tiles of this CTA

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full + s, 1);
      mbar_init(bar_split + s, 128);
      mbar_init(bar_empty + s, 1);
    }
    mbar_init(bar_q, 128);
    mbar_init(bar_s, 1);
    mbar_init(bar_p, 128);
    mbar_init(bar_o, 1);
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      bool ok = true;
      int last[NS];
      for (int s = 0; s < NS; ++s) last[s] = -1;
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % NS;
        ok = mbar_wait(bar_empty + s, ((j / NS) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        const int krow = it.seq_start + (__ldg(ent + j / sub) >> 1) * p.ptile + (j % sub) * KT;
        uint8_t* st = smem + s * C::STAGE_BYTES;
        mbar_expect_tx(bar_full + s, 2 * C::TILE_BYTES);
        for (int a = 0; a < C::ATOMS; ++a) {
          tma_load_3d(st + a * (KT * 128), &tmap_k, bar_full + s, a * 32, kvh, krow);
          tma_load_3d(st + 2 * C::TILE_BYTES + a * (KT * 128), &tmap_v, bar_full + s, a * 32,
                      kvh, krow);
        }
        last[s] = j;
      }
      if (!ok)
        for (int s = 0; s < NS; ++s)
          if (last[s] >= 0) t32_wait_noabort(bar_full + s, (last[s] / NS) & 1);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_s = idesc_tf32_f32(128, KT, 0, 0);
      constexpr uint32_t id_pv = idesc_tf32_f32(128, D, 0, 0);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status);
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % NS;
        ok = mbar_wait(bar_split + s, (j / NS) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t kl = kb + C::TILE_BYTES, vb = kb + 3 * C::TILE_BYTES,
                       vl = kb + 4 * C::TILE_BYTES;
        // S = Q_lo K_hi + Q_hi K_lo + Q_hi K_hi, 8 columns of D per step
#pragma unroll
        for (int kk = 0; kk < D / 8; ++kk) {
          const uint32_t off = (kk / 4) * (KT * 128) + (kk % 4) * 32;
          const uint64_t dkh = sdesc_sw128(kb + off, 16, 1024), dkl = sdesc_sw128(kl + off, 16, 1024);
          mma_tf32_ts(tmem + C::S_COL, tmem + C::QL_COL + kk * 8, dkh, id_s, kk > 0 ? 1u : 0u);
          mma_tf32_ts(tmem + C::S_COL, tmem + C::QH_COL + kk * 8, dkl, id_s, 1u);
          mma_tf32_ts(tmem + C::S_COL, tmem + C::QH_COL + kk * 8, dkh, id_s, 1u);
        }
        mma_commit(bar_s);
        ok = mbar_wait(bar_p, j & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        // O += P_lo V_hi + P_hi V_lo + P_hi V_hi, 8 keys per step; V^T is
        // K-major: D rows of the KT = 32 keys' 128 bytes
#pragma unroll
        for (int kk = 0; kk < KT / 8; ++kk) {
          const uint64_t dvh = sdesc_sw128(vb + kk * 32, 16, 1024);
          const uint64_t dvl = sdesc_sw128(vl + kk * 32, 16, 1024);
          mma_tf32_ts(tmem + C::O_COL, tmem + C::PL_COL + kk * 8, dvh, id_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
          mma_tf32_ts(tmem + C::O_COL, tmem + C::S_COL + kk * 8, dvl, id_pv, 1u);
          mma_tf32_ts(tmem + C::O_COL, tmem + C::S_COL + kk * 8, dvh, id_pv, 1u);
        }
        mma_commit(bar_empty + s);
      }
      if (ok) mma_commit(bar_o);
      mma_commit(bar_fin);
      t32_wait_noabort(bar_fin, 0);
    }
  } else if (warp >= C::SPLIT_WARP0) {
    // ------------------------------------------------------------ splitter
    const int tid = threadIdx.x - C::SPLIT_WARP0 * 32;  // 0..127
    for (int j = 0; j < n; ++j) {
      const int s = j % NS;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_full + s, (j / NS) & 1, abort_flag,
                                                        p.status));
      if (!ok) break;
      uint8_t* st = smem + s * C::STAGE_BYTES;
      {  // K: hi in place, lo beside it (same swizzled layout)
        uint4* hi = reinterpret_cast<uint4*>(st);
        uint4* lo = reinterpret_cast<uint4*>(st + C::TILE_BYTES);
        for (int i = tid; i < C::TILE_BYTES / 16; i += 128) {
          const uint4 x = hi[i];
          const uint4 h = make_uint4(tf32_hi_bits(x.x), tf32_hi_bits(x.y), tf32_hi_bits(x.z),
                                     tf32_hi_bits(x.w));
          lo[i] = make_uint4(__float_as_uint(__uint_as_float(x.x) - __uint_as_float(h.x)),
                             __float_as_uint(__uint_as_float(x.y) - __uint_as_float(h.y)),
                             __float_as_uint(__uint_as_float(x.z) - __uint_as_float(h.z)),
                             __float_as_uint(__uint_as_float(x.w) - __uint_as_float(h.w)));
          hi[i] = h;
        }
      }
      {  // V [keys][D] (32-column boxes, 128-byte swizzle) -> V^T hi / lo
         // [D][32 keys], 128-byte rows with the same swizzle (K-major B)
        const uint8_t* src = st + 2 * C::TILE_BYTES;
        uint8_t* th = st + 3 * C::TILE_BYTES;
        uint8_t* tl = st + 4 * C::TILE_BYTES;
        for (int e = tid; e < KT * D; e += 128) {
          const int key = e / D, d = e % D;
          const int a = d >> 5, cc = d & 31;
          const float x = *reinterpret_cast<const float*>(
              src + a * (KT * 128) + key * 128 + ((((cc >> 2) ^ (key & 7))) << 4) + (cc & 3) * 4);
          const uint32_t hb = tf32_hi_bits(__float_as_uint(x));
          const int off = d * 128 + (((key >> 2) ^ (d & 7)) << 4) + (key & 3) * 4;
          *reinterpret_cast<uint32_t*>(th + off) = hb;
          *reinterpret_cast<float*>(tl + off) = x - __uint_as_float(hb);
        }
      }
      // the MMAs read these through the async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar_split + s);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp;                       // TMEM lane quadrant
    const int r = wq * 32 + lane;              // row of the tile
    const int tok = r / p.hpt, hh = r % p.hpt;
    const int head = head0 + hh;
    const int qi = it.tile_start + tok;
    const bool row_valid = tok < it.tile_len;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const long long row = (long long)(it.seq_start + (row_valid ? qi : it.tile_start)) * p.Hq + head;
    // Q row -> hi / lo columns of tensor memory (rows past the sequence: 0)
    {
      const float4* src = reinterpret_cast<const float4*>(p.q + row * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t h[32], l[32];
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4) {
          float4 x = row_valid ? __ldg(src + c * 8 + v4) : make_float4(0.f, 0.f, 0.f, 0.f);
          const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t hb = tf32_hi_bits(__float_as_uint(xs[e]));
            h[4 * v4 + e] = hb;
            l[4 * v4 + e] = __float_as_uint(xs[e] - __uint_as_float(hb));
          }
        }
        tmem_st32(tmem + lane_off + C::QH_COL + 32 * c, h);
        tmem_st32(tmem + lane_off + C::QL_COL + 32 * c, l);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_q);
    }
    const uint32_t s_addr = tmem + lane_off + C::S_COL;
    const uint32_t pl_addr = tmem + lane_off + C::PL_COL;
    const uint32_t o_addr = tmem + lane_off + C::O_COL;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int e = __ldg(ent + j / sub);
      const int k0 = (e >> 1) * p.ptile + (j % sub) * KT;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s, j & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      float x[KT];
      {
        uint32_t rr[32];
        tmem_ld32(s_addr, rr);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < KT; ++c) {
          asm volatile("" : "+r"(rr[c]));
          x[c] = __uint_as_float(rr[c]);
        }
      }
      if (e & 1) {
        const RowSpan sp = row_span(qi, k0, it.seq_len, p.causal, p.n_sink, p.window);
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (!span_visible(sp, c)) x[c] = -INFINITY;
      }
      if (!row_valid) {
#pragma unroll
        for (int c = 0; c < KT; ++c) x[c] = -INFINITY;
      }
      float mraw = x[0];
#pragma unroll
      for (int c = 1; c < KT; ++c) mraw = fmaxf(mraw, x[c]);
      const float mx = mraw * p.scale_log2;
      const bool need = mx > m + kT32Rescale;
      float corr = 1.f;
      if (need) {
        corr = exp2f(m - mx);
        l *= corr;
      }
      const bool touch_o = need && j > 0 && m != -INFINITY;
      if (__any_sync(0xffffffffu, touch_o)) {
        // P V of the previous sub-tile completed before this S was signalled
        const float f = touch_o ? corr : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(o_addr + c * 32, rr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
          tmem_st32(o_addr + c * 32, rr);
        }
      }
      if (need) m = mx;
      const float mu = (m == -INFINITY) ? 0.f : m;
      uint32_t ph[32], pl[32];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < KT; ++c) {
        const float pv = x[c] == -INFINITY ? 0.f : exp2f(fmaf(x[c], p.scale_log2, -mu));
        rs += pv;
        const uint32_t hb = tf32_hi_bits(__float_as_uint(pv));
        ph[c] = hb;
        pl[c] = __float_as_uint(pv - __uint_as_float(hb));
      }
      l += rs;
      tmem_st32(s_addr, ph);
      tmem_st32(pl_addr, pl);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    const bool have_o =
        __all_sync(0xffffffffu, n > 0 && ok && mbar_wait(bar_o, 0, abort_flag, p.status));
    if (n > 0 && !have_o) ok = false;
    float o_scale = 0.f;
    if (ok && row_valid) {
      const float a2 = p.sink ? __ldg(p.sink + head) * kLog2e : -INFINITY;
      const float mt = fmaxf(m, a2);
      float lse_v = -INFINITY, ss = 0.f;
      if (mt != -INFINITY) {
        const float fr = (m == -INFINITY) ? 0.f : exp2f(m - mt);
        const float lr = l * fr;
        const float den = lr + (p.sink ? exp2f(a2 - mt) : 0.f);
        o_scale = fr / den;
        lse_v = (mt + log2f(den)) * kLn2;
        ss = lr / den;
      }
      p.lse[row] = lse_v;
      if (p.sink_s) p.sink_s[row] = ss;
      if (p.lse_orig) p.lse_orig[row] = (m != -INFINITY && l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
    float4* dst = reinterpret_cast<float4*>(p.out + row * D);
    if (have_o) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(o_addr + c * 32, rr);
        tmem_ld_wait();
        if (ok && row_valid) {
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[c * 8 + v4] = make_float4(__uint_as_float(rr[4 * v4]) * o_scale,
                                          __uint_as_float(rr[4 * v4 + 1]) * o_scale,
                                          __uint_as_float(rr[4 * v4 + 2]) * o_scale,
                                          __uint_as_float(rr[4 * v4 + 3]) * o_scale);
        }
      }
    } else if (ok && row_valid) {
#pragma unroll
      for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
int launch_t32(const AttnProblem& p, void* out, float* lse, float* sink_s, cudaStream_t stream) {
  using C = T32Cfg<D>;
  CUtensorMap mk, mv;
  if (!make_tmap_3d_f32(&mk, p.k, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d_f32(&mv, p.v, p.T_tot, p.Hkv, D, 1, C::KT))
    return SINKATTN_ERR_CUDA;
  T32Params tp{};
  tp.plan = p.plan;
  tp.q = static_cast<const float*>(p.q);
  tp.sink = p.sink;
  tp.out = static_cast<float*>(out);
  tp.lse = lse;
  tp.sink_s = sink_s;
  tp.lse_orig = p.lse_orig;
  tp.status = p.status;
  tp.Hq = p.Hq;
  tp.Hkv = p.Hkv;
  tp.G = p.Hq / p.Hkv;
  tp.causal = p.causal;
  tp.n_sink = p.n_sink;
  tp.window = p.window;
  tp.ptile = p.ps.tile;
  tp.hpt = 128 / (p.ps.tile == 128 ? 128 : 64);  // heads per 128-row query tile
  if (tp.G % tp.hpt != 0) return SINKATTN_ERR_UNSUPPORTED;
  tp.chunks = tp.G / tp.hpt;
  tp.per_item = (p.ps.kh_slots == 1 ? p.Hkv : 1) * tp.chunks;
  tp.scale_log2 = p.scale * kLog2e;
  const long long grid = (long long)p.ps.cap_items * tp.per_item;
  if (grid < 1 || grid > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  auto kern = fwd_tf32_kernel<C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  record_start(SINKATTN_KERNEL_FWD, stream);
  kern<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, stream>>>(mk, mv, tp);
  record_stop(SINKATTN_KERNEL_FWD, stream);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace

int launch_fwd_tf32(const AttnProblem& p, void* out, float* lse, float* sink_s,
                    cudaStream_t stream) {
  return p.D == 64 ? launch_t32<64>(p, out, lse, sink_s, stream)
                   : launch_t32<128>(p, out, lse, sink_s, stream);
}

}  // namespace sk
