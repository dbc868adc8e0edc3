// Forward pass on the 5th-generation tensor cores (tcgen05) for bf16 and f16
// inputs (one template over the 16-bit element type).
//
// Page "Attention Sink, Learnable Sink and dsink": scores and GQA map
// (section 1), the sink logit folded into the softmax denominator with a zero
// value (section 4), LSE_new and the gate sink_s (sections 4 and 9); page
// "Attention Sink and the native MoE in attention layers" (section 5) reads the same gate as
// G = sigma(LSE - sink).
//
// One CTA = NQT query tiles of 128 rows that share a token range and a KV
// head (a tile is 128 tokens of one head, or 64 tokens x 2 heads), and one
// list of key tiles from the plan.  Warp roles:
//   warps [0, 4 NQT)  softmax: warpgroup t owns query tile t, one thread per
//                     row (TMEM lane = row); online softmax in registers,
//                     lazy rescaling of the TMEM O accumulator, epilogue.
//   warp 4 NQT        TMA producer: Q once, then K and V tiles through an
//                     NS-stage mbarrier ring.
//   warp 4 NQT + 1    MMA issuer (one thread): S_t = Q_t K^T (SS, smem
//                     operands) and O_t += P_t V (TS, P read from TMEM where
//                     softmax wrote it over S_t).
// Tensor memory: S_t at columns [t TK, (t+1) TK), O_t after all S tiles.
// The two query tiles ping-pong: while warpgroup 0 exponentiates S_0 the
// tensor core runs tile 1's MMAs and vice versa.  With 64-key blocks at
// D = 64 a CTA holds one query tile, two CTAs share an SM, and consecutive
// score tiles sit in two overlapping regions (SDB below), so the next score
// MMA runs while the softmax works on the current one.
#include <cudaTypedefs.h>

#include "internal.h"

namespace sk {

namespace {

constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when max grows > 2^8

// max of three floats in one instruction (sm_100 three-input max.f32)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// PAIR: the plan's key tiles are 64-key blocks and the kernel stages two of
// them (consecutive entries of the list) as one 128-key tile, so the score MMA
// has N = 128 (N = 64 runs at 2/3 of the tensor rate: its shared-memory
// operand reads become the limit) and the softmax covers 128 columns per pass.
template <int D_, int TQ_, int TK_, int NQT_, bool PAIR_ = false, int MB_ = 1, class E_ = ElemBf16>
struct FwdCfg {
  using E = E_;  // 16-bit element type of Q, K, V, O (and of P)
  static constexpr int D = D_, TQ = TQ_, TK = TK_, NQT = NQT_;
  static constexpr bool PAIR = PAIR_;
  static constexpr int PT = PAIR ? TK / 2 : TK;  // the plan's key tile
  static_assert(!PAIR || TK == 128, "pairs of 64-key blocks");
  static constexpr int HPT = 128 / TQ;           // heads per query tile
  static constexpr int DH = D / 64;              // 64-column halves of a row
  static constexpr int Q_BYTES = 128 * D * 2;    // one query tile
  static constexpr int KV_BYTES = TK * D * 2;    // one K (or V) tile
  static constexpr int SMEM_BUDGET = MB_ == 1 ? 200 * 1024 : 108 * 1024;
  static constexpr int NS_RAW = (SMEM_BUDGET - NQT * Q_BYTES) / (2 * KV_BYTES);
  static constexpr int NS = NS_RAW > 4 ? 4 : NS_RAW;
  static_assert(NS >= 2, "not enough shared memory for a two-stage ring");
  static constexpr int MIN_BLOCKS = MB_;
  // Registers move to the softmax warpgroups: the producer and MMA warps share
  // a warpgroup with two idle warps (setmaxnreg works on whole warpgroups).
  //   two softmax warpgroups, one CTA per SM: 12 warps, 168 registers a thread
  //     at launch, 256 x 208 + 128 x 80 = 384 x 168 (with 56 the producer and
  //     MMA warps spill; 208 still holds a softmax row);
  //   one softmax warpgroup, two CTAs per SM (MB_ = 2, which also halves the
  //     shared-memory budget and the tensor memory of a CTA): 8 warps, 128
  //     registers at launch, 128 x 208 + 128 x 48 = 256 x 128.  Each CTA then
  //     hides the other's prologue and epilogue, which short block-sparse
  //     query tiles expose.
  static constexpr bool REBALANCE = (NQT == 2 && MIN_BLOCKS == 1) || (NQT == 1 && MIN_BLOCKS == 2);
  static constexpr int SOFTMAX_REGS = 208;
  static constexpr int AUX_REGS = MIN_BLOCKS == 1 ? 80 : 48;
  static constexpr int THREADS = (4 * NQT + (REBALANCE ? 4 : 2)) * 32;
  static constexpr int PRODUCER_WARP = 4 * NQT;
  static constexpr int MMA_WARP = 4 * NQT + 1;
  // SDB: one query tile, two CTAs per SM, and the score tiles of consecutive
  // key tiles in two overlapping tensor-memory regions, [0, TK) for even j and
  // [TK/2, 3TK/2) for odd j, with P(j) packed into the half the next region
  // leaves free ([0, TK/2) or [TK, 3TK/2)).  S(j+1) is then issued as soon as
  // the softmax has read S(j) into registers, and the softmax never waits for
  // the PV and S MMAs of its own tile between two key tiles.
  static constexpr bool SDB = PAIR_ && MB_ == 2 && NQT_ == 1;
  static constexpr int S_COL = 0;                // S_t at t * TK
  static constexpr int O_COL = SDB ? TK + TK / 2 : NQT * TK;  // O_t at O_COL + t * D
  static constexpr int TMEM_NEED = SDB ? TK + TK / 2 + D : NQT * (TK + D);
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                 : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(TMEM_NEED <= 512, "tensor memory budget");
  // shared memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
  static constexpr int N_BARS = 1 + 4 * NS + 5 * NQT + 1;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
};

struct FwdParams {
  const int* plan;
  const float* sink;
  __nv_bfloat16* out;
  float* lse;
  float* sink_s;
  float* lse_orig;  // or nullptr
  int* status;
  int Hq, Hkv, G, causal, n_sink, window;
  int per_item, chunks;  // CTAs per plan item, head chunks per KV head
  float scale_log2;
};

// Named barrier over `count` threads that also returns the AND of every
// participant's `in` (the same value in all of them).
__device__ __forceinline__ bool bar_red_and(int id, int count, bool in) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(res)
      : "r"(in ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return res != 0;
}

// Bulk tensor store of a shared-memory box (same box and swizzle as the map's
// loads); the group is committed and waited for by the issuing thread.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ bool wait_noabort(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudgetCycles) return false;
  return true;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::MIN_BLOCKS)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                  const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v,
                  const __grid_constant__ CUtensorMap tmap_o, const FwdParams p) {
  constexpr int D = C::D, TK = C::TK, NQT = C::NQT, HPT = C::HPT, NS = C::NS, DH = C::DH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_kf = bars + 1;
  uint64_t* bar_ke = bar_kf + NS;
  uint64_t* bar_vf = bar_ke + NS;
  uint64_t* bar_ve = bar_vf + NS;
  uint64_t* bar_s = bar_ve + NS;
  uint64_t* bar_p = bar_s + NQT;
  uint64_t* bar_o = bar_p + NQT;
  uint64_t* bar_fin = bar_o + NQT;
  uint64_t* bar_sr = bar_fin + 1;  // SDB: the softmax has read S_t(j)
  uint64_t* bar_pv = bar_sr + NQT;  // SDB: PV_t(j) complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const PlanHdr* hdr = reinterpret_cast<const PlanHdr*>(p.plan);
  const int rank = blockIdx.x / p.per_item;
  if (rank >= hdr->n_fwd_items) return;
  const int rem = blockIdx.x % p.per_item;
  const int idx = p.plan[hdr->off_fwd_order + rank];
  const TileItem it = reinterpret_cast<const TileItem*>(p.plan + hdr->off_fwd_items)[idx];
  const int kvh = it.kvh >= 0 ? it.kvh : rem / p.chunks;
  const int chunk = rem % p.chunks;
  const int head0 = kvh * p.G + chunk * NQT * HPT;
  const int* ent = p.plan + hdr->off_fwd_entries + it.entry_off;
  const int n = it.entry_len;                      // plan entries (key tiles)
  const int nt = C::PAIR ? (n + 1) / 2 : n;        // staged key tiles

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_kf + s, 1);
      mbar_init(bar_ke + s, 1);
      mbar_init(bar_vf + s, 1);
      mbar_init(bar_ve + s, 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(bar_s + t, 1);
      mbar_init(bar_p + t, 128);
      mbar_init(bar_o + t, 1);
      mbar_init(bar_sr + t, 128);
      mbar_init(bar_pv + t, 1);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
    prefetch_tensormap(&tmap_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 * NQT) {
    if constexpr (C::REBALANCE) regs_dec<C::AUX_REGS>();
  }
  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      const int tok0 = it.seq_start + it.tile_start;
      mbar_expect_tx(bar_q, NQT * C::Q_BYTES);
      for (int t = 0; t < NQT; ++t)
        for (int h = 0; h < DH; ++h)
          tma_load_3d(smem + C::OFF_Q + t * C::Q_BYTES + h * (C::Q_BYTES / DH), &tmap_q, bar_q,
                      h * 64, head0 + t * HPT, tok0);
      int last_k[NS], last_v[NS];
      for (int s = 0; s < NS; ++s) last_k[s] = last_v[s] = -1;
      bool ok = true;
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % NS;
        const uint32_t par = ((j / NS) & 1) ^ 1;
        // a missing second block of a pair re-reads the first (its scores
        // are masked; the values stay finite)
        int krow[C::PAIR ? 2 : 1];
        krow[0] = it.seq_start + (__ldg(ent + (C::PAIR ? 2 * j : j)) >> 1) * C::PT;
        if constexpr (C::PAIR)
          krow[1] = 2 * j + 1 < n ? it.seq_start + (__ldg(ent + 2 * j + 1) >> 1) * C::PT : krow[0];
        ok = mbar_wait(bar_ke + s, par, abort_flag, p.status);
        if (!ok) break;
        mbar_expect_tx(bar_kf + s, C::KV_BYTES);
        for (int h = 0; h < DH; ++h)
          for (int b2 = 0; b2 < (C::PAIR ? 2 : 1); ++b2)
            tma_load_3d(smem + C::OFF_K + s * C::KV_BYTES + h * (C::KV_BYTES / DH) +
                            b2 * C::PT * 128,
                        &tmap_k, bar_kf + s, h * 64, kvh, krow[b2]);
        last_k[s] = j;
        ok = mbar_wait(bar_ve + s, par, abort_flag, p.status);
        if (!ok) break;
        mbar_expect_tx(bar_vf + s, C::KV_BYTES);
        for (int h = 0; h < DH; ++h)
          for (int b2 = 0; b2 < (C::PAIR ? 2 : 1); ++b2)
            tma_load_3d(smem + C::OFF_V + s * C::KV_BYTES + h * (C::KV_BYTES / DH) +
                            b2 * C::PT * 128,
                        &tmap_v, bar_vf + s, h * 64, kvh, krow[b2]);
        last_v[s] = j;
      }
      if (!ok) {  // let copies already in flight land before the CTA exits
        wait_noabort(bar_q, 0);
        for (int s = 0; s < NS; ++s) {
          if (last_k[s] >= 0) wait_noabort(bar_kf + s, (last_k[s] / NS) & 1);
          if (last_v[s] >= 0) wait_noabort(bar_vf + s, (last_v[s] / NS) & 1);
        }
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_16_f32(C::E::kFmt, 128, TK, 0, 0);
      constexpr uint32_t idesc_qk16 = idesc_16_f32(C::E::kFmt, 128, 16, 0, 0);
      // staged tile j is a band's sink-only first tile: scores on its first
      // 16 keys only, values from those 16 rows only
      auto narrow = [&](int j) {
        return !C::PAIR && sink_only_tile(__ldg(ent + j) >> 1, it.tile_start, TK, p.n_sink,
                                          p.window);
      };
      constexpr uint32_t idesc_pv = idesc_16_f32(C::E::kFmt, 128, D, 0, 1);
      // descriptors of query tile 0, K stage 0 (both K-major) and V stage 0
      // (B of PV, MN-major: 64-column atoms TK*128 B apart, 8-row groups 1 KB
      // apart); every other operand is a fixed byte offset from these
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(smem + C::OFF_V), TK * 128, 1024);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status);
      if constexpr (C::SDB) {
        // S(j+1) into the other region as soon as the softmax has read S(j)
        // (and after PV(j-1), whose P it overwrites: tcgen05 operations run
        // in issue order); PV(j) once P(j) is written.
        auto issue_s = [&](int j) {
          const uint64_t dk = sdesc_add(dk0, (j % NS) * C::KV_BYTES);
          const uint32_t s_col = (j & 1) ? TK / 2 : 0;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + s_col, sdesc_add(dq0, (kk / 4) * (C::Q_BYTES / DH) + (kk & 3) * 32),
                   sdesc_add(dk, (kk / 4) * (C::KV_BYTES / DH) + (kk & 3) * 32), idesc_qk,
                   kk > 0 ? 1u : 0u);
          mma_commit(bar_s);
          mma_commit(bar_ke + j % NS);
        };
        if (ok) ok = mbar_wait(bar_kf, 0, abort_flag, p.status);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
        for (int j = 0; j < nt && ok; ++j) {
          if (j + 1 < nt) {
            ok = mbar_wait(bar_sr, j & 1, abort_flag, p.status) &&
                 mbar_wait(bar_kf + (j + 1) % NS, ((j + 1) / NS) & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            issue_s(j + 1);
          }
          ok = mbar_wait(bar_p, j & 1, abort_flag, p.status) &&
               mbar_wait(bar_vf + j % NS, (j / NS) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dv = sdesc_add(dv0, (j % NS) * C::KV_BYTES);
          const uint32_t p_col = (j & 1) ? TK : 0;
#pragma unroll
          for (int kk = 0; kk < TK / 16; ++kk)
            mma_ts(tmem + C::O_COL, tmem + p_col + kk * 8, sdesc_add(dv, kk * 16 * 128), idesc_pv,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_ve + j % NS);
          mma_commit(bar_pv);
        }
        if (ok) mma_commit(bar_o);
        mma_commit(bar_fin);
        wait_noabort(bar_fin, 0);
      } else {
      bool narrow_prev = false;
      for (int j = 0; j <= nt && ok; ++j) {
        const bool narrow_j = j < nt && narrow(j);
        if (j < nt) ok = mbar_wait(bar_kf + j % NS, (j / NS) & 1, abort_flag, p.status);
        if (ok && j > 0) ok = mbar_wait(bar_vf + (j - 1) % NS, ((j - 1) / NS) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dv = sdesc_add(dv0, ((j + NS - 1) % NS) * C::KV_BYTES);
        const uint64_t dk = sdesc_add(dk0, (j % NS) * C::KV_BYTES);
        const uint32_t idq = narrow_j ? idesc_qk16 : idesc_qk;
        const int kk_end = narrow_prev ? 1 : TK / 16;
        for (int t = 0; t < NQT && ok; ++t) {
          if (j > 0) {
            ok = mbar_wait(bar_p + t, (j - 1) & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < TK / 16; ++kk) {
              if (kk >= kk_end) break;
              mma_ts(tmem + C::O_COL + t * D, tmem + C::S_COL + t * TK + kk * 8,
                     sdesc_add(dv, kk * 16 * 128), idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
            }
          }
          if (j < nt) {
            const uint64_t dq = sdesc_add(dq0, t * C::Q_BYTES);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // 16 bf16 = 32 B inside the 128-B row; 64-column atoms
              mma_ss(tmem + C::S_COL + t * TK,
                     sdesc_add(dq, (kk / 4) * (C::Q_BYTES / DH) + (kk & 3) * 32),
                     sdesc_add(dk, (kk / 4) * (C::KV_BYTES / DH) + (kk & 3) * 32), idq,
                     kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_s + t);
          }
        }
        narrow_prev = narrow_j;
        if (!ok) break;
        if (j > 0) mma_commit(bar_ve + (j - 1) % NS);
        if (j < nt) mma_commit(bar_ke + j % NS);
      }
      if (ok)
        for (int t = 0; t < NQT; ++t) mma_commit(bar_o + t);
      // drain: every MMA issued by this thread has completed once bar_fin fires
      mma_commit(bar_fin);
      wait_noabort(bar_fin, 0);
      }
    }
  } else if (warp < 4 * NQT) {
    // ------------------------------------------------------------ softmax
    if constexpr (C::REBALANCE) regs_inc<C::SOFTMAX_REGS>();
    const int t = warp / 4;                     // query tile of this warpgroup
    const int wq = warp % 4;                    // TMEM lane quadrant
    const int r = wq * 32 + lane;               // row of the tile
    const int tok = r / HPT, hh = r % HPT;
    const int head = head0 + t * HPT + hh;
    const int qi = it.tile_start + tok;         // sequence-local query position
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + C::S_COL + t * TK;
    const uint32_t o_addr = tmem + lane_off + C::O_COL + t * D;
    // the head's sink logit in log2 units, loaded before the key loop
    const float sink_l2 = p.sink ? __ldg(p.sink + head) * kLog2e : -INFINITY;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int e = __ldg(ent + (C::PAIR ? 2 * j : j));
      const int k0 = (e >> 1) * C::PT;
      // second block of a pair: -1 when the list has no entry for it
      const int e1 = C::PAIR ? (2 * j + 1 < n ? __ldg(ent + 2 * j + 1) : -1) : 0;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s + t, j & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      if (!C::PAIR && sink_only_tile(e >> 1, it.tile_start, TK, p.n_sink, p.window)) {
        // a band's sink-only first tile: 16 score columns, keys [0, n_sink)
        // visible (every row here is past them causally)
        float x16[16];
        {
          uint32_t rr[16];
          tmem_ld16(s_addr, rr);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            asm volatile("" : "+r"(rr[c]));
            x16[c] = c < p.n_sink ? __uint_as_float(rr[c]) : -INFINITY;
          }
        }
        float mraw = x16[0];
#pragma unroll
        for (int c = 1; c < 16; c += 2) mraw = c + 1 < 16 ? fmax3(mraw, x16[c], x16[c + 1]) : fmaxf(mraw, x16[c]);
        const float mx = mraw * p.scale_log2;
        const bool need = mx > m + kRescaleThreshold;
        float corr = 1.f;
        if (need) {
          corr = exp2f(m - mx);
          l *= corr;
        }
        const bool touch_o = need && j > 0 && m != -INFINITY;
        if (__any_sync(0xffffffffu, touch_o)) {
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
        uint32_t pk[8];
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float p0 = fast_exp2(fmaf(x16[2 * i], p.scale_log2, -mu));
          const float p1 = fast_exp2(fmaf(x16[2 * i + 1], p.scale_log2, -mu));
          rs += p0 + p1;
          pk[i] = C::E::pack(p0, p1);
        }
        tmem_st8(s_addr, pk);
        l += rs;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p + t);
        continue;
      }
      // raw scores x = Q.K (the scale is folded into the exponent below)
      // all TK / 32 loads in flight, one wait for them together
      const uint32_t s_cur = C::SDB ? tmem + lane_off + ((j & 1) ? TK / 2 : 0) : s_addr;
      float x[TK];
      {
        uint32_t rr[TK / 32][32];
#pragma unroll
        for (int c = 0; c < TK / 32; ++c) tmem_ld32(s_cur + c * 32, rr[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < TK / 32; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            asm volatile("" : "+r"(rr[c][i]));  // the values exist only after the wait
            x[c * 32 + i] = __uint_as_float(rr[c][i]);
          }
      }
      if constexpr (C::SDB) {
        // S(j) is in registers: the next score tile may overwrite its columns
        tc_fence_before();
        mbar_arrive(bar_sr + t);
      }
      // partial tiles: element mask from the row's visible span
      if constexpr (C::PAIR) {
        if (e & 1) {
          const RowSpan sp = row_span(qi, k0, it.seq_len, p.causal, p.n_sink, p.window);
#pragma unroll
          for (int c = 0; c < C::PT; ++c)
            if (!span_visible(sp, c)) x[c] = -INFINITY;
        }
        if (e1 < 0) {  // no second block
#pragma unroll
          for (int c = C::PT; c < TK; ++c) x[c] = -INFINITY;
        } else if (e1 & 1) {
          const RowSpan sp = row_span(qi, (e1 >> 1) * C::PT - C::PT, it.seq_len, p.causal,
                                      p.n_sink, p.window);
#pragma unroll
          for (int c = C::PT; c < TK; ++c)
            if (!span_visible(sp, c)) x[c] = -INFINITY;
        }
      } else if (e & 1) {
        const RowSpan sp = row_span(qi, k0, it.seq_len, p.causal, p.n_sink, p.window);
#pragma unroll
        for (int c = 0; c < TK; ++c)
          if (!span_visible(sp, c)) x[c] = -INFINITY;
      }
      // row max with eight independent accumulators (short dependency chains)
      float m8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) m8[a] = x[a];
#pragma unroll
      for (int k = 1; k < TK / 8; k += 2) {
#pragma unroll
        for (int a = 0; a < 8; ++a)
          m8[a] = k + 1 < TK / 8 ? fmax3(m8[a], x[8 * k + a], x[8 * k + 8 + a])
                                 : fmaxf(m8[a], x[8 * k + a]);
      }
      const float mraw = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7]));
      const float mx = mraw * p.scale_log2;  // scale > 0: max commutes with it
      // Lazy rescale: the running reference max m only moves when the tile
      // max exceeds it by more than 2^8.  Per-row decision, but the TMEM
      // load/store are warp-collective, so the warp rescales together and
      // rows that need nothing multiply by 1.
      const bool need = mx > m + kRescaleThreshold;  // true on the first visible tile
      float corr = 1.f;
      if (need) {
        corr = exp2f(m - mx);  // 0 when m = -inf
        l *= corr;
      }
      const bool touch_o = need && j > 0 && m != -INFINITY;
      if (__any_sync(0xffffffffu, touch_o)) {
        // O_t row *= corr.  Safe: PV_t(j-1) completed before S_t(j) was
        // signalled (tcgen05 operations complete in issue order); with SDB
        // S_t(j) was issued before PV_t(j-1), whose completion is awaited
        // here (PV_t(j) waits for this tile's P, so the phase is unambiguous).
        if constexpr (C::SDB) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar_pv + t, (j - 1) & 1, abort_flag, p.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
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
      // p = 2^(x * alpha * log2(e) - m): the scaling FMA and the row sums run
      // on element pairs (packed fp32x2 instructions), the exponentials one
      // by one
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-mu, -mu);
      float2 rs4[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) rs4[a] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < TK / 64; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 y = __ffma2_rn(make_float2(x[c * 64 + 2 * i], x[c * 64 + 2 * i + 1]), sc2, nm2);
          const float2 pp = make_float2(fast_exp2(y.x), fast_exp2(y.y));
          rs4[i & 3] = __fadd2_rn(rs4[i & 3], pp);
          pk[i] = C::E::pack(pp.x, pp.y);
        }
        // P over the first TK/2 columns of S_t (with SDB, of the half the
        // next score tile leaves free)
        tmem_st32((C::SDB ? tmem + lane_off + ((j & 1) ? TK : 0) : s_addr) + c * 32, pk);
      }
      const float2 r01 = __fadd2_rn(rs4[0], rs4[1]), r23 = __fadd2_rn(rs4[2], rs4[3]);
      const float2 rsum = __fadd2_rn(r01, r23);
      l += rsum.x + rsum.y;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p + t);
    }
    // epilogue: fold the sink into the denominator (log2 domain), write LSE
    // and sink_s while the last PV runs, then stream O out of tensor memory
    // 32 columns at a time
    const long long row = (long long)(it.seq_start + qi) * p.Hq + head;
    float o_scale = 0.f;
    if (ok && tok < it.tile_len) {
      const float mt = fmaxf(m, sink_l2);
      float lse_v = -INFINITY, ss = 0.f;
      if (mt != -INFINITY) {
        const float fr = (m == -INFINITY) ? 0.f : exp2f(m - mt);
        const float lr = l * fr;
        const float den = lr + (p.sink ? exp2f(sink_l2 - mt) : 0.f);
        o_scale = fr / den;
        lse_v = (mt + log2f(den)) * kLn2;
        ss = lr / den;
      }
      p.lse[row] = lse_v;
      if (p.sink_s) p.sink_s[row] = ss;
      // the raw LSE over the visible keys (before the sink joins)
      if (p.lse_orig) p.lse_orig[row] = (m != -INFINITY && l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
    const bool have_o =
        __all_sync(0xffffffffu, n > 0 && ok && mbar_wait(bar_o + t, 0, abort_flag, p.status));
    if (n > 0 && !have_o) ok = false;
    const bool store = ok && tok < it.tile_len;
    if (store && !have_o) {  // no key tile: O is zero
      uint4* dst = reinterpret_cast<uint4*>(p.out + row * D);
      const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) dst[c] = z;
    }
    if (have_o) {
      // all 32 lanes of the warp take part in the tcgen05.ld
      tc_fence_after();
      // A whole tile (every row stores) goes out through shared memory and a
      // bulk tensor store: the warpgroup writes its rows into its Q buffer
      // (every MMA that read Q is complete) in the layout the Q load used,
      // and one thread stores the box.  A tile cut by the sequence end keeps
      // per-row stores (the box would spill into the next sequence's rows).
      const bool whole = ok && it.tile_len == C::TQ;  // uniform over the warp
      uint8_t* qbuf = smem + C::OFF_Q + t * C::Q_BYTES;
      uint4* dst = reinterpret_cast<uint4*>(p.out + row * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(o_addr + c * 32, rr);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 u;
          u.x = C::E::pack(__uint_as_float(rr[8 * v + 0]) * o_scale, __uint_as_float(rr[8 * v + 1]) * o_scale);
          u.y = C::E::pack(__uint_as_float(rr[8 * v + 2]) * o_scale, __uint_as_float(rr[8 * v + 3]) * o_scale);
          u.z = C::E::pack(__uint_as_float(rr[8 * v + 4]) * o_scale, __uint_as_float(rr[8 * v + 5]) * o_scale);
          u.w = C::E::pack(__uint_as_float(rr[8 * v + 6]) * o_scale, __uint_as_float(rr[8 * v + 7]) * o_scale);
          if (whole) {
            // columns 32c + 8v .. + 7: atom (32c) / 64, 16-byte chunk
            // ((32c) % 64) / 8 + v, 128-byte swizzle over the row
            const int col8 = (32 * c) % 64 / 8 + v;
            *reinterpret_cast<uint4*>(qbuf + (32 * c / 64) * (C::Q_BYTES / DH) + r * 128 +
                                      ((col8 ^ (r & 7)) * 16)) = u;
          } else if (store) {
            dst[c * 4 + v] = u;
          }
        }
      }
    }
    // Every warp of the warpgroup passes this barrier exactly once; the box
    // is stored only if all four staged their rows (a warp whose waits timed
    // out did not, and the outputs of that call are undefined anyway).
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic -> async proxy
    const bool staged = bar_red_and(1 + t, 128, have_o && ok && it.tile_len == C::TQ);
    if (staged && wq == 0 && lane == 0) {
      const int tok0 = it.seq_start + it.tile_start;
      uint8_t* qbuf = smem + C::OFF_Q + t * C::Q_BYTES;
#pragma unroll
      for (int h = 0; h < DH; ++h)
        tma_store_3d(&tmap_o, qbuf + h * (C::Q_BYTES / DH), h * 64, head0 + t * HPT, tok0);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

}  // namespace

// 3-D bf16 tensor map over [T, H, D] (D contiguous), box {64, box_h, box_t},
// 128-byte swizzle.  Out-of-range rows read as zero.
bool make_tmap_3d(CUtensorMap* map, const void* base, int T, int H, int D, int box_h, int box_t) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_h, (cuuint32_t)box_t};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Same, without swizzle: the box lands in shared memory as plain rows of 64
// elements (128 bytes).
bool make_tmap_3d_plain(CUtensorMap* map, const void* base, int T, int H, int D, int box_h,
                        int box_t) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_h, (cuuint32_t)box_t};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [T, H, D] map with 32-element (128-byte) boxes {32, box_h, box_t},
// 128-byte swizzle: used to add dQ tiles into the fp32 accumulator.
bool make_tmap_3d_f32(CUtensorMap* map, const void* base, int T, int H, int D, int box_h,
                      int box_t) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)box_h, (cuuint32_t)box_t};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <class E, int D, int TQ, int TK, int NQT, bool PAIR = false, int MB = 1>
int launch_cfg(const AttnProblem& p, void* out, float* lse, float* sink_s, cudaStream_t stream) {
  using C = FwdCfg<D, TQ, TK, NQT, PAIR, MB, E>;
  CUtensorMap mq, mk, mv, mo;
  if (!make_tmap_3d(&mq, p.q, p.T_tot, p.Hq, D, C::HPT, TQ) ||
      !make_tmap_3d(&mo, out, p.T_tot, p.Hq, D, C::HPT, TQ) ||
      !make_tmap_3d(&mk, p.k, p.T_tot, p.Hkv, D, 1, C::PT) ||
      !make_tmap_3d(&mv, p.v, p.T_tot, p.Hkv, D, 1, C::PT))
    return SINKATTN_ERR_CUDA;
  FwdParams fp{};
  fp.plan = p.plan;
  fp.sink = p.sink;
  fp.out = static_cast<__nv_bfloat16*>(out);
  fp.lse = lse;
  fp.sink_s = sink_s;
  fp.lse_orig = p.lse_orig;
  fp.status = p.status;
  fp.Hq = p.Hq;
  fp.Hkv = p.Hkv;
  fp.G = p.Hq / p.Hkv;
  fp.causal = p.causal;
  fp.n_sink = p.n_sink;
  fp.window = p.window;
  fp.chunks = fp.G / (NQT * C::HPT);
  fp.per_item = (p.ps.kh_slots == 1 ? p.Hkv : 1) * fp.chunks;
  fp.scale_log2 = p.scale * kLog2e;
  const long long grid = (long long)p.ps.cap_items * fp.per_item;
  if (grid < 1 || grid > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  auto kern = fwd_tc_kernel<C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  if constexpr (C::REBALANCE) {
    // the register split assumes the launch-bound count per thread; with
    // fewer, a setmaxnreg.inc would wait for registers that never come
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != 65536 / (C::THREADS * C::MIN_BLOCKS) / 8 * 8)
      return SINKATTN_ERR_UNSUPPORTED;
  }
  record_start(SINKATTN_KERNEL_FWD, stream);
  kern<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, fp);
  record_stop(SINKATTN_KERNEL_FWD, stream);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace

template <class E>
int launch_fwd_e(const AttnProblem& p, void* out, float* lse, float* sink_s, cudaStream_t stream) {
  const int G = p.Hq / p.Hkv;
  const int tile = p.ps.tile;  // 128 (dense masks) or the block size (64/128)
  // a query tile is 128 rows: 128 tokens x 1 head, or 64 tokens x 2 heads
  if (tile == 128) {
    const bool two = (G % 2 == 0);
    if (p.D == 128) return two ? launch_cfg<E, 128, 128, 128, 2>(p, out, lse, sink_s, stream)
                               : launch_cfg<E, 128, 128, 128, 1>(p, out, lse, sink_s, stream);
    return two ? launch_cfg<E, 64, 128, 128, 2>(p, out, lse, sink_s, stream)
               : launch_cfg<E, 64, 128, 128, 1>(p, out, lse, sink_s, stream);
  }
  // 64-token tiles need two heads per query tile; key blocks are staged in
  // pairs as 128-key tiles.  At D = 64 a CTA holds one query tile and two
  // CTAs share an SM.
  if (G % 2 != 0) return SINKATTN_ERR_UNSUPPORTED;
  const bool two = (G % 4 == 0);
  if (p.D == 128) return two ? launch_cfg<E, 128, 64, 128, 2, true>(p, out, lse, sink_s, stream)
                             : launch_cfg<E, 128, 64, 128, 1, true>(p, out, lse, sink_s, stream);
  return launch_cfg<E, 64, 64, 128, 1, true, 2>(p, out, lse, sink_s, stream);
}

int launch_fwd_tc(const AttnProblem& p, void* out, float* lse, float* sink_s, cudaStream_t stream) {
  return p.dt == SINKATTN_FP16 ? launch_fwd_e<ElemF16>(p, out, lse, sink_s, stream)
                               : launch_fwd_e<ElemBf16>(p, out, lse, sink_s, stream);
}

}  // namespace sk
