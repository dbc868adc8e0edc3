// Backward pass on the tensor cores (tcgen05) for bf16 inputs.
//
// Page "Attention Sink, Learnable Sink and dsink", section 8: with the
// probabilities rebuilt from the sink-inclusive LSE, P = exp(x - L_new), and
// Delta taken from the sink-scaled output, the ordinary softmax gradients
//   dS = P * (dP - Delta),  dP = dO V^T
//   dV = P^T dO,  dK = alpha dS^T Q,  dQ = alpha dS K
// already carry the sink's effect; dsink comes from the preprocess
// (section 7) and is not touched here.  Section 10 describes a backward split
// by KV block over reverse lists; this kernel is that split.
//
// One CTA = one 128-key tile of one KV head (the plan's reverse list gives
// the query tiles that see it); it loops over (query tile, query head) pairs.
// Tensor memory (512 columns):
//   S^T  [keys x 128 query rows] fp32, overwritten in place by P^T (bf16,
//        packed two per column at the front of each warpgroup's slice)
//   dP^T [keys x 128] fp32, overwritten by dS^T (bf16, same packing); then reused for the
//        dQ tile [128 query rows x D] once dK has consumed dS^T
//   dK, dV [keys x D] fp32 accumulators for the whole CTA
// MMAs per (query tile, head), issued by one thread in this order:
//   S^T = K Q^T (SS) | dP^T = V dO^T (SS) | dV += P^T dO (TS) |
//   dK += dS^T Q (TS) | dQ = dS K (SS; dS^T also staged in shared memory)
// Warps 0-7 compute (warpgroup c owns query columns [64c, 64c + 64), thread =
// key row), warp 8 is the TMA producer, warp 9 issues MMAs, warp 10 flushes
// dQ.  The compute warps move each dQ tile out of tensor memory into the
// finished stage's shared memory; the reducer adds it into an fp32 buffer with
// bulk tensor reductions (a query row gets one contribution per visible key
// tile); a small kernel converts it to bf16.
#include "internal.h"

namespace sk {

namespace {

// KT = 128: 128-key tiles, query tiles of 128 tokens x 1 head.
// KT = 64 (64-key block selection): M = 64 for the key-side MMAs (tensor-memory
// rows m at lanes m % 16 + 32 (m / 16)), query tiles of 64 tokens x 2 heads so
// the dQ MMA keeps M = 128.
template <int D_, int KT_>
struct BwdCfg {
  static constexpr int D = D_, KT = KT_, TQ = KT_, HPT = 128 / KT_;
  static constexpr int DH = D / 64;
  static constexpr int Q_BYTES = 128 * D * 2;   // Q or dO tile (128 rows)
  static constexpr int KV_BYTES = KT * D * 2;   // K or V tile
  static constexpr int DS_BYTES = KT * 128 * 2; // dS^T tile
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int FIXED = 2 * KV_BYTES + DS_BYTES + 1024 /*lse, delta*/ + 512 /*bars*/ + 1024;
  static constexpr int NS_RAW = (SMEM_LIMIT - FIXED) / (2 * Q_BYTES);
  static constexpr int NS = NS_RAW > 4 ? 4 : NS_RAW;
  static_assert(NS >= 2, "shared memory");
  static constexpr int THREADS = 11 * 32;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, REDUCER_WARP = 10;
  static constexpr int S_COL = 0, DP_COL = 128, DK_COL = 256, DV_COL = 256 + D;
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_DS = OFF_V + KV_BYTES;
  static constexpr int OFF_Q = OFF_DS + DS_BYTES;
  static constexpr int OFF_DO = OFF_Q + NS * Q_BYTES;
  static constexpr int OFF_LSE = OFF_DO + NS * Q_BYTES;   // float[128]
  static constexpr int OFF_DL = OFF_LSE + 512;            // float[128]
  static constexpr int OFF_BAR = OFF_DL + 512;
  static constexpr int N_BARS = 1 + 3 * NS + 7;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static_assert(NS * Q_BYTES >= KT * D * 4, "Q stages must hold an fp32 dK tile");
};

struct BwdParams {
  const int* plan;
  const float* lse2;   // [Hq, T] head-major, log2 domain
  const float* delta;  // [Hq, T]
  float* dq_accum;     // [T, Hq, D] fp32
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int* status;
  int T_tot, Hq, Hkv, G, causal, n_sink, window, per_item;
  float scale_log2, alpha;
};

__device__ __forceinline__ bool wait_noabort(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudgetCycles) return false;
  return true;
}

// Packed bf16 P^T / dS^T columns: warpgroup c writes its 64 query columns
// as 32 packed words at the front of its own fp32 slice [64c, 64c + 64), so
// it never overwrites fp32 values the other warpgroup has yet to read.  K step
// kk (16 query columns) of the TS-MMA A operand therefore starts at:
__device__ __forceinline__ constexpr uint32_t a_col(int kk) { return (kk / 4) * 64 + (kk % 4) * 8; }

// fp32 add of a shared-memory box into global memory through the tensor map
// (bulk reduction; rows past the tensor's extent are skipped by the hardware)
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* smem_src,
                                                  int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                  const __grid_constant__ CUtensorMap tmap_do,
                  const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v,
                  const __grid_constant__ CUtensorMap tmap_dq,
                  const __grid_constant__ CUtensorMap tmap_dkacc,
                  const __grid_constant__ CUtensorMap tmap_dvacc, const BwdParams p) {
  constexpr int D = C::D, KT = C::KT, TQ = C::TQ, HPT = C::HPT, NS = C::NS, DH = C::DH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qf = bars + 1;
  uint64_t* bar_qe = bar_qf + NS;
  uint64_t* bar_dqs = bar_qe + NS;   // dQ tile of stage s staged in smem
  uint64_t* bar_s = bar_dqs + NS;
  uint64_t* bar_dp = bar_s + 1;
  uint64_t* bar_p = bar_dp + 1;
  uint64_t* bar_ds = bar_p + 1;
  uint64_t* bar_dq = bar_ds + 1;
  uint64_t* bar_dqf = bar_dq + 1;
  uint64_t* bar_fin = bar_dqf + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* s_dl = reinterpret_cast<float*>(smem + C::OFF_DL);

  const PlanHdr* hdr = reinterpret_cast<const PlanHdr*>(p.plan);
  const int rank = blockIdx.x / p.per_item;
  if (rank >= min(hdr->n_bwd_units, hdr->cap_units)) return;
  const int rem = blockIdx.x % p.per_item;
  // work unit: a slice of one key tile's reverse list (long lists are split)
  const int4 unit = reinterpret_cast<const int4*>(p.plan + hdr->off_bwd_units)[
      p.plan[hdr->off_bwd_unit_order + rank]];
  const TileItem it = reinterpret_cast<const TileItem*>(p.plan + hdr->off_bwd_items)[unit.x];
  const bool split_tile = unit.w > 1;  // partial dK/dV go through fp32 reductions
  const int kvh = it.kvh >= 0 ? it.kvh : rem;
  const int* ent = p.plan + hdr->off_bwd_entries + it.entry_off + unit.y;
  const int GH = p.G / HPT;             // query-head groups per key tile
  const int n_it = unit.z * GH;         // (query tile, head group) iterations
  const int k0 = it.tile_start;         // sequence-local first key

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_qf + s, 1);
      mbar_init(bar_qe + s, 1);    // released by the reducer warp
      mbar_init(bar_dqs + s, 256); // every compute thread staged its dQ part
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dqf, 256);
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
    prefetch_tensormap(&tmap_do);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
    prefetch_tensormap(&tmap_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_it > 0) {
      const int krow = it.seq_start + k0;
      mbar_expect_tx(bar_kv, 2 * C::KV_BYTES);
      for (int h = 0; h < DH; ++h) {
        tma_load_3d(smem + C::OFF_K + h * (C::KV_BYTES / DH), &tmap_k, bar_kv, h * 64, kvh, krow);
        tma_load_3d(smem + C::OFF_V + h * (C::KV_BYTES / DH), &tmap_v, bar_kv, h * 64, kvh, krow);
      }
      int last[NS];
      for (int s = 0; s < NS; ++s) last[s] = -1;
      bool ok = true;
      for (int i = 0; i < n_it && ok; ++i) {
        const int s = i % NS;
        const int e = __ldg(ent + i / GH);
        const int q_tok = it.seq_start + (e >> 1) * TQ;
        const int h0 = kvh * p.G + (i % GH) * HPT;
        ok = mbar_wait(bar_qe + s, ((i / NS) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        mbar_expect_tx(bar_qf + s, 2 * C::Q_BYTES);
        for (int h = 0; h < DH; ++h) {
          tma_load_3d(smem + C::OFF_Q + s * C::Q_BYTES + h * (C::Q_BYTES / DH), &tmap_q,
                      bar_qf + s, h * 64, h0, q_tok);
          tma_load_3d(smem + C::OFF_DO + s * C::Q_BYTES + h * (C::Q_BYTES / DH), &tmap_do,
                      bar_qf + s, h * 64, h0, q_tok);
        }
        last[s] = i;
      }
      if (!ok) {
        wait_noabort(bar_kv, 0);
        for (int s = 0; s < NS; ++s)
          if (last[s] >= 0) wait_noabort(bar_qf + s, (last[s] / NS) & 1);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_it > 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(KT, 128, 0, 0);   // S^T, dP^T
      constexpr uint32_t id_kv = idesc_bf16_f32(KT, D, 0, 1);    // dV, dK (B MN-major)
      constexpr uint32_t id_q = idesc_bf16_f32(128, D, 1, 1);    // dQ (A, B MN-major)
      const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V),
                     sDS = smem_u32(smem + C::OFF_DS), sQ = smem_u32(smem + C::OFF_Q),
                     sDO = smem_u32(smem + C::OFF_DO);
      bool ok = mbar_wait(bar_kv, 0, abort_flag, p.status);
      for (int i = 0; i < n_it && ok; ++i) {
        const int s = i % NS;
        ok = mbar_wait(bar_qf + s, (i / NS) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_s = sQ + s * C::Q_BYTES, do_s = sDO + s * C::Q_BYTES;
        // S^T = K Q^T (both K-major)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          mma_ss(tmem + C::S_COL,
                 sdesc_sw128(sK + (kk / 4) * (C::KV_BYTES / DH) + off, 16, 1024),
                 sdesc_sw128(q_s + (kk / 4) * (C::Q_BYTES / DH) + off, 16, 1024), id_s,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s);
        // dP^T = V dO^T, into the columns the previous dQ tile occupied
        if (i > 0) {
          ok = mbar_wait(bar_dqf, (i - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          mma_ss(tmem + C::DP_COL,
                 sdesc_sw128(sV + (kk / 4) * (C::KV_BYTES / DH) + off, 16, 1024),
                 sdesc_sw128(do_s + (kk / 4) * (C::Q_BYTES / DH) + off, 16, 1024), id_s,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_dp);
        // dV += P^T dO  (P^T bf16 in tensor memory over S^T; dO MN-major)
        ok = mbar_wait(bar_p, i & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::DV_COL, tmem + C::S_COL + a_col(kk),
                 sdesc_sw128(do_s + kk * 2048, C::Q_BYTES / DH, 1024), id_kv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q  (dS^T bf16 in tensor memory over dP^T)
        ok = mbar_wait(bar_ds, i & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::DK_COL, tmem + C::DP_COL + a_col(kk),
                 sdesc_sw128(q_s + kk * 2048, C::Q_BYTES / DH, 1024), id_kv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        // dQ = dS K  (A = dS from the staged dS^T tile, both MN-major)
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk)
          mma_ss(tmem + C::DP_COL, sdesc_sw128(sDS + kk * 2048, KT * 128, 1024),
                 sdesc_sw128(sK + kk * 2048, C::KV_BYTES / DH, 1024), id_q, kk > 0 ? 1u : 0u);
        mma_commit(bar_dq);  // stage s is released once its dQ tile has been flushed
      }
      mma_commit(bar_fin);
      wait_noabort(bar_fin, 0);
    }
  } else if (warp == C::REDUCER_WARP) {
    // ------------------------------------------------------------ dQ reducer
    // Adds each staged fp32 dQ tile into the global accumulator with bulk
    // tensor reductions, waits until they have read the stage, and hands the
    // stage back to the producer; the compute warps never wait for this.
    if (lane == 0 && n_it > 0) {
      for (int i = 0; i < n_it; ++i) {
        const int s = i % NS;
        if (!mbar_wait(bar_dqs + s, (i / NS) & 1, abort_flag, p.status)) break;
        const int e = __ldg(ent + i / GH);
        const int q_tok = it.seq_start + (e >> 1) * TQ;
        const int h0 = kvh * p.G + (i % GH) * HPT;
#pragma unroll
        for (int cw = 0; cw < 2; ++cw) {
          const uint8_t* stage = smem + (cw == 0 ? C::OFF_Q : C::OFF_DO) + s * C::Q_BYTES;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_reduce_add_3d(&tmap_dq, stage + c * (128 * 128), (D / 2) * cw + 32 * c, h0, q_tok);
        }
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(bar_qe + s);
      }
      bulk_wait0();  // reductions complete before the CTA exits
    }
  } else {
    // ------------------------------------------------------------ compute
    const int cw = warp / 4;          // query-column half
    const int wq = warp % 4;          // TMEM lane quadrant
    const int tw = wq * 32 + lane;    // 0..127 within the warpgroup
    // key row held by this thread's TMEM lane (with KT = 64 only lanes 0-15
    // of each quadrant carry rows; the others join the collective loads)
    const int r = KT == 128 ? tw : wq * 16 + (lane & 15);
    const bool row_ok = KT == 128 || lane < 16;
    const int kj = k0 + r;            // sequence-local key
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const float* lse_s = s_lse + 64 * cw;
    const float* dl_s = s_dl + 64 * cw;
    // The next iteration's entry and (for 64 of the threads) its LSE2 / Delta
    // values are loaded one iteration ahead, so global-load latency stays off
    // the critical path.
    auto fetch = [&](int i, int& e, float& l2, float& dl) {
      e = __ldg(ent + i / GH);
      l2 = INFINITY;
      dl = 0.f;
      if (tw < 64) {
        const int q0 = (e >> 1) * TQ;
        const int col = 64 * cw + tw;
        const int tok = col / HPT, hh = col % HPT;
        const int h0 = kvh * p.G + (i % GH) * HPT;
        if (tok < it.seq_len - q0) {
          const long long gi = (long long)(h0 + hh) * p.T_tot + it.seq_start + q0 + tok;
          l2 = __ldg(p.lse2 + gi);
          dl = __ldg(p.delta + gi);
        }
      }
    };
    int e_nx = 0;
    float l2_nx = INFINITY, dl_nx = 0.f;
    if (n_it > 0) fetch(0, e_nx, l2_nx, dl_nx);
    bool ok = true;
    for (int i = 0; i < n_it; ++i) {
      const int e = e_nx;
      const int q0 = (e >> 1) * TQ;
      const bool partial = (e & 1) != 0;
      const int h0 = kvh * p.G + (i % GH) * HPT;
      const int q_len = min(TQ, it.seq_len - q0);
      named_bar_sync(1 + cw, 128);  // previous iteration's smem reads are done
      if (tw < 64) {
        s_lse[64 * cw + tw] = l2_nx;
        s_dl[64 * cw + tw] = dl_nx;
      }
      named_bar_sync(1 + cw, 128);
      if (i + 1 < n_it) fetch(i + 1, e_nx, l2_nx, dl_nx);
      // P^T = exp2(S^T * alpha * log2e - LSE2), 32 columns at a time
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s, i & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      float P[64];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + C::S_COL + 64 * cw + 32 * h2, a);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c)
          P[32 * h2 + c] = fast_exp2(__uint_as_float(a[c]) * p.scale_log2 - lse_s[32 * h2 + c]);
      }
      if (partial) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int tok = (64 * cw + c) / HPT;
          if (!visible_elem(q0 + tok, kj, it.seq_len, p.causal, p.n_sink, p.window)) P[c] = 0.f;
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(P[2 * c], P[2 * c + 1]);
        tmem_st32(tmem + lane_off + C::S_COL + 64 * cw, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(bar_p);
      // dS^T = P^T * (dP^T - Delta)
      ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, i & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t ds[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + C::DP_COL + 64 * cw + 32 * h2, a);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int x = 32 * h2 + 2 * c;
          ds[16 * h2 + c] = pack_bf16x2(P[x] * (__uint_as_float(a[2 * c]) - dl_s[x]),
                                        P[x + 1] * (__uint_as_float(a[2 * c + 1]) - dl_s[x + 1]));
        }
      }
      tmem_st32(tmem + lane_off + C::DP_COL + 64 * cw, ds);
      // the previous dQ MMA must be done reading the staged dS tile
      if (i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_dq, (i - 1) & 1, abort_flag, p.status));
        if (!ok) break;
      }
      if (row_ok) {
        // row r of the [keys][64 queries] half-tile, 128-byte swizzle
        uint8_t* row = smem + C::OFF_DS + cw * (KT * 128) + r * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) * 16)) =
              make_uint4(ds[4 * j], ds[4 * j + 1], ds[4 * j + 2], ds[4 * j + 3]);
      }
      fence_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds);
      // dQ tile: lanes are query rows; this warpgroup takes D/2 columns, 32
      // at a time.  All MMAs of this iteration are complete, so the stage's
      // Q (warpgroup 0) or dO (warpgroup 1) buffer takes the fp32 values
      // (128-byte swizzle), and one thread adds them into the fp32 dQ buffer
      // with bulk tensor reductions.  Query rows past the sequence end carry
      // exact zeros (their P is 0), so adding them is harmless.
      ok = __all_sync(0xffffffffu, mbar_wait(bar_dq, i & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      {
        const int s = i % NS;
        uint8_t* stage = smem + (cw == 0 ? C::OFF_Q : C::OFF_DO) + s * C::Q_BYTES;
        const int qrow = tw;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::DP_COL + (D / 2) * cw + 32 * c, a);
          tmem_ld_wait();
          if (c == D / 64 - 1) {
            tc_fence_before();
            mbar_arrive(bar_dqf);  // the dP region may be overwritten
          }
          uint8_t* row = stage + c * (128 * 128) + qrow * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(row + ((j ^ (qrow & 7)) * 16)) =
                make_uint4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
        }
        fence_async_smem();
        mbar_arrive(bar_dqs + s);  // the reducer warp takes it from here
      }
    }
    // dK (warpgroup 0) and dV (warpgroup 1) rows of this key tile
    const bool have = n_it > 0 && ok &&
                      __all_sync(0xffffffffu, mbar_wait(bar_fin, 0, abort_flag, p.status));
    if (!split_tile) {
      const bool store = (n_it == 0 || have) && row_ok && kj < it.seq_len;
      __nv_bfloat16* dst_base = (cw == 0 ? p.dk : p.dv);
      uint4* dst = reinterpret_cast<uint4*>(dst_base + ((long long)(it.seq_start + kj) * p.Hkv + kvh) * D);
      const float f = cw == 0 ? p.alpha : 1.f;
      if (have) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + (cw == 0 ? C::DK_COL : C::DV_COL) + 32 * c, a);
          tmem_ld_wait();
          if (store) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[4 * c + v] = make_uint4(
                  pack_bf16x2(__uint_as_float(a[8 * v]) * f, __uint_as_float(a[8 * v + 1]) * f),
                  pack_bf16x2(__uint_as_float(a[8 * v + 2]) * f, __uint_as_float(a[8 * v + 3]) * f),
                  pack_bf16x2(__uint_as_float(a[8 * v + 4]) * f, __uint_as_float(a[8 * v + 5]) * f),
                  pack_bf16x2(__uint_as_float(a[8 * v + 6]) * f, __uint_as_float(a[8 * v + 7]) * f));
          }
        }
      } else if (store) {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      }
    } else if (have) {
      // Split key tile: add this unit's fp32 dK (warpgroup 0) / dV (warpgroup 1)
      // into the zeroed accumulators.  The Q (resp. dO) stages are reused for
      // staging once the reducer warp has released every stage this unit used.
      bool free_ok = true;
      for (int s = 0; s < NS && s < n_it; ++s) {
        const int last = s + ((n_it - 1 - s) / NS) * NS;  // last iteration on stage s
        free_ok = free_ok && mbar_wait(bar_qe + s, (last / NS) & 1, abort_flag, p.status);
      }
      free_ok = __all_sync(0xffffffffu, free_ok);
      tc_fence_after();
      uint8_t* stage = smem + (cw == 0 ? C::OFF_Q : C::OFF_DO);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + (cw == 0 ? C::DK_COL : C::DV_COL) + 32 * c, a);
        tmem_ld_wait();
        if (free_ok && row_ok) {
          // box c: [KT rows][32 floats], 128-byte swizzle
          uint8_t* row = stage + c * (KT * 128) + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) * 16)) =
                make_uint4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
        }
      }
      fence_async_smem();
      named_bar_sync(1 + cw, 128);
      if (free_ok && tw == 0) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          tma_reduce_add_3d(cw == 0 ? &tmap_dkacc : &tmap_dvacc, stage + c * (KT * 128), 32 * c,
                            kvh, it.seq_start + k0);
        bulk_commit();
        bulk_wait0();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Key tiles whose reverse list was split into several work units: zero their
// fp32 dK/dV accumulator rows before the backward kernel, and round them to
// bf16 (dK scaled by alpha) after it.  One CTA per backward item; unsplit
// items return at once.
__global__ void split_tiles_kernel(const int* plan, float* dk_acc, float* dv_acc,
                                   __nv_bfloat16* dk, __nv_bfloat16* dv, int Hkv, int D,
                                   float alpha, int finish) {
  // blockIdx.x = backward item, blockIdx.y = row of its key tile
  const PlanHdr* h = reinterpret_cast<const PlanHdr*>(plan);
  if ((int)blockIdx.x >= h->cap_items) return;
  const TileItem it = reinterpret_cast<const TileItem*>(plan + h->off_bwd_items)[blockIdx.x];
  if (it.entry_len < 0 || bwd_units_of(it.entry_len) <= 1 || (int)blockIdx.y >= it.tile_len) return;
  const int kv0 = it.kvh >= 0 ? it.kvh : 0, kv1 = it.kvh >= 0 ? it.kvh + 1 : Hkv;
  const long long base = ((long long)(it.seq_start + it.tile_start + blockIdx.y) * Hkv + kv0) * D;
  const int n4 = (kv1 - kv0) * D / 4;
  float4* ka = reinterpret_cast<float4*>(dk_acc + base);
  float4* va = reinterpret_cast<float4*>(dv_acc + base);
  for (int e = threadIdx.x; e < n4; e += blockDim.x) {
    if (finish) {
      const float4 x = ka[e], y = va[e];
      reinterpret_cast<uint2*>(dk + base)[e] =
          make_uint2(pack_bf16x2(x.x * alpha, x.y * alpha), pack_bf16x2(x.z * alpha, x.w * alpha));
      reinterpret_cast<uint2*>(dv + base)[e] =
          make_uint2(pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
    } else {
      ka[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      va[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// dQ = alpha * accumulated fp32, rounded to bf16.
__global__ void dq_convert_kernel(const float4* acc, uint2* dq, long long n4, float alpha) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = acc[i];
  dq[i] = make_uint2(pack_bf16x2(v.x * alpha, v.y * alpha), pack_bf16x2(v.z * alpha, v.w * alpha));
}

template <int D, int KT>
int launch_cfg(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  using C = BwdCfg<D, KT>;
  CUtensorMap mq, mdo, mk, mv, mdq, mdk, mdv;
  if (!make_tmap_3d(&mq, p.q, p.T_tot, p.Hq, D, C::HPT, C::TQ) ||
      !make_tmap_3d(&mdo, b.dout, p.T_tot, p.Hq, D, C::HPT, C::TQ) ||
      !make_tmap_3d(&mk, p.k, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d(&mv, p.v, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d_f32(&mdq, b.dq_accum, p.T_tot, p.Hq, D, C::HPT, C::TQ) ||
      !make_tmap_3d_f32(&mdk, b.dk_accum, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d_f32(&mdv, b.dv_accum, p.T_tot, p.Hkv, D, 1, C::KT))
    return SINKATTN_ERR_CUDA;
  BwdParams bp{};
  bp.plan = p.plan;
  bp.lse2 = b.lse2;
  bp.delta = b.delta;
  bp.dq_accum = b.dq_accum;
  bp.dk = static_cast<__nv_bfloat16*>(b.dk);
  bp.dv = static_cast<__nv_bfloat16*>(b.dv);
  bp.status = p.status;
  bp.T_tot = p.T_tot;
  bp.Hq = p.Hq;
  bp.Hkv = p.Hkv;
  bp.G = p.Hq / p.Hkv;
  bp.causal = p.causal;
  bp.n_sink = p.n_sink;
  bp.window = p.window;
  bp.per_item = p.ps.kh_slots == 1 ? p.Hkv : 1;
  bp.scale_log2 = p.scale * kLog2e;
  bp.alpha = p.scale;
  const size_t acc_bytes = sizeof(float) * (size_t)p.T_tot * p.Hq * D;
  if (cudaMemsetAsync(b.dq_accum, 0, acc_bytes, stream) != cudaSuccess) return SINKATTN_ERR_CUDA;
  const long long grid = (long long)p.ps.cap_units * bp.per_item;
  if (grid < 1 || grid > 0x7fffffffLL) return SINKATTN_ERR_INVALID_ARG;
  auto kern = bwd_tc_kernel<C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return SINKATTN_ERR_CUDA;
  const dim3 split_grid(p.ps.cap_items, C::KT);
  split_tiles_kernel<<<split_grid, 256, 0, stream>>>(p.plan, b.dk_accum, b.dv_accum, bp.dk, bp.dv,
                                                     p.Hkv, D, p.scale, 0);
  record_start(SINKATTN_KERNEL_BWD, stream);
  kern<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mdo, mk, mv, mdq, mdk, mdv, bp);
  record_stop(SINKATTN_KERNEL_BWD, stream);
  split_tiles_kernel<<<split_grid, 256, 0, stream>>>(p.plan, b.dk_accum, b.dv_accum, bp.dk, bp.dv,
                                                     p.Hkv, D, p.scale, 1);
  const long long n4 = (long long)p.T_tot * p.Hq * D / 4;
  dq_convert_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(b.dq_accum), reinterpret_cast<uint2*>(b.dq), n4, p.scale);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace

size_t bwd_tc_workspace_bytes(int T_tot, int Hq, int Hkv, int D) {
  return sizeof(float) * (size_t)T_tot * D * (Hq + 2 * Hkv);  // dQ, dK, dV accumulators
}

int launch_bwd_tc(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  if (p.ps.tile == 128)
    return p.D == 128 ? launch_cfg<128, 128>(p, b, stream) : launch_cfg<64, 128>(p, b, stream);
  if ((p.Hq / p.Hkv) % 2 != 0) return SINKATTN_ERR_UNSUPPORTED;  // 64-token tiles pair heads
  return p.D == 128 ? launch_cfg<128, 64>(p, b, stream) : launch_cfg<64, 64>(p, b, stream);
}

}  // namespace sk
