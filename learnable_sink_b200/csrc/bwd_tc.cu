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
// One CTA = one key tile of one KV head (a slice of the plan's reverse list
// gives the query tiles that see it); it loops over (query sub-tile, query
// head) pairs of QR = QT tokens x HPT heads = 64 or 128 query rows.
// Tensor memory (512 columns):
//   S^T  [keys x QR] fp32, overwritten in place by P^T (bf16, packed two per
//        column at the front of each compute warpgroup's slice)
//   dP^T [keys x QR] fp32, overwritten by dS^T (bf16, same packing) when dQ
//        has columns of its own
//   dK, dV [keys x D] fp32 accumulators for the whole CTA
//   dQ   [QR x D] fp32 in its own columns when they fit, else over dP^T once
//        the compute warps have read it
// MMAs of iteration i, issued by one thread:
//   dV += P^T dO (TS) | S^T(i+1) = K Q^T (SS) | dK += dS^T Q | dQ = dS K (SS;
//   dS^T staged in shared memory) | dP^T(i+1) = V dO^T (SS)
// With dQ in its own columns dK reads dS^T from tensor memory (TS) and goes
// first.  With dQ over dP^T, dQ goes first so that its readout overlaps dK
// (dP^T(i+1) waits for that readout), and dK reads the staged tile (SS).
// The tensor cores run dK/dQ of tile i while the compute warps
// exponentiate tile i+1 (S^T(i+1) moves behind dQ(i) when its Q tile has not
// landed yet).  Warps 0-7 compute (warpgroup c owns query columns
// [c QR/2, (c + 1) QR/2), thread = key row); warps 8-11 move each dQ tile out
// of tensor memory into shared memory the iteration's MMAs have finished
// reading (the stage's dO buffer, and the staged dS^T tile or the stage's Q
// buffer); warp 12 is the TMA
// producer, warp 13 issues MMAs and warp 14 adds the staged dQ tiles into an
// fp32 buffer with bulk tensor reductions (a query row gets one contribution
// per visible key tile); a small kernel converts it to bf16.
//
// Two limits shape the schedule: the tensor cores read shared-memory operands
// at about 128 bytes per cycle (a 128 x 128 x 16 SS MMA is already at that
// rate, so every other shared-memory byte slows the MMAs), and an SM drains
// about 20 bytes of dQ reductions per cycle, so a buffer that holds a staged
// fp32 dQ half stays busy until it has left.  Where the staged dS^T tile can
// hold half of dQ it takes it, so the Q buffer, which the next S^T needs
// first, goes back as soon as dK has read it (4 % on the D = 128 backward).
// With 128-key tiles the query side uses 128 rows per
// iteration: 64-row sub-tiles (supported by the template) halve the stage but
// re-read K and V twice as often, which costs more shared-memory bandwidth
// than the extra stages save.
#include "internal.h"

namespace sk {

namespace {

// KT = key-tile tokens (the plan's tile), QT x HPT = query rows per iteration.
//   <D, 128, 128, 1>: 128-key tiles, query tiles of 128 tokens x 1 head.
//   <D, 128, 64, 1>:  the same with 64-token sub-tiles; the dQ MMA then has
//                     M = 64 (tensor-memory rows m at lanes m % 16 + 32 (m / 16)).
//   <D, 64, 64, 2>:   64-key block selection: M = 64 for the key-side MMAs
//                     (same lane layout), query tiles of 64 tokens x 2 heads
//                     so the dQ MMA keeps M = 128.
template <int D_, int KT_, int QT_, int HPT_, class E_ = ElemBf16>
struct BwdCfg {
  using E = E_;  // 16-bit element type of Q, K, V, dO, P^T, dS^T and the gradients
  static constexpr int D = D_, KT = KT_, QT = QT_, HPT = HPT_;
  static constexpr int QR = QT * HPT;           // query rows per iteration
  static constexpr int NSUB = KT / QT;          // sub-tiles per plan tile
  static constexpr int CW = QR / 2;             // query columns per compute warpgroup
  static constexpr int DH = D / 64;
  static_assert(QR == 64 || QR == 128, "query rows");
  static_assert(KT != 64 || QR == 128, "64-key tiles take 128 query rows (two warpgroups of 64)");
  static constexpr int Q_BYTES = QR * D * 2;    // Q or dO tile
  static constexpr int KV_BYTES = KT * D * 2;   // K or V tile
  static constexpr int DS_BYTES = KT * QR * 2;  // dS^T tile
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int FIXED = 2 * KV_BYTES + DS_BYTES + 1024 /*lse, delta*/ + 512 /*bars*/ + 1024;
  static constexpr int NS_RAW = (SMEM_LIMIT - FIXED) / (2 * Q_BYTES);
  static constexpr int NS = NS_RAW > 4 ? 4 : NS_RAW;
  static_assert(NS >= 2, "shared memory");
  static constexpr int THREADS = 16 * 32;
  static constexpr int EPI_WARP0 = 8, PRODUCER_WARP = 12, MMA_WARP = 13, REDUCER_WARP = 14;
  // 2 compute warpgroups, 1 dQ-epilogue warpgroup, 1 warpgroup of single-warp
  // roles.  With 128 query rows a compute thread holds 64 probabilities and
  // registers move to the compute warpgroups; with 64 the launch split fits.
  static constexpr int LAUNCH_REGS = 65536 / THREADS;
  static constexpr bool REBALANCE = QR == 128;
  static constexpr bool DQ_OWN = 2 * QR + 3 * D <= 512;   // dQ in columns of its own
  // dQ over dP^T with a staged dS^T tile large enough for half a dQ tile:
  // that half is staged there, not in the stage's Q buffer
  static constexpr bool DQ_IN_DS = !DQ_OWN && KT * QR * 2 >= QR * D * 2;
  static constexpr int COMPUTE_REGS = REBALANCE ? 184 : LAUNCH_REGS;
  static constexpr int EPI_REGS = REBALANCE ? 72 : LAUNCH_REGS;
  static constexpr int AUX_REGS = REBALANCE ? 72 : LAUNCH_REGS;
  static_assert(256 * COMPUTE_REGS + 128 * EPI_REGS + 128 * AUX_REGS <= 65536,
                "register split exceeds the block's allocation");
  static constexpr int S_COL = 0, DP_COL = QR, DK_COL = 2 * QR, DV_COL = 2 * QR + D;
  static constexpr int DQ_COL = DQ_OWN ? 2 * QR + 2 * D : DP_COL;
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_DS = OFF_V + KV_BYTES;
  static constexpr int OFF_Q = OFF_DS + DS_BYTES;
  static constexpr int OFF_DO = OFF_Q + NS * Q_BYTES;
  static constexpr int OFF_LSE = OFF_DO + NS * Q_BYTES;   // float[QR]
  static constexpr int OFF_DL = OFF_LSE + 512;            // float[QR]
  static constexpr int OFF_BAR = OFF_DL + 512;
  static constexpr int N_BARS = 1 + 6 * NS + 9;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int OFF_ENT = OFF_MISC + 16;           // int[kBwdChunk]: the unit's entries
  static constexpr int SMEM_BYTES = OFF_ENT + 4 * kBwdChunk + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
  static_assert(NS * Q_BYTES >= KT * D * 4, "Q stages must hold an fp32 dK tile");
};

struct BwdParams {
  const int* plan;
  const float* lse2;   // [Hq, T] head-major, log2 domain
  const float* delta;  // [Hq, T]
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

// Packed bf16 P^T / dS^T columns: compute warpgroup c writes its CW query
// columns as CW/2 packed words at the front of its own fp32 slice
// [c CW, c CW + CW), so it never overwrites fp32 values the other warpgroup
// has yet to read.  K step kk (16 query columns) of the TS-MMA A operand
// therefore starts at:
template <int CW>
__device__ __forceinline__ constexpr uint32_t a_col(int kk) {
  return (kk / (CW / 16)) * CW + (kk % (CW / 16)) * 8;
}

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
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }


// M = 64 accumulators put row m at lane m % 16 + 32 (m / 16): the lower 16
// lanes of each warp's quadrant.  The 16x256b / 16x128b shapes spread those
// 16 lanes over all 32 threads: with .x8, thread t gets register 4k + 2h + e
// = (lane t/4 + 8h, column 8k + 2 (t % 4) + e) from a 64-column load, and
// stores register 2k + h to (lane t/4 + 8h, column 4k + t % 4).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_16x128b_x8(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

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
  constexpr int D = C::D, KT = C::KT, QT = C::QT, HPT = C::HPT, QR = C::QR, CW = C::CW;
  constexpr int NS = C::NS, DH = C::DH, NSUB = C::NSUB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars;
  // Each stage is two buffers, Q and dO, with their own barriers.  The dQ
  // tile is staged as columns [D/2, D) in the dO buffer and columns [0, D/2)
  // in the staged dS^T tile when that holds them (DQ_IN_DS: the Q buffer then
  // goes back to the producer as soon as dK has read it), else in the Q
  // buffer; each buffer that takes a half goes back as soon as the bulk
  // reduction has read its half.
  uint64_t* bar_qf = bars + 1;       // Q of stage s landed
  uint64_t* bar_df = bar_qf + NS;    // dO of stage s landed
  uint64_t* bar_qe = bar_df + NS;    // Q buffer of stage s free
  uint64_t* bar_de = bar_qe + NS;    // dO buffer of stage s free
  uint64_t* bar_dqs = bar_de + NS;   // dQ half 0 of stage s staged
  uint64_t* bar_dds = bar_dqs + NS;  // dQ half 1 of stage s staged in the dO buffer
  uint64_t* bar_s = bar_dds + NS;
  uint64_t* bar_dp = bar_s + 1;
  uint64_t* bar_p = bar_dp + 1;
  uint64_t* bar_ds = bar_p + 1;
  uint64_t* bar_dq = bar_ds + 1;
  uint64_t* bar_dqf = bar_dq + 1;
  uint64_t* bar_fin = bar_dqf + 1;
  uint64_t* bar_dk = bar_fin + 1;    // dK of the iteration complete (Q stage read)
  // dQ over dP^T: the dQ half staged in the dS^T buffer has been read, so the
  // next dS^T tile may be written there
  uint64_t* bar_dsf = bar_dk + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* s_ent = reinterpret_cast<int*>(smem + C::OFF_ENT);
  float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* s_dl = reinterpret_cast<float*>(smem + C::OFF_DL);

  const PlanHdr* hdr = reinterpret_cast<const PlanHdr*>(p.plan);
  // KV head slowest (lists shared by the KV heads): the CTAs of one
  // (KV head, sequence) are launched together
  const int rank = blockIdx.x % hdr->cap_units;
  if (rank >= min(hdr->n_bwd_units, hdr->cap_units)) return;
  const int rem = blockIdx.x / hdr->cap_units;
  // work unit: a slice of one key tile's reverse list (long lists are split)
  const int4 unit = reinterpret_cast<const int4*>(p.plan + hdr->off_bwd_units)[
      p.plan[hdr->off_bwd_unit_order + rank]];
  if (unit.z > kBwdChunk) {  // the plan never builds such a unit
    if (threadIdx.x == 0) set_status(p.status, SINKATTN_ERR_PLAN);
    return;
  }
  const TileItem it = reinterpret_cast<const TileItem*>(p.plan + hdr->off_bwd_items)[unit.x];
  const bool split_tile = unit.w > 1;  // partial dK/dV go through fp32 reductions
  const int kvh = it.kvh >= 0 ? it.kvh : rem;
  const int* ent = p.plan + hdr->off_bwd_entries + it.entry_off + unit.y;
  // iteration i: entry i / PER_E, head group (i % PER_E) / NSUB, sub-tile i % NSUB
  const int GH = p.G / HPT;
  const int PER_E = GH * NSUB;
  const int n_it = unit.z * PER_E;
  const int k0 = it.tile_start;         // sequence-local first key

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the unit's reverse-list entries, read from shared memory by every role
  // (a unit has at most kBwdChunk of them)
  if ((int)threadIdx.x < unit.z) s_ent[threadIdx.x] = __ldg(ent + threadIdx.x);
  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_qf + s, 1);
      mbar_init(bar_df + s, 1);
      mbar_init(bar_qe + s, 1);    // released by the reducer or the MMA warp
      mbar_init(bar_de + s, 1);
      mbar_init(bar_dqs + s, 128); // every epilogue thread staged its part of the half
      mbar_init(bar_dds + s, 128);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dqf, 128);
    mbar_init(bar_fin, 1);
    mbar_init(bar_dk, 1);
    mbar_init(bar_dsf, 1);
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

  // sequence-local first query token and first query head of iteration i
  // (entry e of the reverse list)
  auto q_first = [&](int i, int e) { return (e >> 1) * KT + (i % NSUB) * QT; };
  auto h_first = [&](int i) { return kvh * p.G + ((i % PER_E) / NSUB) * HPT; };

  if (warp >= C::PRODUCER_WARP) {
    regs_to<C::AUX_REGS, C::LAUNCH_REGS>();
    if (warp == C::PRODUCER_WARP) {
      // ---------------------------------------------------------- producer
      if (lane == 0 && n_it > 0) {
        const int krow = it.seq_start + k0;
        mbar_expect_tx(bar_kv, 2 * C::KV_BYTES);
        for (int h = 0; h < DH; ++h) {
          tma_load_3d(smem + C::OFF_K + h * (C::KV_BYTES / DH), &tmap_k, bar_kv, h * 64, kvh, krow);
          tma_load_3d(smem + C::OFF_V + h * (C::KV_BYTES / DH), &tmap_v, bar_kv, h * 64, kvh, krow);
        }
        int last[NS], lastd[NS];  // last iteration loaded into each Q / dO buffer
        for (int s = 0; s < NS; ++s) last[s] = lastd[s] = -1;
        bool ok = true;
        for (int i = 0; i < n_it && ok; ++i) {
          const int s = i % NS;
          const int e = s_ent[i / PER_E];
          const int q_tok = it.seq_start + q_first(i, e);
          const int h0 = h_first(i);
          const uint32_t par = ((i / NS) & 1) ^ 1;
          ok = mbar_wait(bar_qe + s, par, abort_flag, p.status);
          if (!ok) break;
          mbar_expect_tx(bar_qf + s, C::Q_BYTES);
          for (int h = 0; h < DH; ++h)
            tma_load_3d(smem + C::OFF_Q + s * C::Q_BYTES + h * (C::Q_BYTES / DH), &tmap_q,
                        bar_qf + s, h * 64, h0, q_tok);
          last[s] = i;
          ok = mbar_wait(bar_de + s, par, abort_flag, p.status);
          if (!ok) break;
          mbar_expect_tx(bar_df + s, C::Q_BYTES);
          for (int h = 0; h < DH; ++h)
            tma_load_3d(smem + C::OFF_DO + s * C::Q_BYTES + h * (C::Q_BYTES / DH), &tmap_do,
                        bar_df + s, h * 64, h0, q_tok);
          lastd[s] = i;
        }
        if (!ok) {
          wait_noabort(bar_kv, 0);
          for (int s = 0; s < NS; ++s) {
            if (last[s] >= 0) wait_noabort(bar_qf + s, (last[s] / NS) & 1);
            if (lastd[s] >= 0) wait_noabort(bar_df + s, (lastd[s] / NS) & 1);
          }
        }
      }
    } else if (warp == C::MMA_WARP) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0 && n_it > 0) {
        constexpr uint32_t id_s = idesc_16_f32(C::E::kFmt, KT, QR, 0, 0);  // S^T, dP^T
        constexpr uint32_t id_kv = idesc_16_f32(C::E::kFmt, KT, D, 0, 1);  // dV, dK (B MN-major)
        constexpr uint32_t id_q = idesc_16_f32(C::E::kFmt, QR, D, 1, 1);   // dQ (A, B MN-major)
        // operand descriptors at the start of each buffer, K-major (k*) and
        // MN-major (m*); every operand is a fixed byte offset from one of them
        const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V),
                       sDS = smem_u32(smem + C::OFF_DS), sQ = smem_u32(smem + C::OFF_Q),
                       sDO = smem_u32(smem + C::OFF_DO);
        const uint32_t kK = sdesc_lo(sK, 16), kV = sdesc_lo(sV, 16), kQ = sdesc_lo(sQ, 16),
                       kDO = sdesc_lo(sDO, 16), kDS = sdesc_lo(sDS, 16);
        const uint32_t mQ = sdesc_lo(sQ, C::Q_BYTES / DH), mDO = sdesc_lo(sDO, C::Q_BYTES / DH),
                       mDS = sdesc_lo(sDS, KT * 128), mK = sdesc_lo(sK, C::KV_BYTES / DH);
        // S^T = K Q^T (both K-major) of iteration j; its Q/dO stage has landed
        auto issue_s = [&](int j) {
          const uint32_t q_off = (j % NS) * C::Q_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_ss(tmem + C::S_COL, sdesc_at(kK, (kk / 4) * (C::KV_BYTES / DH) + off),
                   sdesc_at(kQ, q_off + (kk / 4) * (C::Q_BYTES / DH) + off), id_s,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_s);
        };
        // dP^T = V dO^T of iteration j (its dO tile has landed)
        auto issue_dp = [&](int j) {
          const uint32_t do_off = (j % NS) * C::Q_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_ss(tmem + C::DP_COL, sdesc_at(kV, (kk / 4) * (C::KV_BYTES / DH) + off),
                   sdesc_at(kDO, do_off + (kk / 4) * (C::Q_BYTES / DH) + off), id_s,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_dp);
        };
        bool ok = mbar_wait(bar_kv, 0, abort_flag, p.status) &&
                  mbar_wait(bar_qf, 0, abort_flag, p.status);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          ok = mbar_wait(bar_df, 0, abort_flag, p.status);
          tc_fence_after();
          if (ok) issue_dp(0);
        }
        for (int i = 0; i < n_it && ok; ++i) {
          const int s = i % NS;
          const uint32_t st_off = s * C::Q_BYTES;  // this iteration's Q / dO stage
          const bool more = i + 1 < n_it;
          const int s1 = (i + 1) % NS;
          const uint32_t par1 = ((i + 1) / NS) & 1;
          // dV += P^T dO  (P^T bf16 in tensor memory over S^T; dO MN-major)
          ok = mbar_wait(bar_p, i & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < QR / 16; ++kk)
            mma_ts(tmem + C::DV_COL, tmem + C::S_COL + a_col<CW>(kk),
                   sdesc_at(mDO, st_off + kk * 2048), id_kv,
                   (i > 0 || kk > 0) ? 1u : 0u);
          // S^T of the next iteration right behind dV (which frees the S^T
          // columns), if its tiles are already in shared memory
          bool s_next = false;
          if (more && mbar_try_wait(bar_qf + s1, par1)) {
            tc_fence_after();
            issue_s(i + 1);
            s_next = true;
          }
          ok = mbar_wait(bar_ds, i & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          // dQ = dS K  (A = dS from the staged dS^T tile, both MN-major)
          auto issue_dq = [&]() {
#pragma unroll
            for (int kk = 0; kk < KT / 16; ++kk)
              mma_ss(tmem + C::DQ_COL, sdesc_at(mDS, kk * 2048), sdesc_at(mK, kk * 2048), id_q,
                     kk > 0 ? 1u : 0u);
            mma_commit(bar_dq);  // the stage is released once its dQ tile has been flushed
          };
          if constexpr (C::DQ_OWN) {
            // dK += dS^T Q  (dS^T bf16 in tensor memory over dP^T), then dQ
            // once the previous tile was read out of its columns
#pragma unroll
            for (int kk = 0; kk < QR / 16; ++kk)
              mma_ts(tmem + C::DK_COL, tmem + C::DP_COL + a_col<CW>(kk),
                     sdesc_at(mQ, st_off + kk * 2048), id_kv, (i > 0 || kk > 0) ? 1u : 0u);
            if (i > 0) {
              ok = mbar_wait(bar_dqf, (i - 1) & 1, abort_flag, p.status);
              if (!ok) break;
              tc_fence_after();
            }
            issue_dq();
          } else {
            // dQ first, then dK += dS^T Q with A = the staged tile read K-major
            // (keys are its rows, 64 queries per 128-byte row; Q MN-major)
            issue_dq();
#pragma unroll
            for (int kk = 0; kk < QR / 16; ++kk)
              mma_ss(tmem + C::DK_COL,
                     sdesc_at(kDS, (kk / 4) * (KT * 128) + (kk & 3) * 32),
                     sdesc_at(mQ, st_off + kk * 2048), id_kv,
                     (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar_dk);  // what dK read may now take half of dQ
          if constexpr (C::DQ_IN_DS) mma_commit(bar_qe + s);  // dK read the Q buffer last
          if (more) {
            if (!s_next) {
              ok = mbar_wait(bar_qf + s1, par1, abort_flag, p.status);
              if (!ok) break;
              tc_fence_after();
              issue_s(i + 1);
            }
            if (!C::DQ_OWN) {  // dP^T(i+1) overwrites the dQ tile
              ok = mbar_wait(bar_dqf, i & 1, abort_flag, p.status);
              if (!ok) break;
            }
            ok = mbar_wait(bar_df + s1, par1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            issue_dp(i + 1);
          }
        }
        mma_commit(bar_fin);
        wait_noabort(bar_fin, 0);
      }
    } else if (warp == C::REDUCER_WARP) {
      // ---------------------------------------------------------- dQ reducer
      // Adds each staged fp32 dQ tile into the global accumulator with bulk
      // tensor reductions, waits until they have read each half, and hands
      // the dO buffer (and the Q buffer) back to the producer, or the staged
      // dS^T tile back to the compute warps.
      if (lane == 0 && n_it > 0) {
        for (int i = 0; i < n_it; ++i) {
          const int s = i % NS;
          const int e = s_ent[i / PER_E];
          const int q_tok = it.seq_start + q_first(i, e);
          const int h0 = h_first(i);
          const uint32_t par = (i / NS) & 1;
          bool got = true;
#pragma unroll
          for (int half = 0; half < 2 && got; ++half) {
            got = mbar_wait((half == 0 ? bar_dqs : bar_dds) + s, par, abort_flag, p.status);
            if (!got) break;
            const uint8_t* stage =
                half == 0 ? (C::DQ_IN_DS ? smem + C::OFF_DS : smem + C::OFF_Q + s * C::Q_BYTES)
                          : smem + C::OFF_DO + s * C::Q_BYTES;
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_reduce_add_3d(&tmap_dq, stage + c * (QR * 128), (D / 2) * half + 32 * c, h0,
                                q_tok);
            bulk_commit();
          }
          if (!got) break;
          bulk_wait_read1();         // the first half has been read
          mbar_arrive(C::DQ_IN_DS ? bar_dsf : bar_qe + s);
          bulk_wait_read0();         // the dO-buffer half too
          mbar_arrive(bar_de + s);
        }
        bulk_wait0();  // reductions complete before the CTA exits
      }
    }  // warp 15: idle
  } else if (warp >= C::EPI_WARP0) {
    // ------------------------------------------------------------ dQ epilogue
    // Query row m of the dQ tile sits at lane m (QR = 128) or at lane
    // m % 16 + 32 (m / 16) (QR = 64).  Columns [0, D/2) go to the staged dS^T
    // tile (DQ_IN_DS) or the stage's Q buffer, columns [D/2, D) to its dO
    // buffer, as fp32 boxes of 32 columns with the 128-byte swizzle.  Query
    // rows past the sequence end carry exact zeros (their P is 0), so adding
    // them is harmless.
    regs_to<C::EPI_REGS, C::LAUNCH_REGS>();
    const int wq = warp % 4;
    const bool lane_ok = QR == 128 || lane < 16;
    const int qrow = QR == 128 ? wq * 32 + lane : wq * 16 + (lane & 15);
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    for (int i = 0; i < n_it; ++i) {
      const int s = i % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dq, i & 1, abort_flag, p.status))) break;
      tc_fence_after();
      if constexpr (C::DQ_OWN) {
        // every MMA of the iteration is complete
#pragma unroll
        for (int c32 = 0; c32 < D / 32; ++c32) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::DQ_COL + 32 * c32, a);
          tmem_ld_wait();
          if (c32 == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar_dqf);  // the dQ columns may be overwritten
          }
          const int half = c32 / (D / 64), c = c32 % (D / 64);
          uint8_t* row = smem + (half == 0 ? C::OFF_Q : C::OFF_DO) + s * C::Q_BYTES +
                         c * (QR * 128) + qrow * 128;
          if (lane_ok) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(row + ((j ^ (qrow & 7)) * 16)) =
                  make_uint4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
          }
          if (c == D / 64 - 1) {  // a half is staged: the reducer warp takes it from here
            fence_async_smem();
            mbar_arrive((half == 0 ? bar_dqs : bar_dds) + s);
          }
        }
      } else {
        // Half 1 (columns [D/2, D), into the dO buffer, which dV and dP^T read
        // before dQ ran) first, then, once dK is complete, half 0 (into the
        // staged dS^T tile or the Q buffer, which dK reads); 32 columns at a
        // time.  The dQ columns are
        // released after the last load, so dK(i + 1) cannot complete before
        // this wait for dK(i).
        bool got_dk = true;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          const int hf = q < D / 64 ? 1 : 0;
          const int c = q % (D / 64);  // 32-column box within the half
          if (q == D / 64) got_dk = __all_sync(0xffffffffu, mbar_wait(bar_dk, i & 1, abort_flag, p.status));
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::DQ_COL + hf * (D / 2) + 32 * c, a);
          tmem_ld_wait();
          if (q == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar_dqf);  // the dQ columns may be overwritten
          }
          if (lane_ok && got_dk) {
            uint8_t* row = (hf == 0 ? (C::DQ_IN_DS ? smem + C::OFF_DS : smem + C::OFF_Q + s * C::Q_BYTES)
                                    : smem + C::OFF_DO + s * C::Q_BYTES) +
                           c * (QR * 128) + qrow * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(row + ((j ^ (qrow & 7)) * 16)) =
                  make_uint4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
          }
          if (c == D / 64 - 1) {  // the half is staged: the reducer warp takes it from here
            fence_async_smem();
            mbar_arrive((hf == 0 ? bar_dqs : bar_dds) + s);
          }
        }
        if (!got_dk) break;
      }
    }
  } else {
    // ------------------------------------------------------------ compute
    regs_to<C::COMPUTE_REGS, C::LAUNCH_REGS>();
    const int cw = warp / 4;          // query-column block
    const int wq = warp % 4;          // TMEM lane quadrant
    const int tw = wq * 32 + lane;    // 0..127 within the warpgroup
    // key row held by this thread's TMEM lane (with KT = 64 only lanes 0-15
    // of each quadrant carry rows; the others join the collective loads)
    const int r = KT == 128 ? tw : wq * 16 + (lane & 15);
    const bool row_ok = KT == 128 || lane < 16;
    const int kj = k0 + r;            // sequence-local key
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const float* lse_s = s_lse + CW * cw;
    const float* dl_s = s_dl + CW * cw;
    // KT = 64 (M = 64 tiles): the two key rows and the column offset of this
    // thread in the 16x256b layout
    const int r2[2] = {wq * 16 + lane / 4, wq * 16 + lane / 4 + 8};
    const int cq = 2 * (lane & 3);
    // The next iteration's entry and (for CW of the threads) its LSE2 / Delta
    // values are loaded one iteration ahead, so global-load latency stays off
    // the critical path.
    auto fetch = [&](int i, int& e, float& l2, float& dl) {
      e = s_ent[i / PER_E];
      l2 = INFINITY;
      dl = 0.f;
      if (tw < CW) {
        const int q0 = q_first(i, e);
        const int col = CW * cw + tw;
        const int tok = col / HPT, hh = col % HPT;
        if (tok < it.seq_len - q0) {
          const long long gi = (long long)(h_first(i) + hh) * p.T_tot + it.seq_start + q0 + tok;
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
      const int q0 = q_first(i, e);
      const bool partial = (e & 1) != 0;
      named_bar_sync(1 + cw, 128);  // previous iteration's smem reads are done
      if (tw < CW) {
        s_lse[CW * cw + tw] = l2_nx;
        s_dl[CW * cw + tw] = dl_nx;
      }
      named_bar_sync(1 + cw, 128);
      if (i + 1 < n_it) fetch(i + 1, e_nx, l2_nx, dl_nx);
      // P^T = exp2(S^T * alpha * log2e - LSE2), 32 columns at a time
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s, i & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      // KT = 64: every thread of the warp takes part (rows r2[h], columns
      // 8k + cq + e); otherwise thread = key row, CW columns
      constexpr int NP = KT == 64 ? 32 : CW;
      float P[NP];
      if constexpr (KT == 64) {
        uint32_t a[32];
        tmem_ld_16x256b_x8(tmem + lane_off + C::S_COL + CW * cw, a);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 l = *reinterpret_cast<const float2*>(lse_s + 8 * k + cq);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            P[4 * k + 2 * h] = fast_exp2(__uint_as_float(a[4 * k + 2 * h]) * p.scale_log2 - l.x);
            P[4 * k + 2 * h + 1] = fast_exp2(__uint_as_float(a[4 * k + 2 * h + 1]) * p.scale_log2 - l.y);
          }
        }
        if (partial) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const KeySpan ks = key_span(k0 + r2[h], q0, it.seq_len, p.causal, p.n_sink, p.window);
#pragma unroll
            for (int k = 0; k < 8; ++k)
#pragma unroll
              for (int e2 = 0; e2 < 2; ++e2) {
                const int tok = (CW * cw + 8 * k + cq + e2) / HPT;
                if (tok < ks.lo || tok > ks.hi) P[4 * k + 2 * h + e2] = 0.f;
              }
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
          for (int h = 0; h < 2; ++h) pk[2 * k + h] = C::E::pack(P[4 * k + 2 * h], P[4 * k + 2 * h + 1]);
        tmem_st_16x128b_x8(tmem + lane_off + C::S_COL + CW * cw, pk);
        tmem_st_wait();
      } else {
#pragma unroll
        for (int h2 = 0; h2 < CW / 32; ++h2) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::S_COL + CW * cw + 32 * h2, a);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c)
            P[32 * h2 + c] = fast_exp2(__uint_as_float(a[c]) * p.scale_log2 - lse_s[32 * h2 + c]);
        }
        if (partial) {
          const KeySpan ks = key_span(kj, q0, it.seq_len, p.causal, p.n_sink, p.window);
#pragma unroll
          for (int c = 0; c < CW; ++c) {
            const int tok = (CW * cw + c) / HPT;
            if (tok < ks.lo || tok > ks.hi) P[c] = 0.f;
          }
        }
        {
          uint32_t pk[CW / 2];
#pragma unroll
          for (int c = 0; c < CW / 2; ++c) pk[c] = C::E::pack(P[2 * c], P[2 * c + 1]);
          if constexpr (CW == 64)
            tmem_st32(tmem + lane_off + C::S_COL + CW * cw, pk);
          else
            tmem_st16(tmem + lane_off + C::S_COL + CW * cw, pk);
          tmem_st_wait();
        }
      }
      tc_fence_before();
      mbar_arrive(bar_p);
      // dS^T = P^T * (dP^T - Delta)
      ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, i & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      if constexpr (KT == 64) {
        uint32_t a[32];
        tmem_ld_16x256b_x8(tmem + lane_off + C::DP_COL + CW * cw, a);
        tmem_ld_wait();
        uint32_t dsk[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 d = *reinterpret_cast<const float2*>(dl_s + 8 * k + cq);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            dsk[2 * k + h] = C::E::pack(P[4 * k + 2 * h] * (__uint_as_float(a[4 * k + 2 * h]) - d.x),
                                         P[4 * k + 2 * h + 1] * (__uint_as_float(a[4 * k + 2 * h + 1]) - d.y));
        }
        if constexpr (C::DQ_OWN)  // dK reads dS^T from tensor memory
          tmem_st_16x128b_x8(tmem + lane_off + C::DP_COL + CW * cw, dsk);
        // staged tile (free as below): key row r2[h], queries CW cw + 8k + cq,
        // + 1 as one 4-byte word of 16-byte chunk k
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint8_t* row = smem + C::OFF_DS + ((CW * cw) / 64) * (KT * 128) + r2[h] * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint32_t*>(row + ((k ^ (r2[h] & 7)) * 16) + 2 * cq) = dsk[2 * k + h];
        }
      } else {
        uint32_t ds[CW / 2];
#pragma unroll
        for (int h2 = 0; h2 < CW / 32; ++h2) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::DP_COL + CW * cw + 32 * h2, a);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int x = 32 * h2 + 2 * c;
            ds[16 * h2 + c] = C::E::pack(P[x] * (__uint_as_float(a[2 * c]) - dl_s[x]),
                                          P[x + 1] * (__uint_as_float(a[2 * c + 1]) - dl_s[x + 1]));
          }
        }
        if constexpr (C::DQ_OWN) {  // dK reads dS^T from tensor memory
          if constexpr (CW == 64)
            tmem_st32(tmem + lane_off + C::DP_COL + CW * cw, ds);
          else
            tmem_st16(tmem + lane_off + C::DP_COL + CW * cw, ds);
        }
        // The staged dS tile is free of MMA reads: dP^T of this iteration was
        // issued after the previous dQ and dK MMAs, and its completion covers
        // them (with DQ_IN_DS the wait above covers the dQ half staged there
        // since).  Layout:
        // [QR / 64 atoms][keys][64 queries] with the 128-byte swizzle; dQ reads
        // it MN-major and (with dQ over dP^T) dK K-major.
        if constexpr (C::DQ_IN_DS) {
          if (i > 0) {  // the dQ half staged here in the previous iteration has been read
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dsf, (i - 1) & 1, abort_flag, p.status));
            if (!ok) break;
          }
        }
        if (row_ok) {
          constexpr int CHUNKS = CW / 8;  // 16-byte chunks of this warpgroup's queries
          uint8_t* row = smem + C::OFF_DS + ((CW * cw) / 64) * (KT * 128) + r * 128;
          const int j0 = ((CW * cw) % 64) / 8;
#pragma unroll
          for (int j = 0; j < CHUNKS; ++j)
            *reinterpret_cast<uint4*>(row + (((j0 + j) ^ (r & 7)) * 16)) =
                make_uint4(ds[4 * j], ds[4 * j + 1], ds[4 * j + 2], ds[4 * j + 3]);
        }
      }
      fence_async_smem();
      if constexpr (C::DQ_OWN) tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds);
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
                  C::E::pack(__uint_as_float(a[8 * v]) * f, __uint_as_float(a[8 * v + 1]) * f),
                  C::E::pack(__uint_as_float(a[8 * v + 2]) * f, __uint_as_float(a[8 * v + 3]) * f),
                  C::E::pack(__uint_as_float(a[8 * v + 4]) * f, __uint_as_float(a[8 * v + 5]) * f),
                  C::E::pack(__uint_as_float(a[8 * v + 6]) * f, __uint_as_float(a[8 * v + 7]) * f));
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
        free_ok = free_ok && mbar_wait((cw == 0 ? bar_qe : bar_de) + s, (last / NS) & 1, abort_flag,
                                       p.status);
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
// bf16 (dK scaled by alpha) after it.  CTA (item, chunk of kSplitRows rows of
// its key tile); unsplit items return at once.  A thread moves kSplitVec
// float4 of each accumulator, all loads before the stores.
constexpr int kSplitRows = 16;
constexpr int kSplitVec = 4;
template <class E>
__global__ void __launch_bounds__(256) split_tiles_kernel(const int* plan, float* dk_acc,
                                                          float* dv_acc, __nv_bfloat16* dk,
                                                          __nv_bfloat16* dv, int Hkv, int D,
                                                          float alpha, int finish) {
  const PlanHdr* h = reinterpret_cast<const PlanHdr*>(plan);
  if ((int)blockIdx.x >= h->cap_items) return;
  const TileItem it = reinterpret_cast<const TileItem*>(plan + h->off_bwd_items)[blockIdx.x];
  const int row0 = blockIdx.y * kSplitRows;
  if (it.entry_len < 0 || bwd_units_of(it.entry_len) <= 1 || row0 >= it.tile_len) return;
  const int kv0 = it.kvh >= 0 ? it.kvh : 0, kv1 = it.kvh >= 0 ? it.kvh + 1 : Hkv;
  const int n4 = (kv1 - kv0) * D / 4;  // float4 per token row of the item
  const long long tok0 = it.seq_start + it.tile_start + row0;
  const int total = min(kSplitRows, it.tile_len - row0) * n4;
  for (int e0 = threadIdx.x; e0 < total; e0 += 256 * kSplitVec) {
    long long off[kSplitVec];
#pragma unroll
    for (int u = 0; u < kSplitVec; ++u) {
      const int e = min(e0 + u * 256, total - 1);
      const int row = e / n4;
      off[u] = ((tok0 + row) * Hkv + kv0) * D / 4 + (e - row * n4);
    }
    if (finish) {
      float4 x[kSplitVec], y[kSplitVec];
#pragma unroll
      for (int u = 0; u < kSplitVec; ++u) {
        x[u] = __ldcs(reinterpret_cast<const float4*>(dk_acc) + off[u]);
        y[u] = __ldcs(reinterpret_cast<const float4*>(dv_acc) + off[u]);
      }
#pragma unroll
      for (int u = 0; u < kSplitVec; ++u) {
        if (e0 + u * 256 >= total) break;
        reinterpret_cast<uint2*>(dk)[off[u]] = make_uint2(
            E::pack(x[u].x * alpha, x[u].y * alpha), E::pack(x[u].z * alpha, x[u].w * alpha));
        reinterpret_cast<uint2*>(dv)[off[u]] =
            make_uint2(E::pack(y[u].x, y[u].y), E::pack(y[u].z, y[u].w));
      }
    } else {
#pragma unroll
      for (int u = 0; u < kSplitVec; ++u) {
        if (e0 + u * 256 >= total) break;
        reinterpret_cast<float4*>(dk_acc)[off[u]] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(dv_acc)[off[u]] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

// dQ = alpha * accumulated fp32, rounded to bf16: kDqVec float4 a thread, all
// loads issued before the stores.
constexpr int kDqVec = 4;
template <class E>
__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* acc, uint2* dq, long long n4,
                                                         float alpha) {
  const long long i0 = (long long)blockIdx.x * (256 * kDqVec) + threadIdx.x;
  float4 v[kDqVec];
#pragma unroll
  for (int u = 0; u < kDqVec; ++u) {
    const long long i = i0 + u * 256;
    v[u] = i < n4 ? __ldcs(acc + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < kDqVec; ++u) {
    const long long i = i0 + u * 256;
    if (i < n4)
      dq[i] = make_uint2(E::pack(v[u].x * alpha, v[u].y * alpha),
                         E::pack(v[u].z * alpha, v[u].w * alpha));
  }
}

template <class C>
int launch_cfg(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  constexpr int D = C::D;
  CUtensorMap mq, mdo, mk, mv, mdq, mdk, mdv;
  if (!make_tmap_3d(&mq, p.q, p.T_tot, p.Hq, D, C::HPT, C::QT) ||
      !make_tmap_3d(&mdo, b.dout, p.T_tot, p.Hq, D, C::HPT, C::QT) ||
      !make_tmap_3d(&mk, p.k, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d(&mv, p.v, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d_f32(&mdq, b.dq_accum, p.T_tot, p.Hq, D, C::HPT, C::QT) ||
      !make_tmap_3d_f32(&mdk, b.dk_accum, p.T_tot, p.Hkv, D, 1, C::KT) ||
      !make_tmap_3d_f32(&mdv, b.dv_accum, p.T_tot, p.Hkv, D, 1, C::KT))
    return SINKATTN_ERR_CUDA;
  BwdParams bp{};
  bp.plan = p.plan;
  bp.lse2 = b.lse2;
  bp.delta = b.delta;
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
  if constexpr (C::REBALANCE) {
    // the register split assumes the launch-bound count per thread; with
    // fewer, a setmaxnreg.inc would wait for registers that never come
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != C::LAUNCH_REGS)
      return SINKATTN_ERR_UNSUPPORTED;
  }
  const dim3 split_grid(p.ps.cap_items, (C::KT + kSplitRows - 1) / kSplitRows);
  split_tiles_kernel<typename C::E><<<split_grid, 256, 0, stream>>>(
      p.plan, b.dk_accum, b.dv_accum, bp.dk, bp.dv, p.Hkv, D, p.scale, 0);
  record_start(SINKATTN_KERNEL_BWD, stream);
  kern<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mdo, mk, mv, mdq, mdk, mdv, bp);
  record_stop(SINKATTN_KERNEL_BWD, stream);
  split_tiles_kernel<typename C::E><<<split_grid, 256, 0, stream>>>(
      p.plan, b.dk_accum, b.dv_accum, bp.dk, bp.dv, p.Hkv, D, p.scale, 1);
  const long long n4 = (long long)p.T_tot * p.Hq * D / 4;
  dq_convert_kernel<typename C::E><<<(unsigned)((n4 + 256 * kDqVec - 1) / (256 * kDqVec)), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(b.dq_accum), reinterpret_cast<uint2*>(b.dq), n4, p.scale);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace

size_t bwd_tc_workspace_bytes(int T_tot, int Hq, int Hkv, int D) {
  return sizeof(float) * (size_t)T_tot * D * (Hq + 2 * Hkv);  // dQ, dK, dV accumulators
}

template <class E>
int launch_bwd_e(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  if (p.ps.tile == 128)
    return p.D == 128 ? launch_cfg<BwdCfg<128, 128, 128, 1, E>>(p, b, stream)
                      : launch_cfg<BwdCfg<64, 128, 128, 1, E>>(p, b, stream);
  if ((p.Hq / p.Hkv) % 2 != 0) return SINKATTN_ERR_UNSUPPORTED;  // 64-token tiles pair heads
  return p.D == 128 ? launch_cfg<BwdCfg<128, 64, 64, 2, E>>(p, b, stream)
                    : launch_cfg<BwdCfg<64, 64, 64, 2, E>>(p, b, stream);
}

int launch_bwd_tc(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream) {
  return p.dt == SINKATTN_FP16 ? launch_bwd_e<ElemF16>(p, b, stream)
                               : launch_bwd_e<ElemBf16>(p, b, stream);
}

}  // namespace sk
