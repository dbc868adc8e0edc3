// Host-side launcher declarations shared by the translation units of
// libsinkattn.so.  Not part of the public ABI (see include/sinkattn.h).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sinkattn.h"
#include "common.cuh"
#include "plan.cuh"

namespace sk {

// Events recorded around a main kernel (profiling hook; both null = off).
struct KernelEvents {
  cudaEvent_t start = nullptr, stop = nullptr;
};
KernelEvents kernel_events(int which);
inline void record_start(int which, cudaStream_t s) {
  const KernelEvents e = kernel_events(which);
  if (e.start) cudaEventRecord(e.start, s);
}
inline void record_stop(int which, cudaStream_t s) {
  const KernelEvents e = kernel_events(which);
  if (e.stop) cudaEventRecord(e.stop, s);
}

struct PlanLaunch {
  void* plan;
  PlanSizes sizes;
  const int32_t* cu_seqlens;
  const int32_t* block_indices;
  int* status;
  int T_tot, Hkv, n_seq, causal, n_sink, window, n_qblk, max_blocks, fingerprint;
};
int launch_plan(const PlanLaunch& L, cudaStream_t stream);

// Problem description handed to the attention launchers.
struct AttnProblem {
  int dt;  // sinkattn_dtype
  int T_tot, Hq, Hkv, D;
  float scale;
  const void* q;
  const void* k;
  const void* v;
  const float* sink;  // [Hq] or nullptr
  int causal, n_sink, window;
  const int* plan;    // device plan words
  PlanSizes ps;
  int* status;
  float* lse_orig;    // forward: [T_tot, Hq] LSE over the visible keys only, or nullptr
};

bool make_tmap_3d(CUtensorMap* map, const void* base, int T, int H, int D, int box_h, int box_t);
bool make_tmap_3d_f32(CUtensorMap* map, const void* base, int T, int H, int D, int box_h,
                      int box_t);
bool make_tmap_3d_plain(CUtensorMap* map, const void* base, int T, int H, int D, int box_h,
                        int box_t);

// forward
// fp32 inputs: 3xTF32 tensor-core forward
int launch_fwd_tf32(const AttnProblem& p, void* out, float* lse, float* sink_s,
                    cudaStream_t stream);
int launch_fwd_tc(const AttnProblem& p, void* out, float* lse, float* sink_s,
                  cudaStream_t stream);

// backward pieces
struct BwdBuffers {
  const void* out;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dsink;
  const float* dss;     // [T_tot, Hq] upstream dL/d sink_s, or nullptr
  float* delta;         // [Hq, T_tot] workspace (head-major)
  float* lse2;          // [Hq, T_tot] workspace: LSE_new * log2(e), -inf -> +inf
  float* dsink_part;    // [Hq, n_part_blocks] workspace
  float* dq_accum;      // [T_tot, Hq, D] fp32 workspace (tensor path)
  float* dk_accum;      // [T_tot, Hkv, D] fp32 workspace: split key tiles only
  float* dv_accum;      // [T_tot, Hkv, D] fp32 workspace: split key tiles only
  int n_part_blocks;
};
int preprocess_blocks(int T_tot);
int launch_bwd_preprocess(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream);
int launch_bwd_simt(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream);
int launch_bwd_tc(const AttnProblem& p, const BwdBuffers& b, cudaStream_t stream);
size_t bwd_tc_workspace_bytes(int T_tot, int Hq, int Hkv, int D);

// gate of a sink-free model (sink = first token of each sequence)
struct GateVanillaArgs {
  const void* q;
  const void* k;
  const float* lse;
  float* gate;
  const int32_t* cu;
  const int32_t* bi;
  int n_seq, Hq, Hkv, n_sink, window, n_qblk, block_q, max_blocks;
  float scale;
};
int launch_gate_vanilla(const GateVanillaArgs& a, int dt, int D, int max_seqlen,
                        cudaStream_t stream);

// decode
struct DecodeProblem {
  int dt, B, Hq, Hkv, D, n_sink, window, num_splits;
  float scale;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* cache_seqlens;
  const float* sink;
  void* out;
  float* lse;
  float* sink_s;
  float* part;  // workspace: [B, Hq, num_splits, D + 2] floats
  int* status;
};
int launch_decode(const DecodeProblem& p, cudaStream_t stream);

// Decode over the mixed-precision ring cache: bf16 sink slots, FP8 E4M3
// window slots with per-KV-head scales.  `base.k_cache/v_cache` are unused.
struct DecodeFp8Problem {
  DecodeProblem base;
  const void* k_sink;    // bf16 [B, n_sink, Hkv, D]
  const void* v_sink;
  const void* k_win;     // uint8 E4M3 codes [B, window, Hkv, D]
  const void* v_win;
  const float* k_scale;  // [Hkv]
  const float* v_scale;  // [Hkv]
};
int launch_decode_fp8(const DecodeFp8Problem& p, cudaStream_t stream);
// Units (pieces) per (sequence, KV head) of the mixed-precision cache: sink
// slots in pieces of 16 rows, window slots in pieces of 32.
inline long long fp8_pieces(long long n_sink, long long window) {
  return (n_sink + 15) / 16 + (window + 31) / 32;
}

// The split merge handles up to this many partial results per (sequence,
// query head).
constexpr int kMaxDecodeSplits = 128;
// Cache rows per piece of the streaming decode.
constexpr int kDecodeRows = 16;

// Static schedule of the bf16 streaming decode.  Every (sequence, KV head)
// pair owns np_max pieces of kDecodeRows cache rows; the pairs' pieces are
// laid end to end and warp w streams pieces [w ppw, (w + 1) ppw).  ppw is the
// smallest run that (a) needs no more warps than max_warps and (b) cuts no
// pair into more than num_splits runs (a run of L pieces meets at most
// ceil((L - 1) / ppw) + 1 runs; num_splits = 1 aligns runs to whole pairs).
// A split count beyond the pieces of one pair, or beyond what the merge
// handles, gives the same result with fewer slots.
inline int decode_clamp_units(int num_splits, long long np) {
  long long n = num_splits;
  if (n > np) n = np;
  if (n > kMaxDecodeSplits) n = kMaxDecodeSplits;
  if (n < 1) n = 1;
  return (int)n;
}
inline int decode_clamp_splits(int num_splits, int n_sink, int window) {
  return decode_clamp_units(num_splits, ((long long)n_sink + window + kDecodeRows - 1) / kDecodeRows);
}

struct DecSchedule {
  long long np_max, ppw, n_warps;
};
inline DecSchedule decode_schedule_units(long long B, long long Hkv, long long np_max,
                                         int num_splits, long long max_warps) {
  DecSchedule d{};
  d.np_max = np_max;
  const long long pairs = B * Hkv, total = pairs * d.np_max;
  if (max_warps < 1) max_warps = 1;
  if (num_splits <= 1) {
    d.ppw = d.np_max * ((pairs + max_warps - 1) / max_warps);
  } else {
    d.ppw = (total + max_warps - 1) / max_warps;
    const long long need = (d.np_max - 1 + num_splits - 2) / (num_splits - 1);
    if (need > d.ppw) d.ppw = need;
  }
  if (d.ppw < 1) d.ppw = 1;
  d.n_warps = (total + d.ppw - 1) / d.ppw;
  return d;
}
inline DecSchedule decode_schedule(long long B, long long Hkv, long long S, int num_splits,
                                   long long max_warps) {
  return decode_schedule_units(B, Hkv, (S + kDecodeRows - 1) / kDecodeRows, num_splits,
                               max_warps);
}
// The fewest partial slots per pair that still let max_warps warps take
// equal runs (at most np_max and kMaxDecodeSplits).
inline int decode_auto_splits(long long B, long long Hkv, long long np_max, long long max_warps) {
  if (B < 1 || Hkv < 1 || np_max < 1) return 1;
  const DecSchedule d = decode_schedule_units(B, Hkv, np_max, kMaxDecodeSplits, max_warps);
  long long want = (d.np_max - 1 + d.ppw - 1) / d.ppw + 1;
  if (want > d.np_max) want = d.np_max;
  if (want > kMaxDecodeSplits) want = kMaxDecodeSplits;
  if (want < 1) want = 1;
  return (int)want;
}

// failure-detection self-test: a bounded wait on a barrier nobody arrives at
int launch_wait_selftest(int* status, cudaStream_t stream);

}  // namespace sk
