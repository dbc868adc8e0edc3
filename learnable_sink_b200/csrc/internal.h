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
int launch_fwd_simt(const AttnProblem& p, void* out, float* lse, float* sink_s,
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
  float* dsink_part;    // [n_part_blocks, Hq] workspace
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
  float* part;  // workspace: [B, Hq, splits, D + 2] floats
  int* counter; // workspace: work-item counter of the streaming kernel (zeroed per call)
  int* status;
};
int launch_decode(const DecodeProblem& p, cudaStream_t stream);

// failure-detection self-test: a bounded wait on a barrier nobody arrives at
int launch_wait_selftest(int* status, cudaStream_t stream);

}  // namespace sk
