// C ABI of libsinkattn.so (declared in include/sinkattn.h): argument
// validation on the host, workspace layout, and dispatch to the kernels.
#include <climits>
#include <mutex>

#include "internal.h"

// First error any kernel of this library recorded on this device.
__device__ int g_sinkattn_status;

namespace sk {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};
int g_is_sm100[kMaxDevices] = {};  // 0 unknown, 1 yes, -1 no

bool current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return false;
  return *dev >= 0 && *dev < kMaxDevices;
}

// Device address of the status word (host code cannot use the symbol itself).
int* status_word() {
  int dev;
  if (!current_device(&dev)) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sinkattn_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool device_is_sm100() {
  int dev;
  if (!current_device(&dev)) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_is_sm100[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    g_is_sm100[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_is_sm100[dev] == 1;
}

thread_local KernelEvents g_events[4];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool mask_ok(int T_tot, int Hq, int Hkv, const sinkattn_mask* m) {
  if (!m || T_tot < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return false;
  if (!m->cu_seqlens || !aligned16(m->cu_seqlens)) return false;
  if (m->n_seq < 1 || m->n_seq > T_tot || m->max_seqlen < 1) return false;
  if (m->causal != 0 && m->causal != 1) return false;
  if (m->window < 0 || m->n_sink < 0) return false;
  if (m->window > 0 && !m->causal) return false;
  if (m->block_indices) {
    if (!aligned16(m->block_indices)) return false;
    if (m->block_q != m->block_k) return false;
    if (m->block_q != 64 && m->block_q != 128) return false;
    if (m->max_blocks < 1 || m->max_blocks > 32 || m->n_qblk < 1) return false;
  }
  return true;
}

int fingerprint(int T_tot, int Hq, int Hkv, const sinkattn_mask* m) {
  uint32_t h = 2166136261u;
  auto mix = [&](uint64_t v) {
    for (int i = 0; i < 8; ++i) { h ^= uint32_t(v & 0xff); h *= 16777619u; v >>= 8; }
  };
  mix(T_tot); mix(Hkv); mix(m->causal); mix(m->n_sink); mix(m->window); mix(m->n_seq);
  mix(m->max_seqlen); mix(reinterpret_cast<uintptr_t>(m->cu_seqlens));
  mix(reinterpret_cast<uintptr_t>(m->block_indices));
  if (m->block_indices) { mix(m->n_qblk); mix(m->block_q); mix(m->max_blocks); }
  (void)Hq;
  return int(h & 0x7fffffff);
}

bool sizes_for(int T_tot, int Hkv, const sinkattn_mask* m, PlanSizes* out) {
  const bool sparse = m->block_indices != nullptr;
  const long long cap_tiles = (long long)T_tot / (sparse ? m->block_q : 128) + m->n_seq;
  const long long max_kt = ((long long)m->max_seqlen + 63) / 64;
  const long long items = cap_tiles * (sparse ? Hkv : 1);
  const long long per = sparse ? m->max_blocks : max_kt;
  if (items * per > INT_MAX / 2 || items * 8 > INT_MAX / 4) return false;
  *out = plan_sizes(T_tot, Hkv, m->n_seq, m->max_seqlen, sparse, m->block_q, m->max_blocks);
  return (long long)out->total_words < INT_MAX / 2;
}

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct BwdLayout {
  size_t delta, lse2, part, dq_accum, total;
};
BwdLayout bwd_layout(int dt, int T_tot, int Hq, int Hkv, int D) {
  BwdLayout L{};
  size_t off = 0;
  L.delta = off; off += round_up(sizeof(float) * (size_t)T_tot * Hq);
  L.lse2 = off; off += round_up(sizeof(float) * (size_t)T_tot * Hq);
  L.part = off; off += round_up(sizeof(float) * (size_t)preprocess_blocks(T_tot) * Hq);
  L.dq_accum = off;
  if (dt != SINKATTN_FP32) off += round_up(bwd_tc_workspace_bytes(T_tot, Hq, Hkv, D));
  L.total = off;
  return L;
}

}  // namespace

KernelEvents kernel_events(int which) {
  return (which >= 0 && which < 4) ? g_events[which] : KernelEvents{};
}

}  // namespace sk

using namespace sk;

extern "C" {

size_t sinkattn_plan_bytes(int T_tot, int Hq, int Hkv, const sinkattn_mask* mask) {
  if (!mask_ok(T_tot, Hq, Hkv, mask)) return 0;
  PlanSizes z;
  if (!sizes_for(T_tot, Hkv, mask, &z)) return 0;
  return (size_t)z.total_words * 4;
}

int sinkattn_plan(int T_tot, int Hq, int Hkv, const sinkattn_mask* mask, void* plan,
                  size_t plan_bytes, sinkattn_stream_t stream) {
  if (!mask_ok(T_tot, Hq, Hkv, mask) || !plan || !aligned16(plan)) return SINKATTN_ERR_INVALID_ARG;
  if (!device_is_sm100()) return SINKATTN_ERR_UNSUPPORTED;
  PlanSizes z;
  if (!sizes_for(T_tot, Hkv, mask, &z)) return SINKATTN_ERR_INVALID_ARG;
  if (plan_bytes < (size_t)z.total_words * 4) return SINKATTN_ERR_WORKSPACE;
  PlanLaunch L{};
  L.plan = plan;
  L.sizes = z;
  L.cu_seqlens = mask->cu_seqlens;
  L.block_indices = mask->block_indices;
  L.status = status_word();
  L.T_tot = T_tot;
  L.Hkv = Hkv;
  L.n_seq = mask->n_seq;
  L.causal = mask->causal;
  L.n_sink = mask->n_sink;
  L.window = mask->window;
  L.n_qblk = mask->block_indices ? mask->n_qblk : 0;
  L.max_blocks = mask->block_indices ? mask->max_blocks : 0;
  L.fingerprint = fingerprint(T_tot, Hq, Hkv, mask);
  if (!L.status) return SINKATTN_ERR_CUDA;
  return launch_plan(L, reinterpret_cast<cudaStream_t>(stream));
}

static int attn_common(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D,
                       const void* q, const void* k, const void* v, const float* sink,
                       const sinkattn_mask* mask, const void* plan, size_t plan_bytes,
                       AttnProblem* p) {
  if (dt != SINKATTN_BF16 && dt != SINKATTN_FP16 && dt != SINKATTN_FP32) return SINKATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SINKATTN_ERR_INVALID_ARG;
  if (!mask_ok(T_tot, Hq, Hkv, mask)) return SINKATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !plan) return SINKATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(plan) ||
      (sink && !aligned16(sink)))
    return SINKATTN_ERR_INVALID_ARG;
  PlanSizes z;
  if (!sizes_for(T_tot, Hkv, mask, &z)) return SINKATTN_ERR_INVALID_ARG;
  if (plan_bytes < (size_t)z.total_words * 4) return SINKATTN_ERR_WORKSPACE;
  if (!device_is_sm100()) return SINKATTN_ERR_UNSUPPORTED;
  p->dt = dt;
  p->T_tot = T_tot;
  p->Hq = Hq;
  p->Hkv = Hkv;
  p->D = D;
  p->q = q;
  p->k = k;
  p->v = v;
  p->sink = sink;
  p->causal = mask->causal;
  p->n_sink = mask->n_sink;
  p->window = mask->window;
  p->plan = static_cast<const int*>(plan);
  p->ps = z;
  p->status = status_word();
  return p->status ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

int sinkattn_fwd(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                 const void* q, const void* k, const void* v, const float* learnable_sink,
                 const sinkattn_mask* mask, const void* plan, size_t plan_bytes, void* out,
                 float* lse_new, float* sink_s, sinkattn_stream_t stream) {
  return sinkattn_fwd_ex(dt, T_tot, Hq, Hkv, D, scale, q, k, v, learnable_sink, mask, plan,
                         plan_bytes, out, lse_new, sink_s, nullptr, stream);
}

int sinkattn_fwd_ex(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                    const void* q, const void* k, const void* v, const float* learnable_sink,
                    const sinkattn_mask* mask, const void* plan, size_t plan_bytes, void* out,
                    float* lse_new, float* sink_s, float* lse_orig, sinkattn_stream_t stream) {
  AttnProblem p{};
  int rc = attn_common(dt, T_tot, Hq, Hkv, D, q, k, v, learnable_sink, mask, plan, plan_bytes, &p);
  if (rc != SINKATTN_OK) return rc;
  if (!out || !lse_new || !aligned16(out) || !aligned16(lse_new) || (sink_s && !aligned16(sink_s)) ||
      (lse_orig && !aligned16(lse_orig)))
    return SINKATTN_ERR_INVALID_ARG;
  p.scale = scale;
  p.lse_orig = lse_orig;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dt == SINKATTN_FP32) return launch_fwd_tf32(p, out, lse_new, sink_s, s);
  return launch_fwd_tc(p, out, lse_new, sink_s, s);
}

size_t sinkattn_bwd_workspace_bytes(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D,
                                    const sinkattn_mask* mask) {
  if (!mask_ok(T_tot, Hq, Hkv, mask) || (D != 64 && D != 128)) return 0;
  if (dt != SINKATTN_BF16 && dt != SINKATTN_FP16 && dt != SINKATTN_FP32) return 0;
  return bwd_layout(dt, T_tot, Hq, Hkv, D).total;
}

int sinkattn_bwd(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                 const void* q, const void* k, const void* v, const void* out, const void* dout,
                 const float* lse_new, const float* learnable_sink, const sinkattn_mask* mask,
                 const void* plan, size_t plan_bytes, void* dq, void* dk, void* dv, float* dsink,
                 void* workspace, size_t workspace_bytes, sinkattn_stream_t stream) {
  return sinkattn_bwd_ex(dt, T_tot, Hq, Hkv, D, scale, q, k, v, out, dout, lse_new, nullptr,
                         learnable_sink, mask, plan, plan_bytes, dq, dk, dv, dsink, workspace,
                         workspace_bytes, stream);
}

int sinkattn_bwd_ex(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                    const void* q, const void* k, const void* v, const void* out,
                    const void* dout, const float* lse_new, const float* d_sink_s,
                    const float* learnable_sink, const sinkattn_mask* mask, const void* plan,
                    size_t plan_bytes, void* dq, void* dk, void* dv, float* dsink,
                    void* workspace, size_t workspace_bytes, sinkattn_stream_t stream) {
  AttnProblem p{};
  int rc = attn_common(dt, T_tot, Hq, Hkv, D, q, k, v, learnable_sink, mask, plan, plan_bytes, &p);
  if (rc != SINKATTN_OK) return rc;
  if (!out || !dout || !lse_new || !dq || !dk || !dv || !workspace) return SINKATTN_ERR_INVALID_ARG;
  if (learnable_sink && !dsink) return SINKATTN_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(lse_new) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) || (dsink && !aligned16(dsink)) ||
      (d_sink_s && !aligned16(d_sink_s)))
    return SINKATTN_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(dt, T_tot, Hq, Hkv, D);
  if (workspace_bytes < L.total) return SINKATTN_ERR_WORKSPACE;
  p.scale = scale;
  char* ws = static_cast<char*>(workspace);
  BwdBuffers b{};
  b.out = out;
  b.dout = dout;
  b.lse = lse_new;
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  b.dsink = learnable_sink ? dsink : nullptr;
  b.dss = d_sink_s;  // without a sink, sink_s is 1 on every row that sees a key: no gradient
  b.delta = reinterpret_cast<float*>(ws + L.delta);
  b.lse2 = reinterpret_cast<float*>(ws + L.lse2);
  b.dsink_part = reinterpret_cast<float*>(ws + L.part);
  b.dq_accum = reinterpret_cast<float*>(ws + L.dq_accum);
  b.dk_accum = b.dq_accum + (size_t)T_tot * Hq * D;
  b.dv_accum = b.dk_accum + (size_t)T_tot * Hkv * D;
  b.n_part_blocks = preprocess_blocks(T_tot);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = launch_bwd_preprocess(p, b, s);
  if (rc != SINKATTN_OK) return rc;
  if (dt == SINKATTN_FP32) return launch_bwd_simt(p, b, s);
  return launch_bwd_tc(p, b, s);
}

int sinkattn_gate_vanilla(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                          const void* q, const void* k, const float* lse,
                          const sinkattn_mask* mask, float* gate, sinkattn_stream_t stream) {
  if (dt != SINKATTN_BF16 && dt != SINKATTN_FP16 && dt != SINKATTN_FP32) return SINKATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SINKATTN_ERR_INVALID_ARG;
  if (!mask_ok(T_tot, Hq, Hkv, mask)) return SINKATTN_ERR_INVALID_ARG;
  if (!q || !k || !lse || !gate) return SINKATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(lse) || !aligned16(gate))
    return SINKATTN_ERR_INVALID_ARG;
  if (mask->n_seq > 65535) return SINKATTN_ERR_INVALID_ARG;
  if (!device_is_sm100()) return SINKATTN_ERR_UNSUPPORTED;
  GateVanillaArgs a{};
  a.q = q;
  a.k = k;
  a.lse = lse;
  a.gate = gate;
  a.cu = mask->cu_seqlens;
  a.bi = mask->block_indices;
  a.n_seq = mask->n_seq;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.n_sink = mask->n_sink;
  a.window = mask->window;
  a.n_qblk = mask->block_indices ? mask->n_qblk : 0;
  a.block_q = mask->block_q;
  a.max_blocks = mask->block_indices ? mask->max_blocks : 0;
  a.scale = scale;
  return launch_gate_vanilla(a, dt, D, mask->max_seqlen, reinterpret_cast<cudaStream_t>(stream));
}

namespace {
int sm_count() {
  int sms = 148, dev;
  if (current_device(&dev)) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}
}  // namespace

int sinkattn_decode_num_splits(int B, int Hq, int Hkv, int D, int n_sink, int window) {
  (void)Hq; (void)D;
  const long long S = (long long)n_sink + window;
  if (B < 1 || Hkv < 1 || S < 1) return 1;
  // the fewest partial slots per (sequence, KV head) that still let every
  // warp of the streaming kernel (8 per SM) take an equal run of pieces
  return decode_auto_splits(B, Hkv, (S + kDecodeRows - 1) / kDecodeRows, 8LL * sm_count());
}

size_t sinkattn_decode_workspace_bytes(int B, int Hq, int D, int num_splits) {
  if (B < 1 || Hq < 1 || num_splits < 1 || (D != 64 && D != 128)) return 0;
  // per-(sequence, query head) partial results: num_splits x (acc[D], m, l)
  return round_up(sizeof(float) * (size_t)B * Hq * num_splits * (D + 2));
}

int sinkattn_decode(sinkattn_dtype dt, int B, int Hq, int Hkv, int D, float scale,
                    const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* cache_seqlens, int n_sink, int window,
                    const float* learnable_sink, void* out, float* lse_new, float* sink_s,
                    int num_splits, void* workspace, size_t workspace_bytes,
                    sinkattn_stream_t stream) {
  if (dt != SINKATTN_BF16 && dt != SINKATTN_FP16 && dt != SINKATTN_FP32) return SINKATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (D != 64 && D != 128)) return SINKATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SINKATTN_ERR_UNSUPPORTED;
  if (n_sink < 0 || window < 0 || n_sink + window < 1) return SINKATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return SINKATTN_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !cache_seqlens || !out || !lse_new || !workspace)
    return SINKATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(lse_new) || !aligned16(workspace) || (sink_s && !aligned16(sink_s)) ||
      (learnable_sink && !aligned16(learnable_sink)))
    return SINKATTN_ERR_INVALID_ARG;
  if ((long long)B * (n_sink + (long long)window) > INT_MAX) return SINKATTN_ERR_INVALID_ARG;
  if (num_splits <= 0) num_splits = sinkattn_decode_num_splits(B, Hq, Hkv, D, n_sink, window);
  num_splits = decode_clamp_splits(num_splits, n_sink, window);  // same result, fewer slots
  if (workspace_bytes < sinkattn_decode_workspace_bytes(B, Hq, D, num_splits))
    return SINKATTN_ERR_WORKSPACE;
  if (!device_is_sm100()) return SINKATTN_ERR_UNSUPPORTED;
  DecodeProblem p{};
  p.dt = dt;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.n_sink = n_sink;
  p.window = window;
  p.num_splits = num_splits;
  p.scale = scale;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.cache_seqlens = cache_seqlens;
  p.sink = learnable_sink;
  p.out = out;
  p.lse = lse_new;
  p.sink_s = sink_s;
  p.part = static_cast<float*>(workspace);
  p.status = status_word();
  return launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
}

int sinkattn_decode_fp8_num_splits(int B, int Hq, int Hkv, int D, int n_sink, int window) {
  (void)Hq; (void)D;
  if (B < 1 || Hkv < 1 || n_sink < 0 || window < 0 || n_sink + (long long)window < 1) return 1;
  return decode_auto_splits(B, Hkv, fp8_pieces(n_sink, window), 8LL * sm_count());
}

int sinkattn_decode_fp8(int B, int Hq, int Hkv, int D, float scale, const void* q,
                        const void* k_sink, const void* v_sink, const void* k_win,
                        const void* v_win, const float* k_scale, const float* v_scale,
                        const int32_t* cache_seqlens, int n_sink, int window,
                        const float* learnable_sink, void* out, float* lse_new, float* sink_s,
                        int num_splits, void* workspace, size_t workspace_bytes,
                        sinkattn_stream_t stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (D != 64 && D != 128))
    return SINKATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SINKATTN_ERR_UNSUPPORTED;
  if (n_sink < 0 || window < 0 || n_sink + (long long)window < 1) return SINKATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return SINKATTN_ERR_INVALID_ARG;
  if ((long long)B * n_sink > INT_MAX || (long long)B * window > INT_MAX)
    return SINKATTN_ERR_INVALID_ARG;
  if (!q || !cache_seqlens || !out || !lse_new || !workspace) return SINKATTN_ERR_INVALID_ARG;
  if (n_sink > 0 && (!k_sink || !v_sink || !aligned16(k_sink) || !aligned16(v_sink)))
    return SINKATTN_ERR_INVALID_ARG;
  if (window > 0 && (!k_win || !v_win || !k_scale || !v_scale || !aligned16(k_win) ||
                     !aligned16(v_win) || !aligned16(k_scale) || !aligned16(v_scale)))
    return SINKATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(lse_new) || !aligned16(workspace) ||
      (sink_s && !aligned16(sink_s)) || (learnable_sink && !aligned16(learnable_sink)))
    return SINKATTN_ERR_INVALID_ARG;
  if (num_splits <= 0) num_splits = sinkattn_decode_fp8_num_splits(B, Hq, Hkv, D, n_sink, window);
  num_splits = decode_clamp_units(num_splits, fp8_pieces(n_sink, window));
  if (workspace_bytes < sinkattn_decode_workspace_bytes(B, Hq, D, num_splits))
    return SINKATTN_ERR_WORKSPACE;
  if (!device_is_sm100()) return SINKATTN_ERR_UNSUPPORTED;
  DecodeFp8Problem x{};
  DecodeProblem& p = x.base;
  p.dt = SINKATTN_BF16;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.n_sink = n_sink;
  p.window = window;
  p.num_splits = num_splits;
  p.scale = scale;
  p.q = q;
  p.cache_seqlens = cache_seqlens;
  p.sink = learnable_sink;
  p.out = out;
  p.lse = lse_new;
  p.sink_s = sink_s;
  p.part = static_cast<float*>(workspace);
  p.status = status_word();
  if (!p.status) return SINKATTN_ERR_CUDA;
  x.k_sink = k_sink;
  x.v_sink = v_sink;
  x.k_win = k_win;
  x.v_win = v_win;
  // the kernel loads a KV head's scales for every segment, even without
  // window slots (and then never uses them): keep the pointers valid
  x.k_scale = window > 0 ? k_scale : lse_new;
  x.v_scale = window > 0 ? v_scale : lse_new;
  return launch_decode_fp8(x, reinterpret_cast<cudaStream_t>(stream));
}

int sinkattn_set_kernel_events(int which, void* start, void* stop) {
  if (which < 0 || which > 3 || ((start == nullptr) != (stop == nullptr)))
    return SINKATTN_ERR_INVALID_ARG;
  g_events[which].start = static_cast<cudaEvent_t>(start);
  g_events[which].stop = static_cast<cudaEvent_t>(stop);
  return SINKATTN_OK;
}

int sinkattn_selftest_timeout(sinkattn_stream_t stream) {
  if (!device_is_sm100()) return SINKATTN_ERR_UNSUPPORTED;
  int* st = status_word();
  if (!st) return SINKATTN_ERR_CUDA;
  return launch_wait_selftest(st, reinterpret_cast<cudaStream_t>(stream));
}

int sinkattn_get_status(sinkattn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_sinkattn_status, sizeof(int)) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  return v;
}

int sinkattn_clear_status(sinkattn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_sinkattn_status, &zero, sizeof(int)) != cudaSuccess)
    return SINKATTN_ERR_CUDA;
  return SINKATTN_OK;
}

const char* sinkattn_error_string(int code) {
  switch (code) {
    case SINKATTN_OK: return "ok";
    case SINKATTN_ERR_INVALID_ARG: return "invalid argument";
    case SINKATTN_ERR_UNSUPPORTED: return "unsupported device, dtype or shape";
    case SINKATTN_ERR_CUDA: return "CUDA call failed";
    case SINKATTN_ERR_WORKSPACE: return "workspace or plan buffer too small";
    case SINKATTN_ERR_TIMEOUT: return "device barrier wait timed out";
    case SINKATTN_ERR_BOUNDS: return "index out of range (cu_seqlens or block_indices)";
    case SINKATTN_ERR_PLAN: return "plan does not match the problem";
    default: return "unknown error";
  }
}

int sinkattn_version(void) { return 100; }

}  // extern "C"
