/*
 * sinkattn.h -- C ABI of libsinkattn.so: grouped-query attention whose softmax
 * denominator carries a per-head learnable sink logit, for B200 (sm_100a).
 *
 * The operation (page "Attention Sink, Learnable Sink and dsink",
 * notes.kuangjux.top; section 1 for the scores and GQA head map, section 4
 * for the sink, sections 7-8 for the gradients):
 *
 *   x_ijh   = scale * <Q_ih, K_j,g(h)>,   g(h) = h / (Hq / Hkv)
 *   Z_ih    = sum_{j visible} e^{x_ijh},  L_orig = log Z
 *   L_new   = log(Z + e^{a_h})            (the sink logit a_h is NOT scaled)
 *   sink_s  = Z / (Z + e^{a_h}) = sigma(L_orig - a_h)   (mass on real tokens)
 *   O_ih    = sink_s * sum_j (e^{x_ijh} / Z) V_j,g(h)   (= O_orig scaled by s)
 *   dsink_h = -sum_i Delta_ih * p_sink_ih,  Delta_ih = <dO_ih, O_ih>,
 *             p_sink = e^{a_h - L_new}    (section 7 boxed result; section 10
 *             recommends exp(a - LSE_total) over 1 - sink_s)
 *   dQ/dK/dV: the usual softmax gradients with P = e^{x - L_new} and Delta
 *             computed from the sink-scaled O (section 8).
 *
 * learnable_sink == NULL disables the sink (page 1 section 4: "None"); a sink
 * of 0 still adds e^0 = 1 to the denominator.
 *
 * Visible set (page 1 section 2: block selection, window, causality and
 * sample boundaries all restrict it).  With sequence-local positions qi, kj
 * of the same packed sequence:
 *   causal                 => kj <= qi
 *   window > 0             => kj < n_sink  or  qi - kj < window   (StreamingLLM
 *                             KV set: initial sink tokens plus a recent window)
 *   block_indices != NULL  => kj / block_k is listed for (KV head g(h),
 *                             query block qi / block_q).
 *
 * Layouts (token-major, packed varlen; page 1 sections 1 and 7: out [T, Hq, D],
 * delta [T, Hq], dsink [Hq]):
 *   Q, O, dQ, dO : [T_tot, Hq, D]     K, V, dK, dV : [T_tot, Hkv, D]
 *   LSE_new, sink_s : [T_tot, Hq] float32     learnable_sink, dsink : [Hq] float32
 *   All tensors contiguous, row-major as written.
 *
 * Conventions for every entry point:
 *   - Every pointer is DEVICE memory owned by the caller (except the
 *     sinkattn_mask struct itself, which is read on the host during the call).
 *     The library never allocates device memory; scratch comes from the
 *     caller's workspace, sized by the *_bytes queries.
 *   - Work is enqueued asynchronously on `stream`; a return of SINKATTN_OK
 *     means arguments were valid and kernels were launched.  Errors detected
 *     on the device (a bounded wait that ran out, an out-of-range block index)
 *     are recorded in a per-device status word read by sinkattn_get_status().
 *   - Arguments are validated on the host first; on any invalid argument
 *     nothing is launched and SINKATTN_ERR_INVALID_ARG is returned.
 *   - Device pointers must be 16-byte aligned.
 *   - Nothing is written to the inputs (q, k, v, learnable_sink, masks).
 */
#ifndef SINKATTN_H_
#define SINKATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *sinkattn_stream_t;

/* Return codes. */
#define SINKATTN_OK 0
#define SINKATTN_ERR_INVALID_ARG 1 /* bad pointer, shape, alignment or mask   */
#define SINKATTN_ERR_UNSUPPORTED 2 /* device is not sm_100, or dtype/D combo  */
#define SINKATTN_ERR_CUDA 3        /* a CUDA runtime/driver call failed        */
#define SINKATTN_ERR_WORKSPACE 4   /* workspace/plan buffer too small          */
#define SINKATTN_ERR_TIMEOUT 5     /* device: a bounded barrier wait ran out   */
#define SINKATTN_ERR_BOUNDS 6      /* device: block index out of range         */
#define SINKATTN_ERR_PLAN 7        /* plan built for a different problem       */

/* Element type of Q/K/V/O/dO/dQ/dK/dV.  LSE, sink_s, sinks and dsink are
 * always float32 (page 1 section 9: sink_s is kept in FP32). */
typedef enum {
    SINKATTN_BF16 = 0, /* tensor-core path (tcgen05), fp32 accumulation   */
    SINKATTN_FP16 = 1, /* the same path with f16 operands (kind::f16)     */
    SINKATTN_FP32 = 2  /* fp32: 3xTF32 tensor-core forward, CUDA-core rest */
} sinkattn_dtype;

/* Mask descriptor (read on the host during the call; the arrays it points to
 * are device memory).
 *   causal        1: key kj visible only if kj <= qi (sequence-local).
 *   n_sink        with window > 0: keys [0, n_sink) of each sequence stay
 *                 visible (StreamingLLM keeps 4).
 *   window        > 0: also visible if qi - kj < window (requires causal);
 *                 0: no window restriction.
 *   cu_seqlens    device int32 [n_seq + 1], cu_seqlens[0] = 0,
 *                 cu_seqlens[n_seq] = T_tot, non-decreasing.  Sequences never
 *                 attend across their boundary.  Required.
 *   n_seq         number of packed sequences (>= 1).
 *   max_seqlen    an upper bound on every sequence length (used for sizing).
 *   block_indices NULL, or device int32 [Hkv, n_qblk, max_blocks]: for each
 *                 KV head and each sequence-local query block (numbered
 *                 globally in sequence order: sum over sequences of
 *                 ceil(len / block_q) rows), the sequence-local key blocks it
 *                 may see; -1 entries are padding, duplicates are ignored.
 *                 The diagonal block is NOT added implicitly.  An index
 *                 >= ceil(len / block_k) or < -1 sets SINKATTN_ERR_BOUNDS in
 *                 the status word and is skipped.
 *   n_qblk        rows of block_indices per KV head (ignored when NULL).
 *   block_q, block_k  block sizes; with block_indices both must be equal and
 *                 64 or 128.  Ignored when block_indices is NULL.
 *   max_blocks    entries per row, 1..32 (ignored when NULL). */
typedef struct {
    int32_t causal;
    int32_t n_sink;
    int32_t window;
    const int32_t *cu_seqlens;
    int32_t n_seq;
    int32_t max_seqlen;
    const int32_t *block_indices;
    int32_t n_qblk;
    int32_t block_q;
    int32_t block_k;
    int32_t max_blocks;
} sinkattn_mask;

/* ---- tile schedule ("plan") ---------------------------------------------
 * The mask is turned into a tile schedule once and reused by forward and
 * backward (and by every layer that shares the mask).  For each query tile
 * and KV head it lists the key tiles holding at least one visible pair, each
 * flagged full (no element mask needed) or partial; for each key tile the
 * reverse list of query tiles (reverse CSR, used by the backward).  Fully
 * masked tiles are never visited.  Query tiles are 128 tokens (block_q with
 * block_indices), key tiles 128 keys (block_k with block_indices); tiles are
 * sequence-local (a tile never spans two sequences).
 *
 * sinkattn_plan_bytes returns the plan buffer size needed for this shape and
 * mask (an upper bound; depends on T_tot, Hkv, n_seq, max_seqlen and the
 * block sizes only, not on the contents of cu_seqlens/block_indices), or 0 if
 * the arguments are invalid.  sinkattn_plan fills `plan` (device memory,
 * 16-byte aligned, caller-owned) on `stream`; forward and backward calls
 * later in stream order may read it.  The plan stays valid as long as the
 * mask arrays' contents do not change. */
size_t sinkattn_plan_bytes(int T_tot, int Hq, int Hkv, const sinkattn_mask *mask);
int sinkattn_plan(int T_tot, int Hq, int Hkv, const sinkattn_mask *mask,
                  void *plan, size_t plan_bytes, sinkattn_stream_t stream);

/* ---- forward --------------------------------------------------------------
 * Computes O, LSE_new and sink_s (page 1 section 4; page 4 section 5's gate
 * G = sigma(LSE - sink) equals sink_s).
 *   dt        SINKATTN_BF16 or SINKATTN_FP16 (the tensor-core path; P and the
 *             outputs rounded to dt) or SINKATTN_FP32; D = 64 or 128.
 *   T_tot     total packed tokens (>= 1).   Hq % Hkv == 0.
 *   scale     softmax scale alpha (typically 1/sqrt(D)).
 *   q, k, v   inputs of type dt, layouts above.
 *   learnable_sink  float32 [Hq] or NULL.
 *   mask      the mask the plan was built from.
 *   plan      built by sinkattn_plan for the same T_tot/Hq/Hkv/mask.
 *   out       [T_tot, Hq, D] of type dt (written).
 *   lse_new   float32 [T_tot, Hq] (written; natural log, includes the sink;
 *             -inf for a row that sees no key and has no sink).
 *   sink_s    float32 [T_tot, Hq] or NULL (written if non-NULL; 0 for a row
 *             that sees no key).
 * A row that sees no key gets O = 0 (and LSE = a_h, sink_s = 0 with a sink). */
int sinkattn_fwd(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                 const void *q, const void *k, const void *v,
                 const float *learnable_sink, const sinkattn_mask *mask,
                 const void *plan, size_t plan_bytes,
                 void *out, float *lse_new, float *sink_s,
                 sinkattn_stream_t stream);

/* ---- forward with the raw LSE ------------------------------------------------
 * Same as sinkattn_fwd, plus lse_orig (float32 [T_tot, Hq], 16-byte aligned,
 * or NULL): the log-sum-exp over the visible keys alone, before the sink joins
 * the denominator -- page 1's L_orig (its source notes: the raw LSE is what
 * goes to a teacher), from which page 4's gate sigma(LSE - sink) is formed.
 * Rows with no visible key get -inf.  LSE_new = logaddexp(lse_orig, a_h) and
 * sink_s = exp(lse_orig - lse_new) hold up to rounding. */
int sinkattn_fwd_ex(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                    const void *q, const void *k, const void *v, const float *learnable_sink,
                    const sinkattn_mask *mask, const void *plan, size_t plan_bytes, void *out,
                    float *lse_new, float *sink_s, float *lse_orig, sinkattn_stream_t stream);

/* ---- backward -------------------------------------------------------------
 * Computes dQ, dK, dV and dsink (page 1 sections 7-8).
 *   out, lse_new  the forward's O and LSE_new (sink-inclusive).
 *   dout          upstream gradient dL/dO, [T_tot, Hq, D] of type dt.
 *   learnable_sink  float32 [Hq] or NULL (then dsink is not written).
 *   dq, dk, dv    outputs of type dt (overwritten, not accumulated).
 *   dsink         float32 [Hq] (overwritten; summed over every query of every
 *                 sequence, no division by the token count, section 7).
 *   workspace     device scratch of at least sinkattn_bwd_workspace_bytes().
 * dK/dV sum over the Hq/Hkv query heads of each KV head.  dsink is computed
 * once per query (section 10's double-counting warning) in the Delta
 * preprocess and reduced deterministically. */
size_t sinkattn_bwd_workspace_bytes(sinkattn_dtype dt, int T_tot, int Hq, int Hkv,
                                    int D, const sinkattn_mask *mask);
int sinkattn_bwd(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                 const void *q, const void *k, const void *v, const void *out,
                 const void *dout, const float *lse_new,
                 const float *learnable_sink, const sinkattn_mask *mask,
                 const void *plan, size_t plan_bytes,
                 void *dq, void *dk, void *dv, float *dsink,
                 void *workspace, size_t workspace_bytes, sinkattn_stream_t stream);

/* ---- backward with an upstream gate gradient ---------------------------------
 * Same as sinkattn_bwd, plus d_sink_s: float32 [T_tot, Hq] (16-byte aligned)
 * or NULL, the upstream gradient dL/d sink_s of a loss that reads the gate
 * sink_s = sigma(L_orig - a_h) as well as O -- page "Attention Sink and the
 * native MoE in attention layers" (lvdousha26.github.io), section 5: the
 * sink-aware balance loss is a function of the gate, which is differentiable
 * through LSE and the sink.  With g = d_sink_s[t, h] and p_sink = 1 - sink_s
 * the Delta of every row becomes Delta - g * p_sink (the key-tile kernels are
 * otherwise unchanged) and the row's dsink term becomes
 * -p_sink * (Delta + g * sink_s).  Without a sink (learnable_sink == NULL)
 * sink_s is 1 on every row that sees a key and d_sink_s has no effect.
 * sinkattn_bwd(...) == sinkattn_bwd_ex(..., d_sink_s = NULL, ...). */
int sinkattn_bwd_ex(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                    const void *q, const void *k, const void *v, const void *out,
                    const void *dout, const float *lse_new, const float *d_sink_s,
                    const float *learnable_sink, const sinkattn_mask *mask,
                    const void *plan, size_t plan_bytes,
                    void *dq, void *dk, void *dv, float *dsink,
                    void *workspace, size_t workspace_bytes, sinkattn_stream_t stream);

/* ---- head importance ---------------------------------------------------------
 * Imp[h] = (1 / T_tot) * sum_t sink_s[t, h]: a head's mean gate over every
 * packed token (page "Attention Sink and the native MoE in attention layers",
 * section 4; the gate G = sigma(LSE - sink) is sink_s, section 5).  Rows that
 * see no key count with their gate 0.
 *   sink_s     float32 [T_tot, Hq] as written by the forward (T_tot >= 1,
 *              1 <= Hq <= 256; SINKATTN_ERR_UNSUPPORTED above that).
 *   imp        float32 [Hq] (written).
 *   workspace  device scratch of at least
 *              sinkattn_gate_importance_workspace_bytes(T_tot, Hq) bytes
 *              (0 is returned there for invalid sizes).
 * Partial sums are float64 in a partition fixed by (T_tot, Hq): bitwise
 * reproducible. */
size_t sinkattn_gate_importance_workspace_bytes(int T_tot, int Hq);
int sinkattn_gate_importance(int T_tot, int Hq, const float *sink_s, float *imp,
                             void *workspace, size_t workspace_bytes, sinkattn_stream_t stream);

/* ---- gate of a sink-free model ------------------------------------------------
 * For a model without a learnable sink whose attention sink is the first
 * token k_0 of each sequence, page "Attention Sink and the native MoE in
 * attention layers" (section 5) forms the gate from the LSE the attention
 * forward returns: G = sigma(LSE_not0 - q.k_0 * scale), LSE_not0 the
 * log-sum-exp over the visible keys other than k_0.  With L the sink-free
 * LSE over all visible keys, G = 1 - exp(x_0 - L), x_0 = scale <q, k_0>.
 *   q, k      the forward's inputs (type dt, layouts above, D = 64 or 128).
 *   lse       float32 [T_tot, Hq]: lse_new of sinkattn_fwd run with
 *             learnable_sink = NULL, or lse_orig of sinkattn_fwd_ex, over the
 *             same mask.
 *   mask      the forward's mask (k_0 is visible to query qi unless a window
 *             without sink tokens has passed it, qi >= window with n_sink = 0,
 *             or the block lists leave out key block 0).
 *   gate      float32 [T_tot, Hq] (written): 1 for a row that does not see
 *             k_0, 0 for a row that sees no key (lse = -inf).
 * Reads Q once; no workspace. */
int sinkattn_gate_vanilla(sinkattn_dtype dt, int T_tot, int Hq, int Hkv, int D, float scale,
                          const void *q, const void *k, const float *lse,
                          const sinkattn_mask *mask, float *gate, sinkattn_stream_t stream);

/* ---- ring-buffer decode ---------------------------------------------------
 * One query token per sequence attends over a StreamingLLM KV cache: n_sink
 * fixed slots holding the first tokens plus a circular window of `window`
 * slots holding the most recent ones (page 3: a fixed sink segment plus a
 * sliding window; the oldest non-sink entry is overwritten).
 *   q              [B, Hq, D] of type dt.
 *   k_cache, v_cache  [B, S, Hkv, D], S = n_sink + window.  Token at absolute
 *                  position p lives in slot p if p < n_sink, else in slot
 *                  n_sink + (p - n_sink) % window.
 *   cache_seqlens  device int32 [B]: tokens ever appended to sequence b,
 *                  the current token included (>= 0).  Slots
 *                  [0, min(cache_seqlens[b], S)) hold valid tokens.
 *   learnable_sink float32 [Hq] or NULL.
 *   out [B, Hq, D] (type dt), lse_new / sink_s float32 [B, Hq] (sink_s may be
 *   NULL).
 *   num_splits     partial results per (sequence, KV head) that the
 *                  workspace holds; 0 picks sinkattn_decode_num_splits.  A
 *                  count above ceil(S / 16) or above 128 is lowered to it
 *                  (same result).  bf16 / f16: the streaming kernel gives every warp
 *                  an equal run of 16-row cache pieces and cuts no
 *                  (sequence, KV head) into more than num_splits runs (1 =
 *                  one warp per pair); fp32: num_splits equal key splits.
 *   workspace      at least sinkattn_decode_workspace_bytes(B, Hq, D,
 *                  num_splits) bytes, 16-byte aligned, any contents (every
 *                  partial the merge reads is written by the same call).
 * Launches two kernels: the streaming kernel, then the merge of the partials
 * with the sink (a programmatic dependent launch that waits on the streaming
 * kernel).  B * S must stay below 2^31.  After a call whose device status is
 * SINKATTN_ERR_TIMEOUT, out, lse_new and sink_s are undefined.
 * Since no positional encoding is applied inside, the result depends only on
 * which tokens are in the cache, not on where the ring head is. */
size_t sinkattn_decode_workspace_bytes(int B, int Hq, int D, int num_splits);
int sinkattn_decode_num_splits(int B, int Hq, int Hkv, int D, int n_sink, int window);
int sinkattn_decode(sinkattn_dtype dt, int B, int Hq, int Hkv, int D, float scale,
                    const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *cache_seqlens, int n_sink, int window,
                    const float *learnable_sink, void *out, float *lse_new,
                    float *sink_s, int num_splits, void *workspace,
                    size_t workspace_bytes, sinkattn_stream_t stream);

/* ---- ring-buffer decode over a mixed-precision cache -------------------------
 * Page "Attention Sink / StreamingLLM", on KV-cache quantisation: the first
 * tokens carry much of the attention weight, so they are kept in high
 * precision while the rest of the cache is stored low.  Here the n_sink sink
 * slots stay bf16 and the window slots are FP8 E4M3 codes (the OCP 8-bit
 * format: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, S.1111.111 = NaN), each worth code value x a per-KV-head scale.
 * Same computation and results as sinkattn_decode over the dequantised cache.
 *   q              bf16 [B, Hq, D] (its elements must lie within the f16
 *                  range: the window scores run on f16 tensor-core MMAs).
 *   k_sink, v_sink bf16 [B, n_sink, Hkv, D]: slot s < n_sink of sequence b
 *                  (may be NULL when n_sink = 0).
 *   k_win, v_win   uint8 E4M3 codes [B, window, Hkv, D]: slot n_sink + j of
 *                  sequence b is window row j (may be NULL when window = 0).
 *   k_scale, v_scale  float32 [Hkv]: value = code value x scale of the row's
 *                  KV head.
 *   cache_seqlens, n_sink, window, learnable_sink, out (bf16), lse_new,
 *   sink_s: as for sinkattn_decode (the same slot rule).
 *   num_splits     partial results per (sequence, KV head) that the
 *                  workspace holds; 0 picks sinkattn_decode_fp8_num_splits.
 *                  A count above the pieces of one (sequence, KV head)
 *                  (ceil(n_sink / 16) + ceil(window / 32)) or above 128 is
 *                  lowered to it (same result).
 *   workspace      at least sinkattn_decode_workspace_bytes(B, Hq, D,
 *                  num_splits) bytes, any contents.
 * D in {64, 128}, Hq / Hkv in {1, 2, 4, 8}, 16-byte aligned pointers, B and
 * Hkv <= 65535, B * n_sink and B * window below 2^31 (else
 * SINKATTN_ERR_INVALID_ARG / UNSUPPORTED); launch failures return
 * SINKATTN_ERR_CUDA.  Launches the streaming kernel and the split merge. */
int sinkattn_decode_fp8_num_splits(int B, int Hq, int Hkv, int D, int n_sink, int window);
int sinkattn_decode_fp8(int B, int Hq, int Hkv, int D, float scale, const void *q,
                        const void *k_sink, const void *v_sink, const void *k_win,
                        const void *v_win, const float *k_scale, const float *v_scale,
                        const int32_t *cache_seqlens, int n_sink, int window,
                        const float *learnable_sink, void *out, float *lse_new, float *sink_s,
                        int num_splits, void *workspace, size_t workspace_bytes,
                        sinkattn_stream_t stream);

/* sinkattn_cache_append_fp8 -- one new token per sequence into the
 * mixed-precision cache of sinkattn_decode_fp8 (same slot rule as
 * sinkattn_cache_append).
 *   k_new, v_new   bf16 [B, Hkv, D]: the token being appended.
 *   cache_seqlens  device int32 [B], this token included (position
 *                  cache_seqlens[b] - 1; entries <= 0 write nothing).
 *   A position p < n_sink copies the token into k_sink / v_sink row p; a
 *   later one writes window row (p - n_sink) % window of k_win / v_win as
 *   the E4M3 codes of value / scale of the row's KV head (IEEE division in
 *   float32, round to nearest even, magnitudes past 448 saturated to 448,
 *   NaN stays NaN).
 * D in {64, 128}, 16-byte aligned k_new, v_new and caches (else
 * SINKATTN_ERR_INVALID_ARG); launch failures return SINKATTN_ERR_CUDA. */
int sinkattn_cache_append_fp8(int B, int Hkv, int D, int n_sink, int window, const void *k_new,
                              const void *v_new, const int32_t *cache_seqlens, void *k_sink,
                              void *v_sink, void *k_win, void *v_win, const float *k_scale,
                              const float *v_scale, sinkattn_stream_t stream);

/* ---- ring-cache maintenance -------------------------------------------------
 * Page "Attention Sink / StreamingLLM" (the core-idea section): the cache
 * keeps a sequence's first n_sink tokens in fixed slots and its most recent
 * `window` tokens in a circular segment, each new token overwriting the oldest
 * non-sink one.  Slot rule, the same as sinkattn_decode's: position
 * p < n_sink -> slot p, otherwise n_sink + (p - n_sink) % window.  Caches are
 * [B, S, Hkv, D] of type dt, S = n_sink + window, updated in place.
 *
 * sinkattn_cache_append -- one new token per sequence.
 *   k_new, v_new   [B, Hkv, D] of type dt: the token being appended.
 *   cache_seqlens  device int32 [B]: tokens ever appended, this one included
 *                  (the caller increments it first, as for decode), so the
 *                  token sits at position cache_seqlens[b] - 1; entries <= 0,
 *                  and positions past the sink segment when window = 0, write
 *                  nothing.
 * sinkattn_cache_fill -- a prefill's tokens into caches, one per sequence.
 *   cu_seqlens     device int32 [n_seq + 1]: sequence s is tokens
 *                  [cu_seqlens[s], cu_seqlens[s + 1]) of the packed
 *                  k, v [T_tot, Hkv, D] (type dt).
 *   Every token that survives in the ring -- one of the first n_sink, or one
 *   of the last `window` past them -- is written to its slot of sequence s;
 *   the other slots are left as they are.
 *   cache_seqlens_out  device int32 [n_seq] or NULL: receives each length.
 * Both: D in {64, 128}, dt BF16, FP16 or FP32, 16-byte aligned pointers (else
 * SINKATTN_ERR_INVALID_ARG); launch failures return SINKATTN_ERR_CUDA. */
int sinkattn_cache_append(sinkattn_dtype dt, int B, int Hkv, int D, int n_sink, int window,
                          const void *k_new, const void *v_new, const int32_t *cache_seqlens,
                          void *k_cache, void *v_cache, sinkattn_stream_t stream);
int sinkattn_cache_fill(sinkattn_dtype dt, int n_seq, int T_tot, int Hkv, int D, int n_sink,
                        int window, const int32_t *cu_seqlens, const void *k, const void *v,
                        void *k_cache, void *v_cache, int32_t *cache_seqlens_out,
                        sinkattn_stream_t stream);

/* ---- ring-buffer decode without caller scratch ------------------------------
 * No counterpart on the pages: this is a service for callers of this library.
 * Same computation, arguments and results as sinkattn_decode, minus the
 * workspace.  It is for callers that cannot hand out scratch memory -- e.g. a
 * serving loop that reserves all device memory before requests arrive and may
 * not allocate while they are in flight (cudaMalloc can block on the device and
 * can fail under memory pressure), or a plain C program that owns only its
 * input and output buffers.  The per-split partials go to a fixed 4 MiB array
 * in the library's device image (every GPU that loads the library keeps it
 * until the process exits); nothing is allocated.
 *   - Limit: B * Hq * num_splits * (D + 2) * 4 bytes (rounded up to 256)
 *     must fit in 4 MiB, num_splits counted after the same lowering
 *     sinkattn_decode applies (to ceil(S / 16) and 128).  With num_splits = 0
 *     the automatic count is lowered until it fits; a problem that does not
 *     fit even with one split, or an explicit num_splits that does not fit,
 *     returns SINKATTN_ERR_WORKSPACE and launches nothing.
 *   - The first call on each device looks up the array's device address
 *     (with that device current); make that first call before any stream
 *     capture.
 *   - Every call shares the one array and leaves its contents behind; each
 *     call writes every partial it reads, so nothing needs clearing, but calls
 *     that overlap on the GPU (different streams, or concurrent host threads)
 *     race on the array and must be serialised by the caller.
 *   - After a call whose device status is SINKATTN_ERR_TIMEOUT, some partials
 *     were not written (the merge then read an earlier call's leftovers):
 *     out, lse_new and sink_s are undefined. */
int sinkattn_decode_noalloc(sinkattn_dtype dt, int B, int Hq, int Hkv, int D, float scale,
                            const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *cache_seqlens, int n_sink, int window,
                            const float *learnable_sink, void *out, float *lse_new,
                            float *sink_s, int num_splits, sinkattn_stream_t stream);

/* ---- profiling hook ---------------------------------------------------------
 * Records CUDA events around the main kernel of later calls, on the stream
 * that kernel is launched on, so a caller can time that kernel alone (the
 * other launches of the call stay outside the events).
 *   which   SINKATTN_KERNEL_FWD (the attention forward kernel),
 *           SINKATTN_KERNEL_BWD (the dK/dV/dQ kernel of sinkattn_bwd),
 *           SINKATTN_KERNEL_DECODE (the split-KV streaming kernel),
 *           SINKATTN_KERNEL_GATE (the kernel of sinkattn_gate_vanilla).
 *   start, stop  cudaEvent_t handles created by the caller, or both NULL to
 *           stop recording.  They are recorded by every later call of that
 *           kind on the calling host thread's current device until changed.
 * Returns SINKATTN_ERR_INVALID_ARG for an unknown `which`. */
#define SINKATTN_KERNEL_FWD 0
#define SINKATTN_KERNEL_BWD 1
#define SINKATTN_KERNEL_DECODE 2
#define SINKATTN_KERNEL_GATE 3
int sinkattn_set_kernel_events(int which, void *start, void *stop);

/* ---- failure-detection self-test ---------------------------------------------
 * Launches a one-warp kernel that waits, through the same bounded barrier wait
 * every kernel of this library uses, on a barrier nothing ever arrives at.  The
 * wait gives up after its budget (about one second), records
 * SINKATTN_ERR_TIMEOUT in the status word and the kernel returns normally, so
 * the CUDA context stays usable.  Read the outcome with sinkattn_get_status. */
int sinkattn_selftest_timeout(sinkattn_stream_t stream);

/* ---- status ---------------------------------------------------------------
 * sinkattn_get_status synchronises `stream`, then returns the first error code
 * any kernel of this library recorded on the current device since the last
 * sinkattn_clear_status (SINKATTN_OK if none), or SINKATTN_ERR_CUDA if the
 * synchronisation itself failed. */
int sinkattn_get_status(sinkattn_stream_t stream);
int sinkattn_clear_status(sinkattn_stream_t stream);
const char *sinkattn_error_string(int code);
int sinkattn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SINKATTN_H_ */
