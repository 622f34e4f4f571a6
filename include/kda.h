/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention prefill library (libkda.so).
 *
 * The operations:
 *
 *  kda_chunk_fwd
 *    The chunk-parallel KDA prefill ("max.nn.state_space.kda_chunk": the same recurrence as
 *    single-token decode, evaluated in parallel over fixed-size chunks, mutating the state
 *    pool).  For every sequence b, value head h and token t of that sequence:
 *        g_t  = -exp(a_log[h]) * softplus(raw_gate[t,h,:] + dt_bias[h,:])   (per key channel)
 *               ("safe" gate mode: g_t = max(g_t, gate_lower_bound))
 *        b_t  = sigmoid(beta_logits[t,h])   (or beta_logits[t,h] itself in probability mode)
 *        S    = Diag(exp(g_t)) S                          decay each key row
 *        S    = S + k_t (b_t (v_t - k_t^T S))^T           delta-rule write (predicts from the
 *                                                          decayed state; overwrites along k)
 *        o_t  = q_t^T S                                   readout after the write
 *    ("nx_nofloat_kda.nx source": gate, then delta write, then read, per token.)
 *    S (dk x dv, fp32) starts as state_pool[state_indices[b], h] and is written back there
 *    when the sequence ends.  The key head used by value head h is h / (Hv / Hk).  No query
 *    scaling is applied (GStar Assignment 2: the formulas omit it; scale = 1).
 *
 *  kda_decode
 *    The same step for one token of each sequence in a batch (the single-token path that
 *    "max.nn.state_space.kda_chunk" names kda_decode), in place on the state pool.
 *
 *  kda_segment_summarize_and_scan
 *    Context-parallel segment summary and exclusive scan ("KDA Context Parallelism"): a
 *    single sequence is cut into N segments; each is reduced to the affine map
 *    F_i(S) = M_i S + U_i (M_i: how the segment transforms its incoming state, dk x dk;
 *    U_i: the state it creates from zero, dk x dv); the maps are applied in sequence order
 *    (an exclusive prefix), giving every segment its incoming and outgoing state and the
 *    final state.  A later kda_chunk_fwd call with cu_seqlens = segment offsets, the incoming
 *    stack as the state pool and state_indices = 0..N-1 then produces every segment's
 *    outputs in parallel; afterwards that pool holds the outgoing states.
 *
 *  kda_prefill_host_pipelined
 *    kda_chunk_fwd's result for one sequence held in host memory, its copies over the host link
 *    pipelined with the kernels in segments.
 *
 *  kda_context_parallel_range_summary / kda_context_parallel_range_finish
 *    The same method across GPUs: each rank reduces its own token range of the sequence to one
 *    affine map, the caller gathers the maps and scans them over the ranks, and each rank
 *    finishes its range from the state entering it.
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major and densely
 *    packed in the stated shapes.  The library allocates no device memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream).  The returned status covers the host-side checks and the launch only.
 *  - Host-side checks are always on: null pointers, extents, Hv % Hk == 0, dtype groupings
 *    that bind no kernel, flag combinations, and token counts within int32 (token offsets are
 *    int32, as cu_seqlens; a larger T returns KDA_ERR_INVALID_ARG).  A failed check returns
 *    before any launch and writes nothing.
 *  - device_status (nullable, device int32): kernels record the first device-side finding
 *    there (KDA_ERR_DEVICE_CHECK for a state slot outside [0, max_slots) or decreasing
 *    offsets -- that sequence is skipped and its slot and outputs are left untouched;
 *    KDA_ERR_DEVICE_TIMEOUT if a bounded wait gave up).  The caller zeroes it beforehand and
 *    reads it after synchronising.  Kernels never trap.
 *  - Inputs must not alias outputs.  Two sequences naming the same pool slot is a caller
 *    error with an unspecified result.  Pool slots not named by state_indices are never
 *    touched.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,    /* null pointer, bad extent, Hv % Hk != 0, bad flags          */
  KDA_ERR_UNSUPPORTED = 2,    /* the dtype grouping / head dims bind no kernel               */
  KDA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than kda_workspace_size()      */
  KDA_ERR_CUDA = 4,           /* a CUDA runtime call (attribute set, launch) failed          */
  KDA_ERR_DEVICE_CHECK = 5,   /* device_status value: bad slot or decreasing offsets         */
  KDA_ERR_DEVICE_TIMEOUT = 6  /* device_status value: a bounded wait gave up                 */
} kda_status_t;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/* flags (bitwise OR) -- the kda_chunk keyword arguments gate_mode, beta_mode, state_layout
 * and use_computebound */
enum {
  KDA_GATE_SAFE = 1u << 0,     /* gate_mode="safe": g = max(g, gate_lower_bound); else "original" */
  KDA_BETA_PROB = 1u << 1,     /* beta_mode="probability": beta used as given; else sigmoid(logits) */
  KDA_STATE_V_FIRST = 1u << 2, /* state_layout="V_FIRST": a slot stores S^T as [dv][dk]; else [dk][dv] */
  KDA_FUSED = 1u << 3,         /* use_computebound: accepted; the bf16 path is always the fused kernel */
  KDA_SEG_SCAN_ONLY = 1u << 4, /* segment call: M and U are inputs, only the scan runs           */
  KDA_FORCE_SIMT = 1u << 5,    /* run the fp32 CUDA-core chunk kernel even for bf16 inputs       */
  KDA_READOUT_HEAD_MAJOR = 1u << 6, /* readout_m / readout_u stored [Hv, T, 128] instead of
                                       [T, Hv, 128] (calls that write or read readouts only)     */
  KDA_SCAN_LOGDEPTH = 1u << 7, /* segment call: the scan in log depth (needs the workspace of
                                  kda_scan_workspace_size); without it the log-depth form is
                                  chosen when that workspace is given and it is expected faster */
  KDA_DEBUG_WITHHOLD_HANDOFF = 1u << 8 /* test hook for the bounded waits (kda_chunk_fwd): the bf16
                                  kernel withholds one "scores ready" signal between its two
                                  warp teams in every chain's first chunk, so the waiting team
                                  gives up after its limit (about one second).  device_status
                                  then reads KDA_ERR_DEVICE_TIMEOUT, the outputs and the pool
                                  slots are unspecified, and the context stays usable.  No
                                  effect on the fp32 kernel. */
};

/*
 * kda_chunk_fwd -- chunk-parallel KDA prefill over a varlen batch (kda_chunk, all parameters).
 *
 *   q, k          [total_tokens, num_k_heads, dk]   qkv_dtype
 *   v             [total_tokens, num_v_heads, dv]   qkv_dtype
 *   raw_gate      [total_tokens, num_v_heads, dk]   fp32, forget-gate pre-activation before dt_bias
 *   beta_logits   [total_tokens, num_v_heads]       fp32 (logits, or probabilities with KDA_BETA_PROB)
 *   a_log         [num_v_heads]                     fp32
 *   dt_bias       [num_v_heads, dk]                 fp32
 *   cu_seqlens    [batch + 1]                       int32 exclusive prefix offsets, cu_seqlens[batch]
 *                                                   <= total_tokens; zero-length sequences allowed
 *   state_pool    [max_slots, num_v_heads, dk, dv]  fp32 (K_FIRST) or [.., dv, dk] (V_FIRST); read
 *                                                   and written in place
 *   state_indices [batch]                           int32 pool slot of each sequence
 *   out           [total_tokens, num_v_heads, dv]   out_dtype; rows outside every sequence untouched
 *   gate_lower_bound                                used only with KDA_GATE_SAFE
 *   workspace     optional device scratch, 256-byte aligned.  With at least kda_workspace_size()
 *                 bytes, a bf16 batch of few or uneven sequences (fewer than three chains, i.e.
 *                 sequence-heads, per SM) may take the split route: every sequence is cut into
 *                 chunk-aligned pieces, the pieces are built in parallel (transition,
 *                 contribution and readouts, as in the context-parallel prefill), applied in order
 *                 from the sequence's pool slot, and the outputs formed from the readouts
 *                 ("KDA Context Parallelism": any cut is a segment boundary).  A planner kernel
 *                 on the device keeps the plain route when, with the real lengths, the pieces would
 *                 not shorten the schedule, or when an offset or a slot is bad (the plain route
 *                 then reports it as usual).  Results agree with the plain route up to rounding.
 *                 NULL or a smaller workspace: the plain route.
 *
 * Supported groupings: (qkv F32, out F32) for any 1 <= dk, dv <= 128 on the fp32 CUDA-core
 * kernel; (qkv BF16, out BF16 or F32) with dk = dv = 128 on the fused tensor-core kernel, or on
 * the fp32 kernel with KDA_FORCE_SIMT.  Anything else returns KDA_ERR_UNSUPPORTED.
 */
KDA_API kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                           const float *raw_gate, const float *beta_logits, const float *a_log,
                           const float *dt_bias, const int32_t *cu_seqlens, int32_t batch,
                           int64_t total_tokens, int32_t num_k_heads, int32_t num_v_heads,
                           int32_t dk, int32_t dv, float *state_pool, int32_t max_slots,
                           const int32_t *state_indices, void *out, kda_dtype_t out_dtype,
                           uint32_t flags, float gate_lower_bound, void *workspace,
                           size_t workspace_bytes, int32_t *device_status, void *stream);

/*
 * kda_decode -- one token of each sequence in a batch, in place on the state pool
 * ("max.nn.state_space.kda_chunk": single-token decode is the kda_decode path of the same
 * recurrence; "nx_nofloat_kda.nx source", kda_step: decay, delta write, readout).  For every
 * sequence b and value head h, with S = state_pool[state_indices[b], h]:
 *     S = Diag(exp(g)) S;   S = S + k (beta (v - k^T S))^T;   out[b,h,:] = q^T S
 * with g and beta as in kda_chunk_fwd.  The result equals kda_chunk_fwd on a batch whose every
 * sequence has one token (cu_seqlens = 0, 1, ..., batch).
 *
 *   q, k          [batch, num_k_heads, dk]   qkv_dtype
 *   v             [batch, num_v_heads, dv]   qkv_dtype
 *   raw_gate      [batch, num_v_heads, dk]   fp32;   beta_logits [batch, num_v_heads] fp32
 *   a_log [num_v_heads], dt_bias [num_v_heads, dk]   fp32
 *   state_pool    as kda_chunk_fwd (K_FIRST or V_FIRST), read and written in place
 *   state_indices [batch] int32;  out [batch, num_v_heads, dv] out_dtype
 *   flags         KDA_GATE_SAFE, KDA_BETA_PROB, KDA_STATE_V_FIRST (others: KDA_ERR_INVALID_ARG)
 *
 * Supported: 1 <= dk, dv <= 128; (qkv F32, out F32) or (qkv BF16, out BF16 or F32); fp32
 * arithmetic throughout.  A slot outside [0, max_slots) is reported in device_status and that
 * sequence is skipped (its output row is not written).  batch = 0 does nothing.
 */
KDA_API kda_status_t kda_decode(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                                const float *raw_gate, const float *beta_logits, const float *a_log,
                                const float *dt_bias, int32_t batch, int32_t num_k_heads,
                                int32_t num_v_heads, int32_t dk, int32_t dv, float *state_pool,
                                int32_t max_slots, const int32_t *state_indices, void *out,
                                kda_dtype_t out_dtype, uint32_t flags, float gate_lower_bound,
                                int32_t *device_status, void *stream);

/*
 * kda_segment_summarize_and_scan -- segment summaries and the exclusive affine scan of ONE
 * sequence ("KDA Context Parallelism": Theory; Compose segments in sequence order; Incoming
 * and outgoing states; Implementation order; Requirements).
 *
 *   k             [T, num_k_heads, dk]    kv_dtype      (ignored with KDA_SEG_SCAN_ONLY)
 *   v             [T, num_v_heads, dv]    kv_dtype      (ignored with KDA_SEG_SCAN_ONLY)
 *   raw_gate, beta_logits, a_log, dt_bias  as in kda_chunk_fwd (ignored with KDA_SEG_SCAN_ONLY)
 *   seg_offsets   [num_segments + 1]       int32 device, seg_offsets[0] = 0 ... = T, non-decreasing
 *   initial_state [num_v_heads, <state>]   fp32, <state> = [dk][dv] (K_FIRST) or [dv][dk] (V_FIRST)
 *   M             [num_segments, num_v_heads, dk, dk]   fp32, row-major, F_i(S) = M_i S + U_i
 *                                          (written; read-only input with KDA_SEG_SCAN_ONLY)
 *   U             [num_segments, num_v_heads, <state>]  fp32 (written; input with SCAN_ONLY)
 *   incoming      [num_segments, num_v_heads, <state>]  fp32 out: state entering segment i
 *   outgoing      [num_segments, num_v_heads, <state>]  fp32 out: state leaving segment i
 *   final_state   [num_v_heads, <state>]                fp32 out: outgoing of the last segment
 *
 * num_segments >= 1.  M_i is the segment's transition (the recurrence run from S = I with zero
 * values); U_i is its local contribution (the recurrence from S = 0).  Left multiplication:
 * out_i = M_i in_i + U_i.  initial_state, M and U (in SCAN_ONLY mode) are never written.
 * Summaries need dk <= 128 and dv <= 128 (fp32 or bf16 k/v).
 *
 *   q, readout_m, readout_u  optional (all three or none; bf16 k/v with dk = dv = 128 only):
 *   q [T, Hk, 128] bf16; the build then also writes, per token, the readout through the
 *   transition readout_m[t] = q_t^T M_{<=t} and of the contribution readout_u[t] = q_t^T U_{<=t}
 *   ([T, Hv, 128] bf16 each; [Hv, T, 128] with KDA_READOUT_HEAD_MAJOR, which makes every
 *   head's rows contiguous for the apply), the inputs of kda_context_parallel_apply.
 *
 *   workspace (device, 256-byte aligned, nullable): with dk = 128 and dv a multiple of 32, at
 *   least kda_scan_workspace_size(num_segments, num_v_heads, dk, dv) bytes let the scan run in
 *   log depth ("KDA Context Parallelism", Compose segments in sequence order: the composition is
 *   associative): ceil(log2 N) levels of P_i <- P_i o P_{i - 2^l}, then every prefix applied to
 *   initial_state.  It is used with KDA_SCAN_LOGDEPTH (else KDA_ERR_WORKSPACE without the
 *   workspace, KDA_ERR_UNSUPPORTED for other dk, dv or more than 65535 segments), or without
 *   that flag where kda_scan_logdepth_preferred says it should finish first (few heads, many
 *   segments).  Results equal the sequential scan's up to rounding (both fp32-accurate).
 */
KDA_API kda_status_t kda_segment_summarize_and_scan(
    const void *k, const void *v, kda_dtype_t kv_dtype, const float *raw_gate,
    const float *beta_logits, const float *a_log, const float *dt_bias, int64_t T,
    int32_t num_k_heads, int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t *seg_offsets,
    int32_t num_segments, const float *initial_state, float *M, float *U, float *incoming,
    float *outgoing, float *final_state, const void *q, void *readout_m, void *readout_u,
    uint32_t flags, float gate_lower_bound, void *workspace, size_t workspace_bytes,
    int32_t *device_status, void *stream);

/* Workspace bytes of the log-depth scan: two sets of every segment's prefix map,
 * 2 * N * H * (128 * 128 + 128 * dv) * 4 (0 where it does not apply: dk != 128, dv not a
 * multiple of 32 up to 128, N < 1).  No counterpart on the pages beyond the associativity. */
KDA_API size_t kda_scan_workspace_size(int32_t num_segments, int32_t num_v_heads, int32_t dk, int32_t dv);
/* 1 if the log-depth scan is expected to finish before the sequential one on the current
 * device (both counted in rounds of tile products over its SMs), else 0. */
KDA_API int32_t kda_scan_logdepth_preferred(int32_t num_segments, int32_t num_v_heads, int32_t dv);

/*
 * kda_context_parallel_apply -- outputs of every segment from its local readouts and its
 * incoming state ("KDA Context Parallelism", Theory: a segment applied to any incoming state
 * without replaying its tokens).  Inside a segment the state after token t is
 * M_{<=t} S_in + U_{<=t}, so out_t = readout_m[t] . S_in + readout_u[t] with
 * readout_m[t] = q_t^T M_{<=t} and readout_u[t] = q_t^T U_{<=t}.
 *
 *   readout_m, readout_u [T, Hv, 128] bf16 (from kda_segment_summarize_and_scan), or
 *     [Hv, T, 128] with KDA_READOUT_HEAD_MAJOR
 *   incoming [N, Hv, <state>] fp32 (flags: KDA_STATE_V_FIRST for the transposed layout)
 *   out [T, Hv, 128] out_dtype
 * dv must be 128; bad segment offsets are reported in device_status and that segment skipped.
 */
KDA_API kda_status_t kda_context_parallel_apply(const void *readout_m, const void *readout_u,
                                                const float *incoming, const int32_t *seg_offsets,
                                                int32_t num_segments, int64_t T, int32_t num_v_heads,
                                                int32_t dv, void *out, kda_dtype_t out_dtype,
                                                uint32_t flags, int32_t *device_status, void *stream);

/*
 * kda_context_parallel_prefill -- the whole prefill of ONE long sequence, context-parallel on
 * one GPU ("KDA Context Parallelism": segment summaries, ordered composition, exclusive scan;
 * "max.nn.state_space.kda_chunk" semantics for every token).
 *
 * The sequence is cut at seg_offsets [N+1] (device int32, 0 .. T, non-decreasing).  One pass
 * over all segments in parallel builds each segment's transition M_i, contribution U_i and two
 * local readouts per token -- through the transition (q_t^T M_{<=t}, dk wide) and of the
 * contribution (q_t^T U_{<=t}) -- into the workspace; the exclusive scan gives every segment its
 * incoming state; a last pass forms out_t = (q_t^T M_{<=t}) S_in + q_t^T U_{<=t}, which equals
 * the token-by-token recurrence started from initial_state.
 *
 *   q, k, v, raw_gate, beta_logits, a_log, dt_bias   as kda_chunk_fwd, one sequence of T tokens
 *   initial_state [Hv, <state>] fp32, read only;  final_state [Hv, <state>] fp32, written
 *   out [T, Hv, dv] out_dtype (BF16 or F32)
 *   M [N,Hv,dk,dk], U / incoming / outgoing [N,Hv,<state>] fp32, written (as in
 *     kda_segment_summarize_and_scan)
 *   workspace >= kda_context_parallel_workspace_size(T, num_v_heads, dv) bytes, 256-byte aligned
 *     device memory; its contents on return are unspecified.  Given at least
 *     kda_context_parallel_workspace_preferred(T, N, num_v_heads, dv) bytes, the build runs each
 *     segment as several chunk-aligned pieces (more chains for the SMs; the results are the
 *     same up to rounding) and composes each segment's M_i, U_i from its pieces'.
 * Supported: bf16 q/k/v with dk = dv = 128; otherwise KDA_ERR_UNSUPPORTED.
 */
KDA_API kda_status_t kda_context_parallel_prefill(
    const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype, const float *raw_gate,
    const float *beta_logits, const float *a_log, const float *dt_bias, int64_t T,
    int32_t num_k_heads, int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t *seg_offsets,
    int32_t num_segments, const float *initial_state, void *out, kda_dtype_t out_dtype,
    float *final_state, float *M, float *U, float *incoming, float *outgoing, uint32_t flags,
    float gate_lower_bound, void *workspace, size_t workspace_bytes, int32_t *device_status,
    void *stream);

/*
 * kda_context_parallel_prefill_static -- kda_context_parallel_prefill for callers that cannot
 * allocate device memory where they run it (a host whose device memory belongs to another
 * component's pool, or a serving loop that must not allocate while requests are in flight,
 * since allocation can synchronise the device).  Same arguments and results, without the
 * workspace: the scratch is a fixed 32 MiB array in device memory carried by the library, which
 * every GPU that loads libkda.so holds until the process exits.  No counterpart on the pages:
 * this is an interface convenience, not part of the method.
 *
 * Limit: kda_context_parallel_workspace_size(T, num_v_heads, dv) <= 32 MiB, i.e. at most
 * 65536 token-heads per call with dv = 128 (for example 2048 tokens x 32 heads); larger calls
 * return KDA_ERR_WORKSPACE and do nothing.  The call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.  The first call on a device looks up the array's
 * device address (once per device, with that device current); make that first call before any
 * stream capture.  The address is kept for the process and belongs to the device's primary
 * context: a caller that destroys that context (cudaDeviceReset) and keeps using the library
 * on the device gets a stale address.  Every call shares the one array and leaves its last
 * contents there (nothing in it needs to start at zero); calls whose work overlaps on the GPU
 * (other streams, or other host threads) race on it and must be serialised by the caller.
 * T beyond INT32_MAX (token offsets are int32) returns KDA_ERR_INVALID_ARG.
 */
KDA_API kda_status_t kda_context_parallel_prefill_static(
    const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype, const float *raw_gate,
    const float *beta_logits, const float *a_log, const float *dt_bias, int64_t T,
    int32_t num_k_heads, int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t *seg_offsets,
    int32_t num_segments, const float *initial_state, void *out, kda_dtype_t out_dtype,
    float *final_state, float *M, float *U, float *incoming, float *outgoing, uint32_t flags,
    float gate_lower_bound, int32_t *device_status, void *stream);

/* Workspace bytes kda_context_parallel_prefill needs: the two bf16 readouts, 2 * T * Hv * dv * 2
 * (SIZE_MAX for T beyond INT32_MAX, which no call accepts: token offsets are int32). */
KDA_API size_t kda_context_parallel_workspace_size(int64_t T, int32_t num_v_heads, int32_t dv);

/*
 * kda_segment_compose -- summaries of segments from the summaries of their pieces: segment i
 * consists of `pieces` consecutive pieces i*pieces .. i*pieces + pieces - 1 (as built by
 * kda_segment_summarize_and_scan over the piece boundaries), and its map is their composition
 * in order ("KDA Context Parallelism", Compose segments in sequence order:
 * (M2, U2) o (M1, U1) = (M2 M1, M2 U1 + U2)).
 *
 *   M_pieces [N*pieces, Hv, dk, dk], U_pieces / incoming_pieces [N*pieces, Hv, <state>] fp32
 *   final_state [Hv, <state>] (the scan's final state: the last segment's outgoing state)
 *   M [N, Hv, dk, dk], U / incoming / outgoing [N, Hv, <state>] fp32, written: incoming[i] is
 *     the incoming state of segment i's first piece, outgoing[i] that of segment i + 1's
 *   flags: KDA_STATE_V_FIRST selects <state> = [dv, dk]; dk, dv <= 128 (fp32 CUDA-core kernel)
 */
KDA_API kda_status_t kda_segment_compose(const float *M_pieces, const float *U_pieces,
                                         const float *incoming_pieces, const float *final_state,
                                         int32_t num_segments, int32_t pieces, int32_t num_v_heads,
                                         int32_t dk, int32_t dv, float *M, float *U, float *incoming,
                                         float *outgoing, uint32_t flags, void *stream);

/* Pieces per segment (1..8) that kda_context_parallel_prefill builds on the current device. */
KDA_API int32_t kda_context_parallel_pieces(int64_t T, int32_t num_segments, int32_t num_v_heads);

/* Piece boundaries: piece_offsets [N*pieces + 1] (device int32, written) from seg_offsets [N+1]:
 * piece p of segment [s0, s1) with nch = ceil((s1 - s0) / 64) chunks starts at token
 * s0 + 64 * floor(nch * p / pieces), capped at s1 (short segments give empty pieces); the last
 * entry is seg_offsets[N].  Decreasing seg_offsets give decreasing piece offsets, which the
 * segment build reports as KDA_ERR_DEVICE_CHECK. */
KDA_API kda_status_t kda_context_parallel_piece_offsets(const int32_t *seg_offsets, int32_t num_segments,
                                                        int32_t pieces, int32_t *piece_offsets, void *stream);

/* Workspace bytes with which kda_context_parallel_prefill splits the segments into pieces on
 * the current device (the readouts, plus per piece a transition, a contribution and an incoming
 * state); equal to kda_context_parallel_workspace_size when no split pays off.  Depends on the
 * current device's SM count: query it with the device current that will run the prefill. */
KDA_API size_t kda_context_parallel_workspace_preferred(int64_t T, int32_t num_segments,
                                                        int32_t num_v_heads, int32_t dv);

/*
 * Context parallelism across GPUs ("KDA Context Parallelism", Theory: a segment summarised as the
 * affine map F(S) = M S + U is applied to any incoming state without replaying its tokens;
 * Compose segments in sequence order; Incoming and outgoing states).  One long sequence is cut
 * into consecutive token ranges, one per rank (GPU); a rank holds only its own range's tokens
 * and cuts that range into its own segments.  Per rank, in this order:
 *   1. kda_context_parallel_range_summary: the range built (as chunk-aligned pieces, all in
 *      parallel, with per-token readouts kept in the workspace) and composed into ONE map of the
 *      whole range, range_M [Hv,128,128] and range_U [Hv,<state>];
 *   2. the caller gathers every rank's map in rank order (an all-gather; the library makes no
 *      collective call) and runs the exclusive scan over the ranks from the sequence's initial
 *      state (kda_segment_summarize_and_scan with KDA_SEG_SCAN_ONLY): incoming[r] is the state
 *      entering rank r's range and the scan's final state is the sequence's final state;
 *   3. kda_context_parallel_range_finish: from the state entering the range, the pieces'
 *      incoming states (the exclusive scan over the pieces), the summary and the incoming and
 *      outgoing states of each of the range's segments, and the outputs of every token.
 * Steps 1 and 3 use the same workspace (>= kda_context_parallel_range_workspace_size bytes,
 * 256-byte aligned), which the caller leaves untouched in between, on the same device, with the
 * same T, num_segments, num_v_heads and layout flag.  bf16 q/k/v with dk = dv = 128 only.
 * With one rank the three steps give what kda_context_parallel_prefill gives.
 *
 *   q, k, v, raw_gate, beta_logits, a_log, dt_bias   the range's tokens, as kda_chunk_fwd (T may
 *     be 0: the map is then the identity and zero, and the token pointers may be NULL)
 *   seg_offsets [num_segments + 1] int32 device, 0 .. T, non-decreasing (the range's segments)
 *   range_M, range_U  fp32, written by step 1
 *   range_incoming [Hv,<state>] fp32, read by step 3;  range_outgoing [Hv,<state>] fp32 written
 *     by step 3 (nullable): the state leaving the range
 *   out [T,Hv,128] out_dtype;  M [N,Hv,128,128], U / incoming / outgoing [N,Hv,<state>] fp32,
 *     written by step 3, as kda_context_parallel_prefill's
 * A bad offset is reported in device_status (KDA_ERR_DEVICE_CHECK) and its piece skipped.
 */
KDA_API size_t kda_context_parallel_range_workspace_size(int64_t T, int32_t num_segments,
                                                         int32_t num_v_heads, int32_t dv);
KDA_API kda_status_t kda_context_parallel_range_summary(
    const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype, const float *raw_gate,
    const float *beta_logits, const float *a_log, const float *dt_bias, int64_t T,
    int32_t num_k_heads, int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t *seg_offsets,
    int32_t num_segments, float *range_M, float *range_U, uint32_t flags, float gate_lower_bound,
    void *workspace, size_t workspace_bytes, int32_t *device_status, void *stream);
KDA_API kda_status_t kda_context_parallel_range_finish(
    int64_t T, int32_t num_v_heads, int32_t dk, int32_t dv, int32_t num_segments,
    const float *range_incoming, void *out, kda_dtype_t out_dtype, float *range_outgoing, float *M,
    float *U, float *incoming, float *outgoing, uint32_t flags, void *workspace,
    size_t workspace_bytes, int32_t *device_status, void *stream);

/*
 * kda_prefill_host_pipelined -- the prefill of ONE sequence whose inputs and outputs are in
 * host memory (pinned, for the copies to overlap), as kda_chunk_fwd computes it
 * ("max.nn.state_space.kda_chunk": the recurrence over 64-token chunks, the state carried from
 * chunk to chunk), with the copies over the host link pipelined in segments of
 * segment_tokens tokens (a multiple of 64): segment i's inputs are copied in while segment
 * i - 1 runs and earlier segments' outputs are copied out, both directions at once.  Segment
 * boundaries fall on chunk boundaries, so the outputs and the final state equal
 * kda_chunk_fwd's on the whole sequence bit for bit.
 *
 *   q, k [T, Hk, 128], v [T, Hv, 128] bf16; raw_gate [T, Hv, 128], beta_logits [T, Hv],
 *   a_log [Hv], dt_bias [Hv, 128] fp32; initial_state [Hv, <state>] fp32   HOST, read
 *   out [T, Hv, 128] out_dtype; final_state [Hv, <state>] fp32              HOST, written
 *   workspace: DEVICE, >= kda_prefill_host_workspace_size(...) bytes, 256-byte aligned: the
 *     staged sequence (inputs, outputs, state); its contents on return are unspecified
 *   flags: gate / beta modes and KDA_STATE_V_FIRST; device_status (device, nullable) as for
 *     kda_chunk_fwd
 * Asynchronous on `stream`: the kernels run there and the stream completes after the last
 * copy out; read the host outputs after synchronising it.  The copies run on two helper
 * streams the library creates on a device's first call and keeps (with four events); calls are
 * serialised while they enqueue.  Those streams and events belong to the device's primary
 * context and are kept for the process: a caller that destroys that context
 * (cudaDeviceReset) leaves them stale, and later calls on the device fail.  bf16 q/k/v with
 * dk = dv = 128 only; else KDA_ERR_UNSUPPORTED.
 */
KDA_API size_t kda_prefill_host_workspace_size(int64_t T, int32_t num_k_heads, int32_t num_v_heads,
                                               kda_dtype_t out_dtype, int64_t segment_tokens);
KDA_API kda_status_t kda_prefill_host_pipelined(
    const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype, const float *raw_gate,
    const float *beta_logits, const float *a_log, const float *dt_bias, int64_t T,
    int32_t num_k_heads, int32_t num_v_heads, int32_t dk, int32_t dv, const float *initial_state,
    void *out, kda_dtype_t out_dtype, float *final_state, int64_t segment_tokens, uint32_t flags,
    float gate_lower_bound, void *workspace, size_t workspace_bytes, int32_t *device_status,
    void *stream);

/* Bytes of workspace with which kda_chunk_fwd may take its split route on the current device
 * (0 when the batch has chains enough for the SMs, for dk or dv other than 128, or with
 * KDA_FORCE_SIMT; the workspace is optional either way).  kda_segment_summarize_and_scan needs
 * none.  num_segments is unused. */
KDA_API size_t kda_workspace_size(int64_t total_tokens, int32_t batch, int32_t num_k_heads,
                          int32_t num_v_heads, int32_t dk, int32_t dv, int32_t num_segments,
                          uint32_t flags);

/* Static, human-readable name of a status code. */
KDA_API const char *kda_status_string(kda_status_t status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
KDA_API int32_t kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
