// kda_api.cu -- the C ABI (include/kda.h): host-side validation and kernel dispatch.
//
// Shapes, flags and the state pool follow "max.nn.state_space.kda_chunk" (Parameters, Returns,
// Raises): a dtype grouping that binds no kernel, or ranks/extents that disagree, is an error.
// Unlike that op, whose shape guards are debug-only, every check here is always on.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace kda {
cudaError_t launch_fused_chunk(const FusedArgs& a, cudaStream_t stream);
bool fused_available();
}  // namespace kda

namespace {

constexpr uint32_t kKnownFlags = KDA_GATE_SAFE | KDA_BETA_PROB | KDA_STATE_V_FIRST | KDA_FUSED |
                                 KDA_SEG_SCAN_ONLY | KDA_FORCE_SIMT | KDA_READOUT_HEAD_MAJOR | KDA_SCAN_LOGDEPTH |
                                 KDA_DEBUG_WITHHOLD_HANDOFF;

bool dtype_ok(kda_dtype_t t) { return t == KDA_F32 || t == KDA_BF16; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

// Pieces per segment for the context-parallel segment build.  The fused kernel runs one chain
// (segment piece, head) per SM, so N * Hv chains take ceil(N Hv / SMs) rounds of a whole
// segment's length; k pieces per segment take ceil(k N Hv / SMs) rounds of 1/k of it.  The
// smallest k (up to 8) that saves at least 3 % is taken, with pieces of four chunks or more on
// average.
int choose_pieces(int64_t T, int32_t N, int32_t Hv) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess || sms <= 0)
    return 1;
  const int64_t chains = (int64_t)N * Hv;
  double best = (double)((chains + sms - 1) / sms);
  int best_k = 1;
  for (int k = 2; k <= 8; ++k) {
    if (T < (int64_t)N * k * 256) break;
    const double cost = (double)((chains * k + sms - 1) / sms) / k;
    if (cost < best * 0.97) {
      best = cost;
      best_k = k;
    }
  }
  return best_k;
}

// workspace bytes of the pieces: boundaries, transitions, contributions, incoming states (one
// extra slot: the scan's outgoing state of piece p is the incoming state of piece p + 1)
size_t pieces_bytes(int32_t N, int k, int32_t Hv, int32_t dk, int32_t dv) {
  const size_t np = (size_t)N * k;
  return round256((np + 1) * sizeof(int32_t)) + np * Hv * (size_t)dk * dk * sizeof(float) +
         np * Hv * (size_t)dk * dv * sizeof(float) + (np + 1) * Hv * (size_t)dk * dv * sizeof(float);
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

// Piece length (tokens, a multiple of 64) for the split route of kda_chunk_fwd, or 0 when the
// batch has chains (sequence-heads) enough for the SMs -- more than half as many as SMs -- and
// runs as it is.  Estimated time in chunk steps for piece length P, with sequences of the mean
// length: rounds of chains on the SMs (one chain per SM) times P / 64, plus 0.35 chunk steps
// for every piece the scan applies in order.  The planner on the device still keeps the plain
// route when, with the real lengths, the pieces would not pay.
int choose_piece_len(int64_t T, int32_t batch, int32_t Hv) {
  const int sms = sm_count();
  if (sms <= 0 || T <= 0 || batch <= 0 || 2 * (int64_t)batch * Hv > (int64_t)sms) return 0;
  const int64_t mean = (T + batch - 1) / batch;
  const int64_t top = ((mean + 63) / 64) * 64;
  int best_p = 0;
  double best = 0.0;
  for (int64_t P = 256; P <= top && P <= ((int64_t)1 << 30); P += (P < 4096 ? 64 : P / 16 / 64 * 64)) {
    const int64_t per_seq = (mean + P - 1) / P;
    const int64_t chains = (int64_t)batch * per_seq * Hv;
    const double est = (double)((chains + sms - 1) / sms) * (double)(P / 64) + 0.35 * (double)per_seq;
    if (best_p == 0 || est < best) {
      best = est;
      best_p = (int)P;
    }
  }
  return best_p;
}

int32_t max_pieces_of(int64_t T, int32_t batch, int P) { return batch + (int32_t)((T + P - 1) / P); }

// workspace of the split route: readouts, the pieces' transitions, contributions and incoming
// states, piece boundaries, first piece per sequence, the fallback flag
size_t split_bytes(int64_t T, int32_t batch, int32_t Hv, int P) {
  const size_t np = (size_t)max_pieces_of(T, batch, P);
  const size_t blk = (size_t)Hv * 128 * 128 * sizeof(float);
  return round256((size_t)2 * T * Hv * 128 * 2) + 3 * np * blk + round256((np + 1) * sizeof(int32_t)) +
         round256(((size_t)batch + 1) * sizeof(int32_t)) + 256;
}

}  // namespace

extern "C" kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype,
                                      const float* raw_gate, const float* beta_logits, const float* a_log,
                                      const float* dt_bias, const int32_t* cu_seqlens, int32_t batch,
                                      int64_t total_tokens, int32_t num_k_heads, int32_t num_v_heads,
                                      int32_t dk, int32_t dv, float* state_pool, int32_t max_slots,
                                      const int32_t* state_indices, void* out, kda_dtype_t out_dtype,
                                      uint32_t flags, float gate_lower_bound, void* workspace,
                                      size_t workspace_bytes, int32_t* device_status, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (batch < 0 || total_tokens < 0 || total_tokens > INT32_MAX || num_k_heads <= 0 || num_v_heads <= 0 ||
      dk <= 0 || dv <= 0 || max_slots <= 0)
    return KDA_ERR_INVALID_ARG;  // token offsets are int32, as cu_seqlens
  if (num_v_heads % num_k_heads != 0) return KDA_ERR_INVALID_ARG;
  if ((flags & ~kKnownFlags) != 0 || (flags & KDA_SEG_SCAN_ONLY)) return KDA_ERR_INVALID_ARG;
  if (!cu_seqlens || !state_pool || !state_indices) return KDA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!q || !k || !v || !raw_gate || !beta_logits || !out)) return KDA_ERR_INVALID_ARG;
  if (!a_log || !dt_bias) return KDA_ERR_INVALID_ARG;
  if (!dtype_ok(qkv_dtype) || !dtype_ok(out_dtype)) return KDA_ERR_UNSUPPORTED;
  if (batch == 0) return KDA_OK;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = qkv_dtype == KDA_BF16;
  const bool use_fused = bf16 && !(flags & KDA_FORCE_SIMT) && dk == 128 && dv == 128 && kda::fused_available();
  if (!use_fused) {
    if (dk > 128 || dv > 128) return KDA_ERR_UNSUPPORTED;
    if (!bf16 && out_dtype != KDA_F32) return KDA_ERR_UNSUPPORTED;
    if (bf16 && !(flags & KDA_FORCE_SIMT) && (dk != 128 || dv != 128)) return KDA_ERR_UNSUPPORTED;
    kda::SimtArgs a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.in_bf16 = bf16;
    a.raw_gate = raw_gate;
    a.beta = beta_logits;
    a.a_log = a_log;
    a.dt_bias = dt_bias;
    a.cu = cu_seqlens;
    a.batch = batch;
    a.total_tokens = total_tokens;
    a.Hk = num_k_heads;
    a.Hv = num_v_heads;
    a.dk = dk;
    a.w = dv;
    a.dv_in = dv;
    a.state_in = state_pool;
    a.state_out = state_pool;
    a.max_slots = max_slots;
    a.slots = state_indices;
    a.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
    a.init_mode = 0;
    a.values_zero = 0;
    a.out = out;
    a.out_bf16 = out_dtype == KDA_BF16;
    a.flags = flags;
    a.lb = gate_lower_bound;
    a.status = device_status;
    return kda::launch_simt_chunk(a, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(raw_gate) || !aligned16(dt_bias) ||
      !aligned16(state_pool) || !aligned16(out))
    return KDA_ERR_INVALID_ARG;
  kda::FusedArgs f{};
  f.q = q;
  f.k = k;
  f.v = v;
  f.raw_gate = raw_gate;
  f.beta = beta_logits;
  f.a_log = a_log;
  f.dt_bias = dt_bias;
  f.cu = cu_seqlens;
  f.batch = batch;
  f.total_tokens = total_tokens;
  f.Hk = num_k_heads;
  f.Hv = num_v_heads;
  f.state_in = state_pool;
  f.state_out = state_pool;
  f.max_slots = max_slots;
  f.slots = state_indices;
  f.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  f.init_mode = 0;
  f.values_zero = 0;
  f.out = out;
  f.out_bf16 = out_dtype == KDA_BF16;
  f.flags = flags;
  f.lb = gate_lower_bound;
  f.status = device_status;
  const int P = choose_piece_len(total_tokens, batch, num_v_heads);
  if (P == 0 || !workspace || workspace_bytes < split_bytes(total_tokens, batch, num_v_heads, P) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return kda::launch_fused_chunk(f, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;

  // Split route: sequences cut into pieces of at most P tokens, the pieces built in parallel
  // (transition, contribution, readouts), applied in order from each sequence's pool slot, then
  // the outputs formed from the readouts.  A planner kernel lays the pieces out and, if an
  // offset or a slot is bad or the pieces would not shorten the schedule, sets the fallback
  // flag: then only the plain launch runs.
  const int32_t np = max_pieces_of(total_tokens, batch, P);
  const size_t blk = (size_t)num_v_heads * 128 * 128;
  uint8_t* w = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16_raw* o_m = reinterpret_cast<__nv_bfloat16_raw*>(w);
  __nv_bfloat16_raw* o_u = o_m + (size_t)total_tokens * num_v_heads * 128;
  w += round256((size_t)2 * total_tokens * num_v_heads * 128 * 2);
  float* pM = reinterpret_cast<float*>(w);
  float* pU = pM + (size_t)np * blk;
  float* pIn = pU + (size_t)np * blk;
  w += 3 * (size_t)np * blk * sizeof(float);
  int32_t* piece_offs = reinterpret_cast<int32_t*>(w);
  w += round256(((size_t)np + 1) * sizeof(int32_t));
  int32_t* seq_first = reinterpret_cast<int32_t*>(w);
  w += round256(((size_t)batch + 1) * sizeof(int32_t));
  int32_t* fallback = reinterpret_cast<int32_t*>(w);

  kda::PlanArgs pa{};
  pa.cu = cu_seqlens;
  pa.slots = state_indices;
  pa.batch = batch;
  pa.total_tokens = total_tokens;
  pa.max_slots = max_slots;
  pa.piece_len = P;
  pa.max_pieces = np;
  pa.num_heads = num_v_heads;
  pa.num_sms = sm_count();
  pa.piece_offs = piece_offs;
  pa.seq_first = seq_first;
  pa.fallback = fallback;
  if (kda::launch_plan_pieces(pa, s) != cudaSuccess) return KDA_ERR_CUDA;
  // plain route (runs only on fallback)
  f.gate_flag = fallback;
  f.gate_run_if = 1;
  if (kda::launch_fused_chunk(f, s) != cudaSuccess) return KDA_ERR_CUDA;
  // the pieces: both states and both readouts in one launch
  kda::FusedArgs bf = f;
  bf.cu = piece_offs;
  bf.batch = np;
  bf.state_in = nullptr;
  bf.max_slots = np;
  bf.slots = nullptr;
  bf.init_mode = 0;
  bf.values_zero = 0;
  bf.build = 1;
  bf.state_out = pM;
  bf.state_out2 = pU;
  bf.out = o_m;
  bf.out2 = o_u;
  bf.out_bf16 = 1;
  bf.readout_hm = 1;  // the readouts are this call's own: head-major, contiguous per head
  bf.gate_run_if = 0;
  if (kda::launch_fused_chunk(bf, s) != cudaSuccess) return KDA_ERR_CUDA;
  kda::PoolScanArgs ps{};
  ps.M = pM;
  ps.U = pU;
  ps.seq_first = seq_first;
  ps.slots = state_indices;
  ps.fallback = fallback;
  ps.batch = batch;
  ps.H = num_v_heads;
  ps.dv = 128;
  ps.v_first = f.v_first;
  ps.pool = state_pool;
  ps.incoming = pIn;
  if (kda::launch_pool_scan(ps, s) != cudaSuccess) return KDA_ERR_CUDA;
  kda::ApplyArgs ap{};
  ap.seg_offsets = piece_offs;
  ap.num_segments = np;
  ap.total_tokens = total_tokens;
  ap.Hv = num_v_heads;
  ap.incoming = pIn;
  ap.v_first = f.v_first;
  ap.o_m = o_m;
  ap.o_u = o_u;
  ap.out = out;
  ap.out_bf16 = out_dtype == KDA_BF16;
  ap.status = device_status;
  ap.readout_hm = 1;
  ap.skip_flag = fallback;
  return kda::launch_cp_apply(ap, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_decode(const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype,
                                   const float* raw_gate, const float* beta_logits, const float* a_log,
                                   const float* dt_bias, int32_t batch, int32_t num_k_heads, int32_t num_v_heads,
                                   int32_t dk, int32_t dv, float* state_pool, int32_t max_slots,
                                   const int32_t* state_indices, void* out, kda_dtype_t out_dtype, uint32_t flags,
                                   float gate_lower_bound, int32_t* device_status, void* stream) {
  if (batch < 0 || num_k_heads <= 0 || num_v_heads <= 0 || dk <= 0 || dv <= 0 || max_slots <= 0)
    return KDA_ERR_INVALID_ARG;
  if (num_v_heads % num_k_heads != 0) return KDA_ERR_INVALID_ARG;
  if ((flags & ~(uint32_t)(KDA_GATE_SAFE | KDA_BETA_PROB | KDA_STATE_V_FIRST)) != 0) return KDA_ERR_INVALID_ARG;
  if (!state_pool || !state_indices || !a_log || !dt_bias) return KDA_ERR_INVALID_ARG;
  if (batch > 0 && (!q || !k || !v || !raw_gate || !beta_logits || !out)) return KDA_ERR_INVALID_ARG;
  if (!dtype_ok(qkv_dtype) || !dtype_ok(out_dtype)) return KDA_ERR_UNSUPPORTED;
  if (qkv_dtype == KDA_F32 && out_dtype != KDA_F32) return KDA_ERR_UNSUPPORTED;
  if (dk > 128 || dv > 128) return KDA_ERR_UNSUPPORTED;
  if (batch == 0) return KDA_OK;
  kda::DecodeArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.in_bf16 = qkv_dtype == KDA_BF16;
  a.raw_gate = raw_gate;
  a.beta = beta_logits;
  a.a_log = a_log;
  a.dt_bias = dt_bias;
  a.batch = batch;
  a.Hk = num_k_heads;
  a.Hv = num_v_heads;
  a.dk = dk;
  a.dv = dv;
  a.pool = state_pool;
  a.max_slots = max_slots;
  a.slots = state_indices;
  a.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  a.out = out;
  a.out_bf16 = out_dtype == KDA_BF16;
  a.flags = flags;
  a.lb = gate_lower_bound;
  a.status = device_status;
  return kda::launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_segment_summarize_and_scan(
    const void* k, const void* v, kda_dtype_t kv_dtype, const float* raw_gate, const float* beta_logits,
    const float* a_log, const float* dt_bias, int64_t T, int32_t num_k_heads, int32_t num_v_heads,
    int32_t dk, int32_t dv, const int32_t* seg_offsets, int32_t num_segments, const float* initial_state,
    float* M, float* U, float* incoming, float* outgoing, float* final_state, const void* q, void* readout_m,
    void* readout_u, uint32_t flags, float gate_lower_bound, void* workspace, size_t workspace_bytes,
    int32_t* device_status, void* stream) {
  if (num_segments < 1 || num_v_heads <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
  const bool readouts = q || readout_m || readout_u;
  if (readouts && (!q || !readout_m || !readout_u)) return KDA_ERR_INVALID_ARG;
  if (readouts && (flags & KDA_SEG_SCAN_ONLY)) return KDA_ERR_INVALID_ARG;
  if ((flags & ~kKnownFlags) != 0) return KDA_ERR_INVALID_ARG;
  if (!initial_state || !M || !U || !incoming || !outgoing || !final_state) return KDA_ERR_INVALID_ARG;
  if (dk > 128 || dv > 128) return KDA_ERR_UNSUPPORTED;
  // the scan's form: log depth when forced (and possible) or when given its workspace and expected
  // to finish first; the checks come before any launch
  const size_t log_need = kda::logdepth_scan_bytes(num_segments, num_v_heads, dk, dv);
  const bool log_possible = log_need > 0 && num_segments <= 65535;
  const bool log_ws = workspace && workspace_bytes >= log_need && !(reinterpret_cast<uintptr_t>(workspace) & 255u);
  if (flags & KDA_SCAN_LOGDEPTH) {
    if (!log_possible) return KDA_ERR_UNSUPPORTED;
    if (!log_ws) return KDA_ERR_WORKSPACE;
  }
  const bool use_log = log_possible && log_ws &&
                       ((flags & KDA_SCAN_LOGDEPTH) || kda::logdepth_scan_preferred(num_segments, num_v_heads, dv));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  if (!(flags & KDA_SEG_SCAN_ONLY)) {
    if (T < 0 || T > INT32_MAX || num_k_heads <= 0 || num_v_heads % num_k_heads != 0) return KDA_ERR_INVALID_ARG;
    if (!seg_offsets || !a_log || !dt_bias) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!k || !v || !raw_gate || !beta_logits)) return KDA_ERR_INVALID_ARG;
    if (!dtype_ok(kv_dtype)) return KDA_ERR_UNSUPPORTED;
    const bool use_fused = kv_dtype == KDA_BF16 && !(flags & KDA_FORCE_SIMT) && dk == 128 && dv == 128 &&
                           kda::fused_available();
    if (readouts && !use_fused) return KDA_ERR_UNSUPPORTED;
    if (readouts && (!aligned16(q) || !aligned16(readout_m) || !aligned16(readout_u))) return KDA_ERR_INVALID_ARG;
    if (use_fused) {
      if (!aligned16(k) || !aligned16(v) || !aligned16(raw_gate) || !aligned16(dt_bias) || !aligned16(M) ||
          !aligned16(U))
        return KDA_ERR_INVALID_ARG;
      kda::FusedArgs f{};
      f.q = q;
      f.k = k;
      f.v = v;
      f.raw_gate = raw_gate;
      f.beta = beta_logits;
      f.a_log = a_log;
      f.dt_bias = dt_bias;
      f.cu = seg_offsets;
      f.batch = num_segments;
      f.total_tokens = T;
      f.Hk = num_k_heads;
      f.Hv = num_v_heads;
      f.max_slots = num_segments;
      f.slots = nullptr;
      f.out = readout_m;
      f.out2 = readout_u;
      f.out_bf16 = 1;
      f.readout_hm = (flags & KDA_READOUT_HEAD_MAJOR) ? 1 : 0;
      f.flags = flags;
      f.lb = gate_lower_bound;
      f.status = device_status;
      f.state_in = nullptr;
      // one launch carries both: transition M_i (from I, zero values, row-major) and the local
      // contribution U_i (from 0, the real values, in the state layout)
      f.build = 1;
      f.state_out = M;
      f.state_out2 = U;
      f.v_first = v_first;
      if (kda::launch_fused_chunk(f, s) != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (!use_fused) {
      kda::SimtArgs a{};
      a.q = nullptr;
      a.k = k;
      a.v = v;
      a.in_bf16 = kv_dtype == KDA_BF16;
      a.raw_gate = raw_gate;
      a.beta = beta_logits;
      a.a_log = a_log;
      a.dt_bias = dt_bias;
      a.cu = seg_offsets;
      a.batch = num_segments;
      a.total_tokens = T;
      a.Hk = num_k_heads;
      a.Hv = num_v_heads;
      a.dk = dk;
      a.dv_in = dv;
      a.max_slots = num_segments;
      a.slots = nullptr;
      a.out = nullptr;
      a.flags = flags;
      a.lb = gate_lower_bound;
      a.status = device_status;
      // transition M_i: state started at I (width dk), zero values, stored row-major
      a.w = dk;
      a.state_in = nullptr;
      a.state_out = M;
      a.v_first = 0;
      a.init_mode = 2;
      a.values_zero = 1;
      if (kda::launch_simt_chunk(a, s) != cudaSuccess) return KDA_ERR_CUDA;
      // local contribution U_i: state started at 0, real values, stored in the state layout
      a.w = dv;
      a.state_out = U;
      a.v_first = v_first;
      a.init_mode = 1;
      a.values_zero = 0;
      if (kda::launch_simt_chunk(a, s) != cudaSuccess) return KDA_ERR_CUDA;
    }
  }
  kda::ScanArgs sa{};
  sa.M = M;
  sa.U = U;
  sa.initial = initial_state;
  sa.N = num_segments;
  sa.H = num_v_heads;
  sa.dk = dk;
  sa.dv = dv;
  sa.v_first = v_first;
  sa.incoming = incoming;
  sa.outgoing = outgoing;
  sa.final_state = final_state;
  if (use_log)
    return kda::launch_affine_scan_logdepth(sa, reinterpret_cast<float*>(workspace), s) == cudaSuccess ? KDA_OK
                                                                                                      : KDA_ERR_CUDA;
  return kda::launch_affine_scan(sa, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" size_t kda_scan_workspace_size(int32_t num_segments, int32_t num_v_heads, int32_t dk, int32_t dv) {
  return kda::logdepth_scan_bytes(num_segments, num_v_heads, dk, dv);
}

extern "C" int32_t kda_scan_logdepth_preferred(int32_t num_segments, int32_t num_v_heads, int32_t dv) {
  if (num_segments < 1 || num_segments > 65535 || num_v_heads < 1 || dv < 32 || dv > 128 || dv % 32) return 0;
  return kda::logdepth_scan_preferred(num_segments, num_v_heads, dv) ? 1 : 0;
}

extern "C" size_t kda_context_parallel_workspace_size(int64_t T, int32_t num_v_heads, int32_t dv) {
  if (T < 0 || num_v_heads <= 0 || dv <= 0) return 0;
  if (T > INT32_MAX) return SIZE_MAX;  // beyond the int32 token offsets: no workspace can serve it
  return (size_t)2 * (size_t)T * (size_t)num_v_heads * (size_t)dv * 2;
}

extern "C" int32_t kda_context_parallel_pieces(int64_t T, int32_t num_segments, int32_t num_v_heads) {
  if (T < 0 || num_segments < 1 || num_v_heads <= 0) return 1;
  return choose_pieces(T, num_segments, num_v_heads);
}

extern "C" kda_status_t kda_context_parallel_piece_offsets(const int32_t* seg_offsets, int32_t num_segments,
                                                           int32_t pieces, int32_t* piece_offsets, void* stream) {
  if (num_segments < 1 || pieces < 1 || !seg_offsets || !piece_offsets) return KDA_ERR_INVALID_ARG;
  return kda::launch_split_offsets(seg_offsets, num_segments, pieces, piece_offsets,
                                   reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_segment_compose(const float* M_pieces, const float* U_pieces,
                                            const float* incoming_pieces, const float* final_state,
                                            int32_t num_segments, int32_t pieces, int32_t num_v_heads, int32_t dk,
                                            int32_t dv, float* M, float* U, float* incoming, float* outgoing,
                                            uint32_t flags, void* stream) {
  if (num_segments < 1 || pieces < 1 || num_v_heads <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
  if ((flags & ~kKnownFlags) != 0) return KDA_ERR_INVALID_ARG;
  if (!M_pieces || !U_pieces || !incoming_pieces || !final_state || !M || !U || !incoming || !outgoing)
    return KDA_ERR_INVALID_ARG;
  if (dk > 128 || dv > 128) return KDA_ERR_UNSUPPORTED;
  kda::ComposeArgs ca{};
  ca.M = M_pieces;
  ca.U = U_pieces;
  ca.inc = incoming_pieces;
  ca.final_state = final_state;
  ca.N = num_segments;
  ca.k = pieces;
  ca.H = num_v_heads;
  ca.dk = dk;
  ca.dv = dv;
  ca.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  ca.M_out = M;
  ca.U_out = U;
  ca.incoming = incoming;
  ca.outgoing = outgoing;
  return kda::launch_compose_pieces(ca, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? KDA_OK
                                                                                                 : KDA_ERR_CUDA;
}

extern "C" size_t kda_context_parallel_workspace_preferred(int64_t T, int32_t num_segments, int32_t num_v_heads,
                                                           int32_t dv) {
  const size_t base = kda_context_parallel_workspace_size(T, num_v_heads, dv);
  if (base == 0 || base == SIZE_MAX || num_segments < 1) return base;
  const int k = choose_pieces(T, num_segments, num_v_heads);
  return k > 1 ? round256(base) + pieces_bytes(num_segments, k, num_v_heads, dv, dv) : base;
}

extern "C" kda_status_t kda_context_parallel_apply(const void* readout_m, const void* readout_u,
                                                   const float* incoming, const int32_t* seg_offsets,
                                                   int32_t num_segments, int64_t T, int32_t num_v_heads, int32_t dv,
                                                   void* out, kda_dtype_t out_dtype, uint32_t flags,
                                                   int32_t* device_status, void* stream) {
  if (num_segments < 1 || T < 0 || T > INT32_MAX || num_v_heads <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
  if ((flags & ~kKnownFlags) != 0) return KDA_ERR_INVALID_ARG;
  if (!readout_m || !readout_u || !incoming || !seg_offsets || !out) return KDA_ERR_INVALID_ARG;
  if (!dtype_ok(out_dtype)) return KDA_ERR_UNSUPPORTED;
  if (dv != 128) return KDA_ERR_UNSUPPORTED;
  if (!aligned16(readout_m) || !aligned16(readout_u) || !aligned16(out)) return KDA_ERR_INVALID_ARG;
  kda::ApplyArgs ap{};
  ap.seg_offsets = seg_offsets;
  ap.num_segments = num_segments;
  ap.total_tokens = T;
  ap.Hv = num_v_heads;
  ap.incoming = incoming;
  ap.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  ap.o_m = readout_m;
  ap.o_u = readout_u;
  ap.out = out;
  ap.out_bf16 = out_dtype == KDA_BF16;
  ap.status = device_status;
  ap.readout_hm = (flags & KDA_READOUT_HEAD_MAJOR) ? 1 : 0;
  return kda::launch_cp_apply(ap, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_context_parallel_prefill(
    const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype, const float* raw_gate,
    const float* beta_logits, const float* a_log, const float* dt_bias, int64_t T, int32_t num_k_heads,
    int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t* seg_offsets, int32_t num_segments,
    const float* initial_state, void* out, kda_dtype_t out_dtype, float* final_state, float* M, float* U,
    float* incoming, float* outgoing, uint32_t flags, float gate_lower_bound, void* workspace,
    size_t workspace_bytes, int32_t* device_status, void* stream) {
  if (num_segments < 1 || T < 0 || T > INT32_MAX || num_k_heads <= 0 || num_v_heads <= 0 || dk <= 0 || dv <= 0)
    return KDA_ERR_INVALID_ARG;  // token offsets are int32
  if ((flags & ~kKnownFlags) != 0 || (flags & (KDA_SEG_SCAN_ONLY | KDA_FORCE_SIMT))) return KDA_ERR_INVALID_ARG;
  if (!q || !out) return KDA_ERR_INVALID_ARG;
  if (!dtype_ok(qkv_dtype) || !dtype_ok(out_dtype)) return KDA_ERR_UNSUPPORTED;
  if (qkv_dtype != KDA_BF16 || dk != 128 || dv != 128 || !kda::fused_available()) return KDA_ERR_UNSUPPORTED;
  const size_t need = kda_context_parallel_workspace_size(T, num_v_heads, dv);
  if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
    return KDA_ERR_WORKSPACE;
  __nv_bfloat16_raw* o_m = reinterpret_cast<__nv_bfloat16_raw*>(workspace);
  __nv_bfloat16_raw* o_u = o_m + (size_t)T * num_v_heads * dv;
  const int kp = choose_pieces(T, num_segments, num_v_heads);
  if (kp > 1 && workspace_bytes >= round256(need) + pieces_bytes(num_segments, kp, num_v_heads, dk, dv)) {
    // more chains than segments: every segment is built as kp chunk-aligned pieces, the scan
    // runs over the pieces, and each segment's summary is composed from its pieces'
    const int32_t np = num_segments * kp;
    uint8_t* w = reinterpret_cast<uint8_t*>(workspace) + round256(need);
    int32_t* sub = reinterpret_cast<int32_t*>(w);
    w += round256((size_t)(np + 1) * sizeof(int32_t));
    float* pM = reinterpret_cast<float*>(w);
    float* pU = pM + (size_t)np * num_v_heads * dk * dk;
    float* pIn = pU + (size_t)np * num_v_heads * dk * dv;
    const size_t blk = (size_t)num_v_heads * dk * dv;
    kda_status_t st = kda_context_parallel_piece_offsets(seg_offsets, num_segments, kp, sub, stream);
    if (st != KDA_OK) return st;
    st = kda_segment_summarize_and_scan(
        k, v, qkv_dtype, raw_gate, beta_logits, a_log, dt_bias, T, num_k_heads, num_v_heads, dk, dv, sub, np,
        initial_state, pM, pU, pIn, pIn + blk, final_state, q, o_m, o_u, flags | KDA_READOUT_HEAD_MAJOR,
        gate_lower_bound, nullptr, 0, device_status, stream);
    if (st != KDA_OK) return st;
    st = kda_segment_compose(pM, pU, pIn, final_state, num_segments, kp, num_v_heads, dk, dv, M, U, incoming,
                             outgoing, flags & KDA_STATE_V_FIRST, stream);
    if (st != KDA_OK) return st;
    return kda_context_parallel_apply(o_m, o_u, pIn, sub, np, T, num_v_heads, dv, out, out_dtype,
                                      (flags & KDA_STATE_V_FIRST) | KDA_READOUT_HEAD_MAJOR, device_status, stream);
  }
  // every segment in parallel (M_i, U_i and both readouts), then the exclusive scan
  kda_status_t st = kda_segment_summarize_and_scan(k, v, qkv_dtype, raw_gate, beta_logits, a_log, dt_bias, T,
                                                   num_k_heads, num_v_heads, dk, dv, seg_offsets, num_segments,
                                                   initial_state, M, U, incoming, outgoing, final_state, q, o_m,
                                                   o_u, flags | KDA_READOUT_HEAD_MAJOR, gate_lower_bound, nullptr, 0,
                                                   device_status, stream);
  if (st != KDA_OK) return st;
  // the incoming state's share added to the readouts
  return kda_context_parallel_apply(o_m, o_u, incoming, seg_offsets, num_segments, T, num_v_heads, dv, out,
                                    out_dtype, (flags & KDA_STATE_V_FIRST) | KDA_READOUT_HEAD_MAJOR, device_status,
                                    stream);
}

// ------------------------------------------------------------------------------------------
// Context parallelism across GPUs: each rank holds one range of consecutive segments of the
// sequence.  The range is built as pieces (with readouts) and composed into one summary; the
// summaries are exchanged and scanned by the caller; the range is then finished from the state
// entering it.  The workspace carries the readouts and the pieces' summaries between the two
// calls.
// ------------------------------------------------------------------------------------------
namespace {

struct RangeWorkspace {
  __nv_bfloat16_raw* o_m;  // [T][Hv][128] readout through the transition
  __nv_bfloat16_raw* o_u;  // [T][Hv][128] readout of the contribution
  int32_t* offs;           // [np + 1] piece boundaries
  float* pM;               // [np][Hv][128][128]
  float* pU;               // [np][Hv][state]
  float* pIn;              // [np + 1][Hv][state]: slot p + 1 holds the outgoing state of piece p
  int32_t np;
};

size_t range_workspace_bytes(int64_t T, int32_t N, int32_t Hv, int kp) {
  return round256((size_t)2 * T * Hv * 128 * 2) + pieces_bytes(N, kp, Hv, 128, 128);
}

RangeWorkspace range_workspace(void* ws, int64_t T, int32_t N, int32_t Hv, int kp) {
  RangeWorkspace r{};
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  r.np = N * kp;
  r.o_m = reinterpret_cast<__nv_bfloat16_raw*>(w);
  r.o_u = r.o_m + (size_t)T * Hv * 128;
  w += round256((size_t)2 * T * Hv * 128 * 2);
  r.offs = reinterpret_cast<int32_t*>(w);
  w += round256((size_t)(r.np + 1) * sizeof(int32_t));
  r.pM = reinterpret_cast<float*>(w);
  r.pU = r.pM + (size_t)r.np * Hv * 128 * 128;
  r.pIn = r.pU + (size_t)r.np * Hv * 128 * 128;
  return r;
}

bool range_workspace_ok(const void* ws, size_t bytes, int64_t T, int32_t N, int32_t Hv, int kp) {
  return ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0 && bytes >= range_workspace_bytes(T, N, Hv, kp);
}

}  // namespace

extern "C" size_t kda_context_parallel_range_workspace_size(int64_t T, int32_t num_segments, int32_t num_v_heads,
                                                            int32_t dv) {
  if (T < 0 || num_segments < 1 || num_v_heads <= 0 || dv != 128) return 0;
  if (T > INT32_MAX) return SIZE_MAX;
  return range_workspace_bytes(T, num_segments, num_v_heads, choose_pieces(T, num_segments, num_v_heads));
}

extern "C" kda_status_t kda_context_parallel_range_summary(
    const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype, const float* raw_gate,
    const float* beta_logits, const float* a_log, const float* dt_bias, int64_t T, int32_t num_k_heads,
    int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t* seg_offsets, int32_t num_segments,
    float* range_M, float* range_U, uint32_t flags, float gate_lower_bound, void* workspace,
    size_t workspace_bytes, int32_t* device_status, void* stream) {
  if (num_segments < 1 || T < 0 || T > INT32_MAX || num_k_heads <= 0 || num_v_heads <= 0 || dk <= 0 || dv <= 0)
    return KDA_ERR_INVALID_ARG;
  if (num_v_heads % num_k_heads != 0) return KDA_ERR_INVALID_ARG;
  if ((flags & ~kKnownFlags) != 0 || (flags & (KDA_SEG_SCAN_ONLY | KDA_FORCE_SIMT))) return KDA_ERR_INVALID_ARG;
  if (T > 0 && (!q || !k || !v || !raw_gate || !beta_logits)) return KDA_ERR_INVALID_ARG;
  if (!a_log || !dt_bias || !seg_offsets || !range_M || !range_U) return KDA_ERR_INVALID_ARG;
  if (!dtype_ok(qkv_dtype)) return KDA_ERR_UNSUPPORTED;
  if (qkv_dtype != KDA_BF16 || dk != 128 || dv != 128 || !kda::fused_available()) return KDA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(raw_gate) || !aligned16(dt_bias) ||
      !aligned16(range_M) || !aligned16(range_U))
    return KDA_ERR_INVALID_ARG;
  const int kp = choose_pieces(T, num_segments, num_v_heads);
  if (!range_workspace_ok(workspace, workspace_bytes, T, num_segments, num_v_heads, kp)) return KDA_ERR_WORKSPACE;
  const RangeWorkspace L = range_workspace(workspace, T, num_segments, num_v_heads, kp);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (kda::launch_split_offsets(seg_offsets, num_segments, kp, L.offs, s) != cudaSuccess) return KDA_ERR_CUDA;
  // the pieces in parallel: transition, contribution and both readouts in one launch
  kda::FusedArgs f{};
  f.q = q;
  f.k = k;
  f.v = v;
  f.raw_gate = raw_gate;
  f.beta = beta_logits;
  f.a_log = a_log;
  f.dt_bias = dt_bias;
  f.cu = L.offs;
  f.batch = L.np;
  f.total_tokens = T;
  f.Hk = num_k_heads;
  f.Hv = num_v_heads;
  f.max_slots = L.np;
  f.out = L.o_m;
  f.out2 = L.o_u;
  f.out_bf16 = 1;
  f.readout_hm = 1;
  f.flags = flags;
  f.lb = gate_lower_bound;
  f.status = device_status;
  f.build = 1;
  f.state_out = L.pM;
  f.state_out2 = L.pU;
  f.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  if (kda::launch_fused_chunk(f, s) != cudaSuccess) return KDA_ERR_CUDA;
  // the whole range as one map: the pieces composed in order
  kda::ComposeArgs ca{};
  ca.M = L.pM;
  ca.U = L.pU;
  ca.inc = nullptr;
  ca.N = 1;
  ca.k = L.np;
  ca.H = num_v_heads;
  ca.dk = 128;
  ca.dv = 128;
  ca.v_first = f.v_first;
  ca.M_out = range_M;
  ca.U_out = range_U;
  return kda::launch_compose_pieces(ca, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_context_parallel_range_finish(
    int64_t T, int32_t num_v_heads, int32_t dk, int32_t dv, int32_t num_segments, const float* range_incoming,
    void* out, kda_dtype_t out_dtype, float* range_outgoing, float* M, float* U, float* incoming, float* outgoing,
    uint32_t flags, void* workspace, size_t workspace_bytes, int32_t* device_status, void* stream) {
  if (num_segments < 1 || T < 0 || T > INT32_MAX || num_v_heads <= 0 || dk <= 0 || dv <= 0)
    return KDA_ERR_INVALID_ARG;
  if ((flags & ~kKnownFlags) != 0) return KDA_ERR_INVALID_ARG;
  if (!range_incoming || !M || !U || !incoming || !outgoing || (T > 0 && !out)) return KDA_ERR_INVALID_ARG;
  if (!dtype_ok(out_dtype)) return KDA_ERR_UNSUPPORTED;
  if (dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
  if (!aligned16(out)) return KDA_ERR_INVALID_ARG;
  const int kp = choose_pieces(T, num_segments, num_v_heads);
  if (!range_workspace_ok(workspace, workspace_bytes, T, num_segments, num_v_heads, kp)) return KDA_ERR_WORKSPACE;
  const RangeWorkspace L = range_workspace(workspace, T, num_segments, num_v_heads, kp);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  const size_t blk = (size_t)num_v_heads * 128 * 128;
  // the incoming state of every piece, from the state entering the range
  kda::ScanArgs sa{};
  sa.M = L.pM;
  sa.U = L.pU;
  sa.initial = range_incoming;
  sa.N = L.np;
  sa.H = num_v_heads;
  sa.dk = 128;
  sa.dv = 128;
  sa.v_first = v_first;
  sa.incoming = L.pIn;
  sa.outgoing = L.pIn + blk;
  sa.final_state = range_outgoing;
  if (kda::launch_affine_scan(sa, s) != cudaSuccess) return KDA_ERR_CUDA;
  // each segment's summary and states from its pieces'
  kda::ComposeArgs ca{};
  ca.M = L.pM;
  ca.U = L.pU;
  ca.inc = L.pIn;
  ca.final_state = L.pIn + (size_t)L.np * blk;
  ca.N = num_segments;
  ca.k = kp;
  ca.H = num_v_heads;
  ca.dk = 128;
  ca.dv = 128;
  ca.v_first = v_first;
  ca.M_out = M;
  ca.U_out = U;
  ca.incoming = incoming;
  ca.outgoing = outgoing;
  if (kda::launch_compose_pieces(ca, s) != cudaSuccess) return KDA_ERR_CUDA;
  // the outputs: every piece's readouts with its incoming state
  kda::ApplyArgs ap{};
  ap.seg_offsets = L.offs;
  ap.num_segments = L.np;
  ap.total_tokens = T;
  ap.Hv = num_v_heads;
  ap.incoming = L.pIn;
  ap.v_first = v_first;
  ap.o_m = L.o_m;
  ap.o_u = L.o_u;
  ap.readout_hm = 1;
  ap.out = out;
  ap.out_bf16 = out_dtype == KDA_BF16;
  ap.status = device_status;
  return kda::launch_cp_apply(ap, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" size_t kda_workspace_size(int64_t total_tokens, int32_t batch, int32_t num_k_heads,
                                     int32_t num_v_heads, int32_t dk, int32_t dv, int32_t num_segments,
                                     uint32_t flags) {
  (void)num_k_heads;
  (void)num_segments;
  // the split route of kda_chunk_fwd (bf16 fast path only; unused otherwise)
  if (dk != 128 || dv != 128 || (flags & KDA_FORCE_SIMT) || total_tokens < 0 || batch <= 0 || num_v_heads <= 0)
    return 0;
  const int P = choose_piece_len(total_tokens, batch, num_v_heads);
  return P > 0 ? split_bytes(total_tokens, batch, num_v_heads, P) : 0;
}

extern "C" const char* kda_status_string(kda_status_t status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null pointer, bad extent or bad flags";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: dtype grouping or head dims bind no kernel";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA runtime call failed";
    case KDA_ERR_DEVICE_CHECK: return "KDA_ERR_DEVICE_CHECK: bad state slot or decreasing offsets";
    case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
  }
  return "KDA_ERR_UNKNOWN";
}

extern "C" int32_t kda_version(void) { return 100; }
