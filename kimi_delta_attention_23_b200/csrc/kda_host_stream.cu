// kda_host_stream.cu -- the prefill of ONE sequence whose inputs and outputs are in (pinned)
// host memory, pipelined in segments so the copies over the host link overlap each other and
// the kernels.
//
// The step is the chunk-parallel prefill ("max.nn.state_space.kda_chunk": the recurrence
// evaluated over 64-token chunks, the state carried from chunk to chunk): segment i's inputs
// are copied in on one stream while segment i - 1 runs on the caller's stream and segment
// i - 2's outputs are copied out on a third, so the link carries both directions at once and the
// kernels hide under the copies.  Segments are cut at multiples of 64 tokens, so every chunk
// is the chunk of the unsegmented pass and the fp32 state passes from segment to segment
// through memory unchanged: the result is kda_chunk_fwd's on the whole sequence, bit for bit.
#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace kda {
namespace {

__global__ void even_offsets_kernel(int32_t* offs, int32_t n, int64_t seg, int64_t T) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i <= n) {
    const int64_t t = (int64_t)i * seg;
    offs[i] = (int32_t)(t < T ? t : T);
  }
}

// helper streams and events, created once per device on first use and kept for the process
struct Pipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in = nullptr, out = nullptr, done = nullptr;
  bool ready = false;
};
constexpr int kMaxDevices = 64;
Pipe g_pipe[kMaxDevices];
std::mutex g_mu;  // one enqueue sequence at a time (the events are reused)

cudaError_t pipe_for(int dev, Pipe** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  Pipe& p = g_pipe[dev];
  if (!p.ready) {
    cudaError_t e;
    if ((e = cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
    for (cudaEvent_t* ev : {&p.start, &p.in, &p.out, &p.done})
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    p.ready = true;
  }
  *out = &p;
  return cudaSuccess;
}

size_t r256(size_t n) { return (n + 255) & ~size_t(255); }

// device staging: the whole sequence's inputs and outputs, the parameters, the state and the
// segment offsets, each 256-byte aligned
struct HostLayout {
  size_t q, k, v, raw, beta, alog, dtb, state, out, offs, total;
};
HostLayout host_layout(int64_t T, int32_t Hk, int32_t Hv, int out_es, int32_t nseg) {
  HostLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += r256(bytes);
    return at;
  };
  L.q = take((size_t)T * Hk * 128 * 2);
  L.k = take((size_t)T * Hk * 128 * 2);
  L.v = take((size_t)T * Hv * 128 * 2);
  L.raw = take((size_t)T * Hv * 128 * 4);
  L.beta = take((size_t)T * Hv * 4);
  L.alog = take((size_t)Hv * 4);
  L.dtb = take((size_t)Hv * 128 * 4);
  L.state = take((size_t)Hv * 128 * 128 * 4);
  L.out = take((size_t)T * Hv * 128 * out_es);
  L.offs = take(((size_t)nseg + 1) * 4);
  L.total = o;
  return L;
}

int32_t num_segments(int64_t T, int64_t seg) { return T == 0 ? 1 : (int32_t)((T + seg - 1) / seg); }

}  // namespace

bool fused_available();
cudaError_t launch_fused_chunk(const FusedArgs& a, cudaStream_t stream);

}  // namespace kda

extern "C" size_t kda_prefill_host_workspace_size(int64_t T, int32_t num_k_heads, int32_t num_v_heads,
                                                   kda_dtype_t out_dtype, int64_t segment_tokens) {
  if (T < 0 || num_k_heads <= 0 || num_v_heads <= 0 || segment_tokens <= 0 || segment_tokens % 64 != 0) return 0;
  if (T / segment_tokens > (int64_t)1 << 30) return 0;
  return kda::host_layout(T, num_k_heads, num_v_heads, out_dtype == KDA_BF16 ? 2 : 4,
                          kda::num_segments(T, segment_tokens))
      .total;
}

extern "C" kda_status_t kda_prefill_host_pipelined(
    const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype, const float* raw_gate,
    const float* beta_logits, const float* a_log, const float* dt_bias, int64_t T, int32_t num_k_heads,
    int32_t num_v_heads, int32_t dk, int32_t dv, const float* initial_state, void* out, kda_dtype_t out_dtype,
    float* final_state, int64_t segment_tokens, uint32_t flags, float gate_lower_bound, void* workspace,
    size_t workspace_bytes, int32_t* device_status, void* stream) {
  constexpr uint32_t kAllowed = KDA_GATE_SAFE | KDA_BETA_PROB | KDA_STATE_V_FIRST | KDA_FUSED;
  if (T < 0 || num_k_heads <= 0 || num_v_heads <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
  if (num_v_heads % num_k_heads != 0 || (flags & ~kAllowed) != 0) return KDA_ERR_INVALID_ARG;
  if (segment_tokens <= 0 || segment_tokens % 64 != 0) return KDA_ERR_INVALID_ARG;
  if (!a_log || !dt_bias || !initial_state || !final_state) return KDA_ERR_INVALID_ARG;
  if (T > 0 && (!q || !k || !v || !raw_gate || !beta_logits || !out)) return KDA_ERR_INVALID_ARG;
  if ((qkv_dtype != KDA_F32 && qkv_dtype != KDA_BF16) || (out_dtype != KDA_F32 && out_dtype != KDA_BF16))
    return KDA_ERR_UNSUPPORTED;
  if (qkv_dtype != KDA_BF16 || dk != 128 || dv != 128 || !kda::fused_available()) return KDA_ERR_UNSUPPORTED;
  if (T > INT32_MAX) return KDA_ERR_INVALID_ARG;  // token offsets are int32, as cu_seqlens
  const int out_es = out_dtype == KDA_BF16 ? 2 : 4;
  const int32_t nseg = kda::num_segments(T, segment_tokens);
  const kda::HostLayout L = kda::host_layout(T, num_k_heads, num_v_heads, out_es, nseg);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KDA_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(kda::g_mu);
  kda::Pipe* p = nullptr;
  if (kda::pipe_for(dev, &p) != cudaSuccess) return KDA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = reinterpret_cast<uint8_t*>(workspace);
  const int32_t Hk = num_k_heads, Hv = num_v_heads;
  const size_t st_bytes = (size_t)Hv * 128 * 128 * 4;
  bool ok = true;
  auto chk = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
  auto h2d = [&](size_t off, const void* src, size_t bytes) {
    if (bytes) chk(cudaMemcpyAsync(w + off, src, bytes, cudaMemcpyHostToDevice, p->h2d));
  };

  // the helper streams start after the work already queued on the caller's stream
  chk(cudaEventRecord(p->start, s));
  chk(cudaStreamWaitEvent(p->h2d, p->start, 0));
  chk(cudaStreamWaitEvent(p->d2h, p->start, 0));
  // parameters, the initial state, then the offsets (computed on the device)
  h2d(L.alog, a_log, (size_t)Hv * 4);
  h2d(L.dtb, dt_bias, (size_t)Hv * 128 * 4);
  h2d(L.state, initial_state, st_bytes);
  int32_t* offs = reinterpret_cast<int32_t*>(w + L.offs);
  kda::even_offsets_kernel<<<(nseg + 1 + 255) / 256, 256, 0, s>>>(offs, nseg, segment_tokens, T);
  chk(cudaGetLastError());

  kda::FusedArgs f{};
  f.q = w + L.q;
  f.k = w + L.k;
  f.v = w + L.v;
  f.raw_gate = reinterpret_cast<const float*>(w + L.raw);
  f.beta = reinterpret_cast<const float*>(w + L.beta);
  f.a_log = reinterpret_cast<const float*>(w + L.alog);
  f.dt_bias = reinterpret_cast<const float*>(w + L.dtb);
  f.batch = 1;
  f.total_tokens = T;
  f.Hk = Hk;
  f.Hv = Hv;
  f.state_in = reinterpret_cast<const float*>(w + L.state);
  f.state_out = reinterpret_cast<float*>(w + L.state);
  f.max_slots = 1;
  f.slots = nullptr;
  f.v_first = (flags & KDA_STATE_V_FIRST) ? 1 : 0;
  f.init_mode = 0;
  f.values_zero = 0;
  f.out = w + L.out;
  f.out_bf16 = out_dtype == KDA_BF16;
  f.flags = flags;
  f.lb = gate_lower_bound;
  f.status = device_status;

  for (int32_t i = 0; i < nseg && ok; ++i) {
    const int64_t s0 = (int64_t)i * segment_tokens;
    const int64_t n = (s0 + segment_tokens < T ? s0 + segment_tokens : T) - s0;
    // segment i in ...
    h2d(L.q + (size_t)s0 * Hk * 256, static_cast<const uint8_t*>(q) + (size_t)s0 * Hk * 256, (size_t)n * Hk * 256);
    h2d(L.k + (size_t)s0 * Hk * 256, static_cast<const uint8_t*>(k) + (size_t)s0 * Hk * 256, (size_t)n * Hk * 256);
    h2d(L.v + (size_t)s0 * Hv * 256, static_cast<const uint8_t*>(v) + (size_t)s0 * Hv * 256, (size_t)n * Hv * 256);
    h2d(L.raw + (size_t)s0 * Hv * 512, reinterpret_cast<const uint8_t*>(raw_gate) + (size_t)s0 * Hv * 512,
        (size_t)n * Hv * 512);
    h2d(L.beta + (size_t)s0 * Hv * 4, reinterpret_cast<const uint8_t*>(beta_logits) + (size_t)s0 * Hv * 4,
        (size_t)n * Hv * 4);
    chk(cudaEventRecord(p->in, p->h2d));
    // ... run from the state the previous segment left ...
    chk(cudaStreamWaitEvent(s, p->in, 0));
    f.cu = offs + i;
    chk(kda::launch_fused_chunk(f, s));
    chk(cudaEventRecord(p->out, s));
    // ... and out
    chk(cudaStreamWaitEvent(p->d2h, p->out, 0));
    if (n > 0)
      chk(cudaMemcpyAsync(static_cast<uint8_t*>(out) + (size_t)s0 * Hv * 128 * out_es,
                          w + L.out + (size_t)s0 * Hv * 128 * out_es, (size_t)n * Hv * 128 * out_es,
                          cudaMemcpyDeviceToHost, p->d2h));
  }
  // the final state once the last segment ran (its event was the last the copy-out stream waited on)
  if (ok) chk(cudaMemcpyAsync(final_state, w + L.state, st_bytes, cudaMemcpyDeviceToHost, p->d2h));
  // the caller's stream completes after the last copy
  chk(cudaEventRecord(p->done, p->d2h));
  chk(cudaStreamWaitEvent(s, p->done, 0));
  return ok ? KDA_OK : KDA_ERR_CUDA;
}
