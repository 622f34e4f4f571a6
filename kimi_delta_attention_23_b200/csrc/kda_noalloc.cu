// kda_noalloc.cu -- the context-parallel prefill without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they run the prefill: a host
// program whose device memory is owned by another component's pool (and which may not call
// cudaMalloc behind that pool's back), or a serving loop that must not allocate while
// requests are in flight, because cudaMalloc/cudaFree can synchronise the device and stall
// every stream.  For them this file keeps the prefill's scratch (the two per-token readouts)
// in a fixed array in device memory that the library itself carries.
//
// The array is a file-scope __device__ variable: every GPU that loads this library holds its
// kStaticScratchBytes until the process exits.  Host code cannot use the array's name as a
// device address (on the host it names a stand-in object), so the entry point looks the
// address up with cudaGetSymbolAddress, once per device, with that device current, and passes
// the pointer to the kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kda.h"

namespace {

// 32 MiB: two bf16 readouts of 128 values per token-head, i.e. up to 65536 token-heads
// (for example 2048 tokens x 32 heads, or 4096 tokens x 16 heads) per call.
constexpr size_t kStaticScratchBytes = (size_t)32 << 20;

__device__ __align__(256) unsigned char g_cp_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_cp_scratch on the current device (looked up on the first call per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_cp_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" kda_status_t kda_context_parallel_prefill_static(
    const void* q, const void* k, const void* v, kda_dtype_t qkv_dtype, const float* raw_gate,
    const float* beta_logits, const float* a_log, const float* dt_bias, int64_t T, int32_t num_k_heads,
    int32_t num_v_heads, int32_t dk, int32_t dv, const int32_t* seg_offsets, int32_t num_segments,
    const float* initial_state, void* out, kda_dtype_t out_dtype, float* final_state, float* M, float* U,
    float* incoming, float* outgoing, uint32_t flags, float gate_lower_bound, int32_t* device_status,
    void* stream) {
  // token offsets are int32; checked before the size, whose product would be meaningless beyond
  if (T < 0 || T > INT32_MAX || num_v_heads <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
  const size_t need = kda_context_parallel_workspace_size(T, num_v_heads, dv);
  if (need > kStaticScratchBytes) return KDA_ERR_WORKSPACE;  // beyond the fixed scratch: refuse
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
  return kda_context_parallel_prefill(q, k, v, qkv_dtype, raw_gate, beta_logits, a_log, dt_bias, T, num_k_heads,
                                      num_v_heads, dk, dv, seg_offsets, num_segments, initial_state, out, out_dtype,
                                      final_state, M, U, incoming, outgoing, flags, gate_lower_bound, scratch,
                                      kStaticScratchBytes, device_status, stream);
}
