// kda_internal.h -- launch arguments and launchers shared between the C-ABI layer and kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

// fp32 CUDA-core chunk kernel.  One block per (sequence, value head).
struct SimtArgs {
  const void* q;
  const void* k;
  const void* v;
  int32_t in_bf16;
  const float* raw_gate;
  const float* beta;
  const float* a_log;
  const float* dt_bias;
  const int32_t* cu;        // [batch+1]
  int32_t batch;
  int64_t total_tokens;
  int32_t Hk, Hv, dk;
  int32_t w;                // state width (value columns carried by the state)
  int32_t dv_in;            // row length of v
  const float* state_in;    // read when init_mode == 0
  float* state_out;         // final state destination (may equal state_in)
  int32_t max_slots;
  const int32_t* slots;     // [batch] or NULL (slot = sequence index)
  int32_t v_first;          // state blocks stored transposed ([w][dk])
  int32_t init_mode;        // 0: state_in slot, 1: zero, 2: identity
  int32_t values_zero;      // 1: all values are zero (transition build)
  void* out;                // [T,Hv,w] or NULL
  int32_t out_bf16;
  uint32_t flags;
  float lb;
  int32_t* status;
};

struct ScanArgs {
  const float* M;
  const float* U;
  const float* initial;
  int32_t N, H, dk, dv, v_first;
  float* incoming;
  float* outgoing;
  float* final_state;
};

// One level of the log-depth scan over the maps' prefixes.
struct ScanLevelArgs {
  const float* M;   // [N][H][128][128] the level's input prefixes (row-major)
  const float* U;   // [N][H][state]
  float* M_out;     // the level's output prefixes
  float* U_out;
  int32_t N, H, dv, v_first, stride;
};

// Fused tensor-core chunk kernel (bf16 q/k/v, dk = dv = 128).
struct FusedArgs {
  const void* q;            // bf16 [T,Hk,128]
  const void* k;            // bf16 [T,Hk,128]
  const void* v;            // bf16 [T,Hv,128]
  const float* raw_gate;
  const float* beta;
  const float* a_log;
  const float* dt_bias;
  const int32_t* cu;
  int32_t batch;
  int64_t total_tokens;
  int32_t Hk, Hv;
  const float* state_in;    // read when init_mode == 0 (pool base)
  float* state_out;         // final state destination (pool base; may equal state_in); with
                            // build: the transitions M [N][Hv][128][128]
  float* state_out2;        // build only: the contributions U [N][Hv][128][128] (layout v_first)
  int32_t build;            // 1: segment build -- transition (from I, zero values) and contribution
                            // (from 0, real values) carried together, no readout
  int32_t max_slots;
  const int32_t* slots;     // [batch] or NULL (slot = sequence index)
  int32_t v_first;          // state blocks stored transposed ([dv][dk])
  int32_t init_mode;        // 0: state_in slot, 1: zero, 2: identity
  int32_t values_zero;      // 1: all values are zero (transition build)
  void* out;                // [T,Hv,128] or NULL (no readout); with build: readout of the transition
  void* out2;               // build only: readout of the contribution [T,Hv,128] bf16 (or NULL)
  int32_t readout_hm;       // build only: both readouts stored [Hv][T][128] instead
  int32_t out_bf16;
  uint32_t flags;
  float lb;
  int32_t* status;
  // launch gate (nullable): the kernel runs only if *gate_flag == gate_run_if
  const int32_t* gate_flag;
  int32_t gate_run_if;
};

// Context-parallel prefill, last step: out = O_M . S_in(segment) + O_U.
struct ApplyArgs {
  const int32_t* seg_offsets;  // [N+1]
  int32_t num_segments;
  int64_t total_tokens;
  int32_t Hv;
  const float* incoming;       // [N][Hv][128][128] in the state layout
  int32_t v_first;
  const void* o_m;             // bf16 [T][Hv][128] readout through the transition
  const void* o_u;             // bf16 [T][Hv][128] readout of the contribution
  int32_t readout_hm;          // both readouts stored [Hv][T][128] instead
  void* out;                   // [T][Hv][128]
  int32_t out_bf16;
  int32_t* status;
  const int32_t* skip_flag;  // nullable: the kernel does nothing if *skip_flag != 0
};

// A varlen batch cut into pieces of at most piece_len tokens (chunk-aligned, at least one per
// sequence): piece boundaries and each sequence's first piece, or the fallback flag (1) when an
// offset or a slot is out of range or the pieces would not shorten the schedule (the plain
// kernel then handles the batch).
struct PlanArgs {
  const int32_t* cu;
  const int32_t* slots;  // nullable: sequence b uses slot b
  int32_t batch;
  int64_t total_tokens;
  int32_t max_slots;
  int32_t piece_len;
  int32_t max_pieces;
  int32_t num_heads;     // value heads (chains per piece)
  int32_t num_sms;       // SMs of the device (one chain each at a time)
  int32_t* piece_offs;   // [max_pieces + 1]
  int32_t* seq_first;    // [batch + 1]
  int32_t* fallback;     // [1]
};

// The pieces' summaries applied in order from each sequence's pool slot (dk = 128): the
// incoming state of every piece, and the final state written back to the slot.
struct PoolScanArgs {
  const float* M;        // [pieces][H][128][128]
  const float* U;        // [pieces][H][state]
  const int32_t* seq_first;
  const int32_t* slots;  // nullable
  const int32_t* fallback;
  int32_t batch, H, dv, v_first;
  float* pool;           // [slots][H][state]
  float* incoming;       // [pieces][H][state]
};

// Summaries of segments split into k pieces each, rebuilt from the pieces' summaries.
struct ComposeArgs {
  const float* M;            // [N*k][H][dk][dk] the pieces' transitions (row-major)
  const float* U;            // [N*k][H][state] the pieces' contributions
  const float* inc;          // [N*k][H][state] the pieces' incoming states, or NULL (then
                             // final_state, incoming and outgoing are unused)
  const float* final_state;  // [H][state]
  int32_t N, k, H, dk, dv, v_first;
  float* M_out;              // [N][H][dk][dk]
  float* U_out;              // [N][H][state]
  float* incoming;           // [N][H][state]
  float* outgoing;           // [N][H][state]
};

// Single-token step of a batch of sequences (one token each), in place on the pool.
struct DecodeArgs {
  const void* q;            // [batch,Hk,dk]
  const void* k;            // [batch,Hk,dk]
  const void* v;            // [batch,Hv,dv]
  int32_t in_bf16;
  const float* raw_gate;    // [batch,Hv,dk]
  const float* beta;        // [batch,Hv]
  const float* a_log;       // [Hv]
  const float* dt_bias;     // [Hv,dk]
  int32_t batch;
  int32_t Hk, Hv, dk, dv;
  float* pool;              // [max_slots][Hv][dk][dv] (K_FIRST) or [..][dv][dk] (V_FIRST)
  int32_t max_slots;
  const int32_t* slots;     // [batch]
  int32_t v_first;
  void* out;                // [batch,Hv,dv]
  int32_t out_bf16;
  uint32_t flags;
  float lb;
  int32_t* status;
};

size_t simt_smem_bytes(int dk, int w);
cudaError_t launch_split_offsets(const int32_t* offs, int32_t N, int32_t k, int32_t* sub, cudaStream_t stream);
cudaError_t launch_compose_pieces(const ComposeArgs& a, cudaStream_t stream);
cudaError_t launch_plan_pieces(const PlanArgs& a, cudaStream_t stream);
cudaError_t launch_pool_scan(const PoolScanArgs& a, cudaStream_t stream);
cudaError_t launch_cp_apply(const ApplyArgs& a, cudaStream_t stream);
cudaError_t launch_simt_chunk(const SimtArgs& a, cudaStream_t stream);
cudaError_t launch_affine_scan(const ScanArgs& a, cudaStream_t stream);
// the log-depth form (dk = 128, dv a multiple of 32 up to 128); `work` holds
// logdepth_scan_bytes(N, H, dk, dv) bytes
size_t logdepth_scan_bytes(int N, int H, int dk, int dv);
bool logdepth_scan_preferred(int N, int H, int dv);
cudaError_t launch_affine_scan_logdepth(const ScanArgs& a, float* work, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

}  // namespace kda
