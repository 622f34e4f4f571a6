// kda_common.cuh -- small device helpers shared by the KDA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

__device__ __forceinline__ float load_in(const void* p, size_t idx, int is_bf16) {
  if (is_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[idx]);
  return reinterpret_cast<const float*>(p)[idx];
}

__device__ __forceinline__ void store_out(void* p, size_t idx, float x, int is_bf16) {
  if (is_bf16) reinterpret_cast<__nv_bfloat16*>(p)[idx] = __float2bfloat16_rn(x);
  else reinterpret_cast<float*>(p)[idx] = x;
}

// First device-side finding wins; later ones are dropped.
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Forget gate of one (token, head, channel):
//   g = -exp(a_log) * softplus(raw + dt_bias), clamped below at lb in "safe" mode
// ("max.nn.state_space.kda_chunk", Parameters: raw_gate is the pre-activation before dt_bias;
// gate_mode "safe" names a lower bound -- read here as a clamp).
__device__ __forceinline__ float gate_f32(float raw, float a_log, float dt_bias, bool safe, float lb) {
  float x = raw + dt_bias;
  float sp = fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
  float g = -expf(a_log) * sp;
  return safe ? fmaxf(g, lb) : g;
}

__device__ __forceinline__ float beta_f32(float x, bool prob) {
  return prob ? x : 1.0f / (1.0f + expf(-x));
}

// Offset of element (i, j) of a dk x w state block: K_FIRST stores [dk][w], V_FIRST [w][dk].
__device__ __forceinline__ size_t state_off(int i, int j, int dk, int w, int v_first) {
  return v_first ? (size_t)j * dk + i : (size_t)i * w + j;
}

}  // namespace kda
