// kda_fused.cu -- fused tensor-core chunk kernel (bf16 q/k/v, dk = dv = 128).
#include "kda_internal.h"

namespace kda {

bool fused_available() { return false; }

cudaError_t launch_fused_chunk(const FusedArgs& a, cudaStream_t stream) {
  (void)a;
  (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace kda
