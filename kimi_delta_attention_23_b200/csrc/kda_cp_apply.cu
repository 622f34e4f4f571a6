// kda_cp_apply.cu -- last step of the context-parallel prefill: every token's output from the
// local readouts of its segment and the segment's incoming state.
//
// Inside a segment the state after token t is S_t = M_{<=t} S_in + U_{<=t} (the segment's map
// applied to its incoming state -- "KDA Context Parallelism", Theory: a segment can be applied
// to any incoming state without replaying its tokens), so the readout is affine in S_in:
//     o_t = (q_t^T M_{<=t}) S_in + q_t^T U_{<=t} = O_M[t] . S_in + O_U[t].
// The segment-build pass writes O_M and O_U; this kernel adds the incoming state's share.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 256;
constexpr int kTile = 64;   // tokens per tile
constexpr int kLd = 136;    // padded row length (bf16) of the staged tiles: conflict-free ldmatrix

}  // namespace

// One block per (value head, segment); the incoming state stays in shared memory (bf16, as the
// B operand) while the block walks the segment in 64-token tiles.  Warp w computes rows
// 16 (w % 4) .. +16 and columns 64 (w / 4) .. +64 of each tile.
__global__ void __launch_bounds__(kThreads) cp_apply_kernel(ApplyArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sB = reinterpret_cast<__nv_bfloat16*>(smem);  // [j][j'] = S_in[j'][j]
  __nv_bfloat16* sA = sB + D * kLd;                              // [r][j'] = O_M[t0 + r][j']
  const int h = blockIdx.x, seg = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t s0 = a.seg_offsets[seg], s1 = a.seg_offsets[seg + 1];
  if (s0 < 0 || s1 < s0 || s1 > a.total_tokens) {
    if (tid == 0) report(a.status, KDA_ERR_DEVICE_CHECK);
    return;
  }
  const float* S = a.incoming + ((size_t)seg * a.Hv + h) * (size_t)(D * D);
  for (int e = tid; e < D * D; e += kThreads) {
    const int jp = a.v_first ? e % D : e / D, j = a.v_first ? e / D : e % D;
    sB[j * kLd + jp] = __float2bfloat16_rn(S[e]);
  }
  const int g = lane >> 2, t = lane & 3, m = lane >> 3;
  const int r0 = 16 * (warp & 3), n0 = 64 * (warp >> 2);
  const uint32_t sA_addr = smem_addr(sA), sB_addr = smem_addr(sB);
  const __nv_bfloat16* om = reinterpret_cast<const __nv_bfloat16*>(a.o_m);
  const __nv_bfloat16* ou = reinterpret_cast<const __nv_bfloat16*>(a.o_u);
#pragma unroll 1
  for (int64_t c0 = s0; c0 < s1; c0 += kTile) {
    const int L = (int)((s1 - c0) < kTile ? (s1 - c0) : kTile);
    __syncthreads();  // the previous tile's reads of sA are done (and sB is in place)
    for (int e = tid; e < kTile * 16; e += kThreads) {
      const int r = e >> 4, c = e & 15;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (r < L) val = *reinterpret_cast<const uint4*>(om + ((size_t)(c0 + r) * a.Hv + h) * D + c * 8);
      *reinterpret_cast<uint4*>(sA + r * kLd + c * 8) = val;
    }
    __syncthreads();
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[nt][u] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a0, a1, a2, a3;
      const int ar = r0 + (m & 1) * 8 + (lane & 7), ak = 16 * kk + (m >> 1) * 8;
      ldsm_x4(sA_addr + (ar * kLd + ak) * 2, a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b00, b01, b10, b11;
        const int br = n0 + 16 * np + (m >> 1) * 8 + (lane & 7), bk = 16 * kk + (m & 1) * 8;
        ldsm_x4(sB_addr + (br * kLd + bk) * 2, b00, b01, b10, b11);
        mma16816(acc[2 * np], a0, a1, a2, a3, b00, b01);
        mma16816(acc[2 * np + 1], a0, a1, a2, a3, b10, b11);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = r0 + g + 8 * hh;
        if (r >= L) continue;
        const int j = n0 + 8 * nt + 2 * t;
        const size_t o = ((size_t)(c0 + r) * a.Hv + h) * D + j;
        const float2 u = unpack_bf16(*reinterpret_cast<const uint32_t*>(ou + o));
        const float x0 = acc[nt][2 * hh] + u.x, x1 = acc[nt][2 * hh + 1] + u.y;
        if (a.out_bf16)
          *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(a.out) + o) = pack_bf16(x0, x1);
        else
          *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + o) = make_float2(x0, x1);
      }
    }
  }
}

cudaError_t launch_cp_apply(const ApplyArgs& a, cudaStream_t stream) {
  const int smem = (D + kTile) * kLd * 2;
  cudaError_t err = cudaFuncSetAttribute(cp_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  dim3 grid(a.Hv, a.num_segments);
  cp_apply_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
