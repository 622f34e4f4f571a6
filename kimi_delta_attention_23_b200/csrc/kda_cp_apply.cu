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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  // 16-byte global -> shared copy; rows past the segment read zeros (src-size 0)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The work is the flat list of 64-token tiles ordered by (segment, value head, tile); a
// persistent grid of two blocks per SM splits it into equal contiguous ranges, so a block
// touches only one or two (segment, head) pairs and loads each pair's incoming state once
// (bf16, as the B operand).  The next tile's two readout tiles are copied asynchronously while
// the current one is multiplied; warp w computes rows 32 (w % 2) .. +32 and columns
// 32 (w / 2) .. +32 of a tile -- its share of the incoming state stays in registers as B
// fragments for all tiles of a pair -- and adds the contribution readout.  A bf16 result overwrites the
// contribution tile in place (each thread rewrites exactly the elements it read) and leaves in
// 16-byte row stores.
struct TilePos {
  int seg, h, tile;
};

__global__ void __launch_bounds__(kThreads, 2) cp_apply_kernel(ApplyArgs a) {
  if (a.skip_flag && *a.skip_flag) return;
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sB = reinterpret_cast<__nv_bfloat16*>(smem);  // [j][j'] = S_in[j'][j]
  __nv_bfloat16* sM = sB + D * kLd;                              // 2 x [r][j'] readout through M
  __nv_bfloat16* sU = sM + 2 * kTile * kLd;                      // 2 x [r][j]  contribution readout
  __shared__ int64_t s_range[2];
  __shared__ int s_pos[3];
  __shared__ int s_bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.num_segments, Hv = a.Hv;
  const int32_t* offs = a.seg_offsets;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int i = tid; i < N; i += kThreads) {
    const int64_t b = offs[i], e = offs[i + 1];
    if (b < 0 || e < b || e > a.total_tokens) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) report(a.status, KDA_ERR_DEVICE_CHECK);
    return;
  }
  auto ntiles = [&](int seg) { return (int)((offs[seg + 1] - offs[seg] + kTile - 1) / kTile); };
  if (tid == 0) {
    int64_t total = 0;
    for (int i = 0; i < N; ++i) total += (int64_t)ntiles(i) * Hv;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t first = per * blockIdx.x, last = first + per < total ? first + per : total;
    s_range[0] = first;
    s_range[1] = last;
    int64_t before = 0;  // tiles of the segments before seg
    int seg = 0;
    while (seg < N && before + (int64_t)ntiles(seg) * Hv <= first) before += (int64_t)ntiles(seg++) * Hv;
    int h = 0, tile = 0;
    if (seg < N) {
      const int nt = ntiles(seg);
      h = (int)((first - before) / nt);
      tile = (int)((first - before) % nt);
    }
    s_pos[0] = seg;
    s_pos[1] = h;
    s_pos[2] = tile;
  }
  __syncthreads();
  const int64_t count = s_range[1] - s_range[0];
  if (count <= 0) return;
  const __nv_bfloat16* om = reinterpret_cast<const __nv_bfloat16*>(a.o_m);
  const __nv_bfloat16* ou = reinterpret_cast<const __nv_bfloat16*>(a.o_u);
  const uint32_t sM_addr = smem_addr(sM), sU_addr = smem_addr(sU), sB_addr = smem_addr(sB);
  auto advance = [&](TilePos p) {
    if (++p.tile == ntiles(p.seg)) {
      p.tile = 0;
      if (++p.h == Hv) {
        p.h = 0;
        do ++p.seg;
        while (p.seg < N && offs[p.seg + 1] == offs[p.seg]);
      }
    }
    return p;
  };
  auto issue_tile = [&](TilePos p, int buf) {
    const int64_t c0 = offs[p.seg] + (int64_t)kTile * p.tile, s1 = offs[p.seg + 1];
    const int L = (int)((s1 - c0) < kTile ? (s1 - c0) : kTile);
    for (int e = tid; e < kTile * 16; e += kThreads) {
      const int r = e >> 4, c = e & 15;
      const size_t go = ((size_t)(c0 + (r < L ? r : 0)) * Hv + p.h) * D + c * 8;
      const uint32_t so = (uint32_t)(((buf * kTile + r) * kLd + c * 8) * 2);
      cp_async16(sM_addr + so, om + go, r < L);
      cp_async16(sU_addr + so, ou + go, r < L);
    }
    cp_async_commit();
  };
  TilePos cur{s_pos[0], s_pos[1], s_pos[2]};
  issue_tile(cur, 0);
  const int g = lane >> 2, t = lane & 3, m = lane >> 3;
  // warp tile: rows r0 .. +32 (two 16-row MMA tiles), columns n0 .. +32 (four 8-column tiles);
  // its B fragments (the incoming state, the same for every tile of a (segment, head) pair)
  // stay in registers, so only the readout tiles are read from shared memory per tile
  const int r0 = 32 * (warp & 1), n0 = 32 * (warp >> 1);
  uint32_t bfrag[8][2][4];
  int loaded_seg = -1, loaded_h = -1, buf = 0;
#pragma unroll 1
  for (int64_t i = 0; i < count; ++i, buf ^= 1) {
    cp_async_wait_all();
    __syncthreads();  // this tile has landed; every thread is done with the previous tile
    const TilePos nxt = advance(cur);
    if (i + 1 < count) issue_tile(nxt, buf ^ 1);
    if (cur.seg != loaded_seg || cur.h != loaded_h) {
      const float4* S = reinterpret_cast<const float4*>(a.incoming + ((size_t)cur.seg * Hv + cur.h) * (size_t)(D * D));
      for (int e = tid; e < D * D / 4; e += kThreads) {
        if (a.v_first) {  // stored [j][j']: four consecutive elements of a row of sB
          const float4 x = S[e];
          const int row = e >> 5, col = (e & 31) * 4;
          *reinterpret_cast<uint2*>(sB + row * kLd + col) = make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
        } else {  // stored [j'][j]: columns of sB; consecutive lanes take consecutive stored rows,
                  // so each 2-byte store instruction hits 32 consecutive elements of a row of sB
          const int row = e & (D - 1), col = (e >> 7) * 4;
          const float4 x = S[row * (D / 4) + (col >> 2)];
          sB[(col + 0) * kLd + row] = __float2bfloat16_rn(x.x);
          sB[(col + 1) * kLd + row] = __float2bfloat16_rn(x.y);
          sB[(col + 2) * kLd + row] = __float2bfloat16_rn(x.z);
          sB[(col + 3) * kLd + row] = __float2bfloat16_rn(x.w);
        }
      }
      loaded_seg = cur.seg;
      loaded_h = cur.h;
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          const int br = n0 + 16 * np + (m >> 1) * 8 + (lane & 7), bk = 16 * kk + (m & 1) * 8;
          ldsm_x4(sB_addr + (br * kLd + bk) * 2, bfrag[kk][np][0], bfrag[kk][np][1], bfrag[kk][np][2],
                  bfrag[kk][np][3]);
        }
    }
    const int64_t c0 = offs[cur.seg] + (int64_t)kTile * cur.tile, s1 = offs[cur.seg + 1];
    const int L = (int)((s1 - c0) < kTile ? (s1 - c0) : kTile);
    float acc[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[mt][nt][u] = 0.f;
    const uint32_t aM = sM_addr + (uint32_t)(buf * kTile * kLd * 2);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        uint32_t a0, a1, a2, a3;
        const int ar = r0 + 16 * mt + (m & 1) * 8 + (lane & 7), ak = 16 * kk + (m >> 1) * 8;
        ldsm_x4(aM + (ar * kLd + ak) * 2, a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          mma16816(acc[mt][2 * np], a0, a1, a2, a3, bfrag[kk][np][0], bfrag[kk][np][1]);
          mma16816(acc[mt][2 * np + 1], a0, a1, a2, a3, bfrag[kk][np][2], bfrag[kk][np][3]);
        }
      }
    }
    __nv_bfloat16* tU = sU + buf * kTile * kLd;
    float* out32 = reinterpret_cast<float*>(a.out);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int mt = q >> 2, nt = q & 3;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = r0 + 16 * mt + g + 8 * hh, j = n0 + 8 * nt + 2 * t;
        uint32_t* cell = reinterpret_cast<uint32_t*>(tU + r * kLd + j);
        const float2 u = unpack_bf16(*cell);
        const float y0 = acc[mt][nt][2 * hh] + u.x, y1 = acc[mt][nt][2 * hh + 1] + u.y;
        if (a.out_bf16)
          *cell = pack_bf16(y0, y1);
        else if (r < L)
          *reinterpret_cast<float2*>(out32 + ((size_t)(c0 + r) * Hv + cur.h) * D + j) = make_float2(y0, y1);
      }
    }
    if (a.out_bf16) {
      __syncthreads();  // the bf16 result tile is complete
      __nv_bfloat16* out16 = reinterpret_cast<__nv_bfloat16*>(a.out);
      for (int e = tid; e < kTile * 16; e += kThreads) {
        const int r = e >> 4, c = e & 15;
        if (r < L)
          *reinterpret_cast<uint4*>(out16 + ((size_t)(c0 + r) * Hv + cur.h) * D + c * 8) =
              *reinterpret_cast<const uint4*>(tU + r * kLd + c * 8);
      }
    }
    cur = nxt;
  }
}

cudaError_t launch_cp_apply(const ApplyArgs& a, cudaStream_t stream) {
  const int smem = (D + 4 * kTile) * kLd * 2;
  cudaError_t err = cudaFuncSetAttribute(cp_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  cp_apply_kernel<<<2 * sms, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
