// kda_cp_apply.cu -- last step of the context-parallel prefill: every token's output from the
// local readouts of its segment and the segment's incoming state.
//
// Inside a segment the state after token t is S_t = M_{<=t} S_in + U_{<=t} (the segment's map
// applied to its incoming state -- "KDA Context Parallelism", Theory: a segment can be applied
// to any incoming state without replaying its tokens), so the readout is affine in S_in:
//     o_t = (q_t^T M_{<=t}) S_in + q_t^T U_{<=t} = O_M[t] . S_in + O_U[t].
// The segment-build pass writes O_M and O_U; this kernel adds the incoming state's share.
//
// Per 128-token tile of one (segment, head) pair the product O_M (128 x 128) . S_in (128 x 128)
// runs on tcgen05 into a TMEM accumulator; both readout tiles arrive by tensor copies through a
// three-stage ring, so two tiles' loads are in flight while one is finished.  All eight warps
// work in step: after a tile's epilogue (which adds O_U and writes the bf16 result over the O_U
// tile in place) one thread issues the copies two tiles ahead and the next tile's MMA, into the
// other of two accumulators; a full tile leaves through tensor stores, a partial last tile of a segment
// through row stores (rows past the segment belong to the next one).
#include <cuda.h>
#include <string.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

// tensor map of a [tokens][heads][128] tensor (kda_fused.cu): box = box_x channels x 1 head x 64
// tokens; head_major: a [heads][tokens][128] tensor, coordinates (channel, token, head)
bool encode_token_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t esize, int64_t tokens,
                       int heads, uint32_t box_x, CUtensorMapSwizzle swz, bool head_major);

namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 256;
constexpr int kRows = 128;            // tokens per tile: the MMA's M
constexpr int kStages = 3;
constexpr int kTileBytes = 32768;     // one 128 x 128 bf16 tile
constexpr int kStageBytes = 2 * kTileBytes;  // O_M tile, then O_U tile
constexpr int OFF_B = kStages * kStageBytes;  // the incoming state as the bf16 B operand
constexpr int OFF_BAR = OFF_B + kTileBytes;   // mbarriers: full[kStages], acc[2], fin; TMEM address
constexpr int kSmemAlloc = OFF_BAR + 64 + 1024;  // + slack for the 1024-byte alignment
constexpr uint32_t kTmemCols = 256;   // two 128-column fp32 accumulators
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct ApplyMaps {
  CUtensorMap om, ou, out;
};

// Byte offset of element (row r, column j) of a 128 x 128 bf16 tile kept as two K-major
// 128-byte-swizzle halves: columns 64 c .. +63 at c * 16384, row r at r * 128, the 16-byte chunk
// k of a row at k ^ (r % 8) -- the layout of the tensor copies and of the MMA operands.
__device__ __forceinline__ uint32_t tile_off(int r, int j) {
  return (uint32_t)((j >> 6) * 16384 + r * 128 + ((((j & 63) >> 3) ^ (r & 7)) << 4) + (j & 7) * 2);
}

struct TilePos {
  int seg, h, tile;
};

}  // namespace

// The work is the flat list of 128-token tiles ordered by (segment, value head, tile); a
// persistent grid of one block per SM splits it into equal contiguous ranges.
__global__ void __launch_bounds__(kThreads, 1) cp_apply_kernel(ApplyArgs a, const __grid_constant__ ApplyMaps tm) {
  if (a.skip_flag && *a.skip_flag) return;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_addr(sm);
  __shared__ int64_t s_range[2];
  __shared__ int s_pos[3];
  __shared__ int s_bad;
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.num_segments, Hv = a.Hv;
  const int32_t* offs = a.seg_offsets;
  if (tid == 0) {
    s_bad = 0;
    s_abort = 0;
  }
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
  auto ntiles = [&](int seg) { return (int)((offs[seg + 1] - offs[seg] + kRows - 1) / kRows); };
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

  const uint32_t bar_full = sbase + OFF_BAR, bar_acc = bar_full + 8 * kStages, bar_fin = bar_acc + 16;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 8 * (kStages + 3));
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bar_full + 8 * s, 1);
    mbar_init(bar_acc, 1);
    mbar_init(bar_acc + 8, 1);
    mbar_init(bar_fin, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

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
  auto row0 = [&](const TilePos& p) { return (int)(offs[p.seg] + (int64_t)kRows * p.tile); };
  uint32_t nload[kStages] = {0u, 0u, 0u};  // (thread 0) copies issued per stage
  // both readout tiles of tile p into stage s: four 64 x 64 boxes each (column half, row half)
  auto issue_loads = [&](const TilePos& p, int s) {
    const uint32_t dst = sbase + s * kStageBytes, bar = bar_full + 8 * s;
    ++nload[s];
    const int t0 = row0(p);
    mbar_arrive_expect_tx(bar, (uint32_t)kStageBytes);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int ch = q >> 1, rh = q & 1;
      const int y = a.readout_hm ? t0 + 64 * rh : p.h, z = a.readout_hm ? p.h : t0 + 64 * rh;
      tma_load_3d(dst + ch * 16384 + rh * 8192, &tm.om, 64 * ch, y, z, bar);
      tma_load_3d(dst + kTileBytes + ch * 16384 + rh * 8192, &tm.ou, 64 * ch, y, z, bar);
    }
  };
  auto fail = [&]() {
    s_abort = 1;
    report(a.status, KDA_ERR_DEVICE_TIMEOUT);
  };
  // the incoming state of a pair as the K-major B operand: B[n = j][k = i] = S_in[i][j], bf16;
  // one 16-byte chunk (8 consecutive i of one j) per step, consecutive lanes on consecutive
  // global addresses in either stored layout
  auto stage_state = [&](const TilePos& p) {
    const float* S = a.incoming + ((size_t)p.seg * Hv + p.h) * (size_t)(D * D);
    for (int e = tid; e < D * 16; e += kThreads) {
      int j, cg;
      float x[8];
      if (a.v_first) {  // stored [j][i]: row j of the operand is a stored row
        j = e >> 4;
        cg = e & 15;
        const float4 u = *reinterpret_cast<const float4*>(S + (size_t)j * D + cg * 8);
        const float4 w = *reinterpret_cast<const float4*>(S + (size_t)j * D + cg * 8 + 4);
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
      } else {  // stored [i][j]: eight rows i at column j
        j = e & (D - 1);
        cg = e >> 7;
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = S[(size_t)(cg * 8 + u) * D + j];
      }
      *reinterpret_cast<uint4*>(sm + OFF_B + tile_off(j, cg * 8)) =
          make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
    }
    fence_async_smem();  // generic-proxy writes, read next by the tensor cores
  };
  // D[acc] = O_M tile (stage s) . S_in, eight K = 16 steps; completion on bar_acc + 8 acc
  auto issue_mma = [&](int s, int acc) {
    tc_fence_after();
    const uint32_t am = sbase + s * kStageBytes, bm = sbase + OFF_B;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
      mma_bf16(tmem + acc * 128, desc_sw128(am + koff), desc_sw128(bm + koff), idesc_bf16_f32(128), kk > 0);
    }
    mma_commit(bar_acc + 8 * acc);
  };

  TilePos cur{s_pos[0], s_pos[1], s_pos[2]};
  // prologue: the first two tiles' copies, the first pair's state, the first product
  TilePos lpos = cur;  // the tile whose copies are issued next
  for (int s = 0; s < 2 && s < count; ++s) {
    if (tid == 0) issue_loads(lpos, s);
    if (s + 1 < count) lpos = advance(lpos);  // never past the block's last tile
  }
  stage_state(cur);
  __syncthreads();
  if (tid == 0) {
    if (mbar_wait_bounded(bar_full, 0, kWaitLimitNs))
      issue_mma(0, 0);
    else
      fail();
  }
  const int q = warp & 3, r = 32 * q + lane, chh = warp >> 2;  // epilogue: row r, columns 64 chh .. +63
  const uint32_t lane_base = (uint32_t)(32 * q) << 16;
  __nv_bfloat16* out16 = reinterpret_cast<__nv_bfloat16*>(a.out);
  float* out32 = reinterpret_cast<float*>(a.out);
  bool aborted = false;
#pragma unroll 1
  for (int64_t i = 0; i < count; ++i) {
    const int s = (int)(i % kStages), acc = (int)(i & 1);
    const bool has_next = i + 1 < count;
    const TilePos nxt = has_next ? advance(cur) : cur;
    const bool same_pair = has_next && nxt.seg == cur.seg && nxt.h == cur.h;
    const bool ok = mbar_wait_bounded(bar_acc + 8 * acc, (uint32_t)((i >> 1) & 1), kWaitLimitNs) &&
                    mbar_wait_bounded(bar_full + 8 * s, (uint32_t)((i / kStages) & 1), kWaitLimitNs);
    if (!ok) fail();
    tc_fence_after();
    const int t0 = row0(cur);
    const int L = (int)((offs[cur.seg + 1] - t0) < kRows ? (offs[cur.seg + 1] - t0) : kRows);
    const bool full = L == kRows && a.out_bf16;
    if (ok) {
      float d[64];
      tmem_ld64(tmem + acc * 128 + lane_base + 64 * chh, d);
      tmem_wait_ld();
      uint8_t* tU = sm + s * kStageBytes + kTileBytes;
      if (a.out_bf16) {
        uint4 res[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(tU + tile_off(r, 64 * chh + 8 * c));
          const float2 u0 = unpack_bf16(u.x), u1 = unpack_bf16(u.y), u2 = unpack_bf16(u.z), u3 = unpack_bf16(u.w);
          const float* dd = d + 8 * c;
          res[c] = make_uint4(pack_bf16(dd[0] + u0.x, dd[1] + u0.y), pack_bf16(dd[2] + u1.x, dd[3] + u1.y),
                              pack_bf16(dd[4] + u2.x, dd[5] + u2.y), pack_bf16(dd[6] + u3.x, dd[7] + u3.y));
        }
        if (full) {
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(tU + tile_off(r, 64 * chh + 8 * c)) = res[c];
        } else if (r < L) {
          uint4* dst = reinterpret_cast<uint4*>(out16 + ((size_t)(t0 + r) * Hv + cur.h) * D + 64 * chh);
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[c] = res[c];
        }
      } else if (r < L) {
        float4* dst = reinterpret_cast<float4*>(out32 + ((size_t)(t0 + r) * Hv + cur.h) * D + 64 * chh);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(tU + tile_off(r, 64 * chh + 8 * c));
          const float2 u0 = unpack_bf16(u.x), u1 = unpack_bf16(u.y), u2 = unpack_bf16(u.z), u3 = unpack_bf16(u.w);
          const float* dd = d + 8 * c;
          dst[2 * c] = make_float4(dd[0] + u0.x, dd[1] + u0.y, dd[2] + u1.x, dd[3] + u1.y);
          dst[2 * c + 1] = make_float4(dd[4] + u2.x, dd[5] + u2.y, dd[6] + u3.x, dd[7] + u3.y);
        }
      }
    }
    if (full) fence_async_smem();  // the in-place result, read next by the tensor stores
    tc_fence_before();
    __syncthreads();  // epilogue done: accumulator acc is free, stage s once its stores read it
    if (s_abort) {
      aborted = true;
      break;
    }
    if (tid == 0) {
      if (full) {
        const uint32_t src = sbase + s * kStageBytes + kTileBytes;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int ch = qq >> 1, rh = qq & 1;
          tma_store_3d(&tm.out, src + ch * 16384 + rh * 8192, 64 * ch, cur.h, t0 + 64 * rh);
        }
      }
      bulk_commit();  // one group per tile (empty without stores), so groups count tiles
    }
    if (has_next && !same_pair) {
      // a new pair: its state replaces the B operand (this tile's product, its last reader, is
      // complete)
      stage_state(nxt);
      tc_fence_before();
      __syncthreads();
    }
    // tile i + 2 goes to the stage of tile i - 1, whose stores (the group before this tile's)
    // have read it by now
    if (i + 2 < count) {
      if (tid == 0) {
        bulk_wait_read_prev();
        issue_loads(lpos, (int)((i + 2) % kStages));
      }
      if (i + 3 < count) lpos = advance(lpos);
    }
    // the next tile's product, into the other accumulator (its last reader, the epilogue of tile
    // i - 1, is done): its copies were issued one epilogue ago, so they have had this tile's
    // epilogue to land
    if (tid == 0 && has_next) {
      const int s1 = (int)((i + 1) % kStages);
      if (mbar_wait_bounded(bar_full + 8 * s1, (uint32_t)(((i + 1) / kStages) & 1), kWaitLimitNs))
        issue_mma(s1, acc ^ 1);
      else
        fail();
    }
    cur = nxt;
  }
  if (tid == 0) {
    bulk_wait_all();
    if (aborted) {
      // products and copies still in flight finish before the tensor memory and the block go
      mma_commit(bar_fin);
      mbar_wait_bounded(bar_fin, 0, kWaitLimitNs);
      for (int s = 0; s < kStages; ++s)
        if (nload[s] > 0) mbar_wait_bounded(bar_full + 8 * s, (nload[s] - 1) & 1u, kWaitLimitNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

cudaError_t launch_cp_apply(const ApplyArgs& a, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(cp_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (err != cudaSuccess) return err;
  if (a.total_tokens == 0) return cudaSuccess;
  ApplyMaps tm;
  memset(&tm, 0, sizeof(tm));
  const bool ok =
      encode_token_rows(&tm.om, a.o_m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.total_tokens, a.Hv, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B, a.readout_hm != 0) &&
      encode_token_rows(&tm.ou, a.o_u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.total_tokens, a.Hv, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B, a.readout_hm != 0) &&
      (!a.out_bf16 || encode_token_rows(&tm.out, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.total_tokens, a.Hv,
                                        64, CU_TENSOR_MAP_SWIZZLE_128B, false));
  if (!ok) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  cp_apply_kernel<<<sms, kThreads, kSmemAlloc, stream>>>(a, tm);
  return cudaGetLastError();
}

}  // namespace kda
