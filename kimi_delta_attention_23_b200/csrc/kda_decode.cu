// kda_decode.cu -- single-token KDA step over a batch of sequences, in place on the state pool.
//
// "max.nn.state_space.kda_chunk" names kda_decode as the single-token path of the same
// recurrence the chunked prefill evaluates; "nx_nofloat_kda.nx source" (kda_step) fixes the
// order of one step: decay, delta write predicting from the decayed state, readout after the
// write.  Per (sequence b, value head h), with S = state_pool[state_indices[b], h] (dk x dv,
// fp32) and the token's per-channel decay alpha_i = exp(g_i):
//
//   Sd    = Diag(alpha) S
//   pred  = k^T Sd,   delta = beta (v - pred)
//   S'    = Sd + k delta^T                        (written back to the slot)
//   o     = q^T S' = q^T Sd + (q . k) delta
//
// Every state element is read once and written once, so the step is bound by HBM:
// 2 * dk * dv * 4 bytes per (sequence, head), next to which q, k, v, the gate and the output
// are small.  One CTA per (sequence, head); its 256 threads hold the state block in registers
// (up to 64 elements each) between the read and the write.  The loads of the block are issued
// before the gate is evaluated, so the per-channel vectors are computed under their latency.
//
// Thread mapping for dk = dv = 128 (kVec): the same split, with lane l taking the four
// consecutive elements 4l .. 4l + 3 of each stored row, so every state access is 16 bytes.
// Thread mapping (any 1 <= dk, dv <= 128):
//   K_FIRST ([dk][dv] row-major): warp w takes rows i = w + 8m, lane l takes columns
//     j = l + 32c; a warp load is 32 consecutive floats of one row.  Column sums over i
//     (pred, q^T Sd) cross warps and are combined in shared memory.
//   V_FIRST ([dv][dk]): warp w takes columns j = w + 8m, lane l takes rows i = l + 32c; a warp
//     load is 32 consecutive floats of one stored row S^T[j].  Column sums are warp reductions.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <bool kVFirst, bool kVec>
__global__ void __launch_bounds__(kDecThreads, 2) decode_kernel(const DecodeArgs a) {
  __shared__ __align__(16) float sAlpha[128], sK[128], sQ[128], sV[128], sDelta[128];
  __shared__ __align__(16) float sRed[2][kDecWarps][128];
  __shared__ float sBeta, sQK;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // four consecutive floats at 4 lane (kVec): one 16-byte access, no bank conflict
  auto get4 = [&](const float* arr, float (&o)[4]) {
    if constexpr (kVec) {
      const float4 v4 = *reinterpret_cast<const float4*>(arr + 4 * lane);
      o[0] = v4.x;
      o[1] = v4.y;
      o[2] = v4.z;
      o[3] = v4.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) o[c] = arr[(lane + 32 * c) & 127];
    }
  };
  const int64_t bh = blockIdx.x;
  const int h = (int)(bh % a.Hv);
  const int64_t b = bh / a.Hv;
  const int dk = a.dk, dv = a.dv;
  const int32_t slot = a.slots[b];
  if (slot < 0 || slot >= a.max_slots) {
    if (tid == 0) report(a.status, KDA_ERR_DEVICE_CHECK);
    return;  // this sequence is skipped: its slot and output row stay untouched
  }
  float* blk = a.pool + ((size_t)slot * a.Hv + h) * (size_t)dk * dv;

  // ---- issue the loads of this thread's state elements first.  Element c of stored row
  // r = warp + 8m is at stored column col(c) = 4 lane + c (kVec) or lane + 32 c.
  auto col = [&](int c) { return kVec ? 4 * lane + c : lane + 32 * c; };
  float s[16][4];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if constexpr (kVec) {
      const float4 v4 = *reinterpret_cast<const float4*>(blk + (size_t)(warp + 8 * m) * 128 + 4 * lane);
      s[m][0] = v4.x;
      s[m][1] = v4.y;
      s[m][2] = v4.z;
      s[m][3] = v4.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int i = kVFirst ? col(c) : warp + 8 * m;  // key channel (row of S)
        const int j = kVFirst ? warp + 8 * m : col(c);  // value column
        s[m][c] = (i < dk && j < dv) ? blk[kVFirst ? (size_t)j * dk + i : (size_t)i * dv + j] : 0.f;
      }
    }
  }

  // ---- per-channel vectors of this token: decay, k, q (threads 0..127), v (threads 128..255)
  const int kh = h / (a.Hv / a.Hk);
  const bool safe = a.flags & KDA_GATE_SAFE, prob = a.flags & KDA_BETA_PROB;
  if (tid < 128) {
    float al = 1.f, kv = 0.f, qv = 0.f;
    if (tid < dk) {
      const float g = gate_f32(a.raw_gate[((size_t)b * a.Hv + h) * dk + tid], a.a_log[h],
                               a.dt_bias[(size_t)h * dk + tid], safe, a.lb);
      al = expf(g);
      const size_t qi = ((size_t)b * a.Hk + kh) * dk + tid;
      kv = load_in(a.k, qi, a.in_bf16);
      qv = load_in(a.q, qi, a.in_bf16);
    }
    sAlpha[tid] = al;
    sK[tid] = kv;
    sQ[tid] = qv;
    if (tid < 32) {  // q . k over the key channels
      float p = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int i = tid + 32 * c;
        if (i < dk) {
          const size_t qi = ((size_t)b * a.Hk + kh) * dk + i;
          p += load_in(a.q, qi, a.in_bf16) * load_in(a.k, qi, a.in_bf16);
        }
      }
      p = warp_sum(p);
      if (tid == 0) {
        sQK = p;
        sBeta = beta_f32(a.beta[(size_t)b * a.Hv + h], prob);
      }
    }
  } else {
    const int j = tid - 128;
    sV[j] = j < dv ? load_in(a.v, ((size_t)b * a.Hv + h) * dv + j, a.in_bf16) : 0.f;
  }
  __syncthreads();

  const float beta = sBeta, qk = sQK;
  void* out = a.out;
  const size_t out_row = ((size_t)b * a.Hv + h) * dv;

  if constexpr (kVFirst) {
    float al[4], kc[4], qc[4];
    get4(sAlpha, al);
    get4(sK, kc);
    get4(sQ, qc);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      float pk = 0.f, pq = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[m][c] *= al[c];
        pk = fmaf(kc[c], s[m][c], pk);
        pq = fmaf(qc[c], s[m][c], pq);
      }
      pk = warp_sum(pk);
      pq = warp_sum(pq);
      const int j = warp + 8 * m;
      if (j < dv) {
        const float delta = beta * (sV[j] - pk);
        if (lane == 0) store_out(out, out_row + j, fmaf(qk, delta, pq), a.out_bf16);
        if constexpr (kVec) {
          *reinterpret_cast<float4*>(blk + (size_t)j * 128 + 4 * lane) =
              make_float4(fmaf(kc[0], delta, s[m][0]), fmaf(kc[1], delta, s[m][1]), fmaf(kc[2], delta, s[m][2]),
                          fmaf(kc[3], delta, s[m][3]));
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int i = col(c);
            if (i < dk) blk[(size_t)j * dk + i] = fmaf(kc[c], delta, s[m][c]);
          }
        }
      }
    }
  } else {
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int i = (warp + 8 * m) & 127;
      const float al = sAlpha[i], kv = sK[i], qv = sQ[i];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[m][c] *= al;
        pk[c] = fmaf(kv, s[m][c], pk[c]);
        pq[c] = fmaf(qv, s[m][c], pq[c]);
      }
    }
    if constexpr (kVec) {
      *reinterpret_cast<float4*>(&sRed[0][warp][4 * lane]) = make_float4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<float4*>(&sRed[1][warp][4 * lane]) = make_float4(pq[0], pq[1], pq[2], pq[3]);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sRed[0][warp][col(c)] = pk[c];
        sRed[1][warp][col(c)] = pq[c];
      }
    }
    __syncthreads();
    if (tid < dv) {
      float p = 0.f, r = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        p += sRed[0][w][tid];
        r += sRed[1][w][tid];
      }
      const float delta = beta * (sV[tid] - p);
      sDelta[tid] = delta;
      store_out(out, out_row + tid, fmaf(qk, delta, r), a.out_bf16);
    }
    __syncthreads();
    float dl[4];
    get4(sDelta, dl);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int i = warp + 8 * m;
      if (i < dk) {
        const float kv = sK[i];
        if constexpr (kVec) {
          *reinterpret_cast<float4*>(blk + (size_t)i * 128 + 4 * lane) =
              make_float4(fmaf(kv, dl[0], s[m][0]), fmaf(kv, dl[1], s[m][1]), fmaf(kv, dl[2], s[m][2]),
                          fmaf(kv, dl[3], s[m][3]));
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int j = col(c);
            if (j < dv) blk[(size_t)i * dv + j] = fmaf(kv, dl[c], s[m][c]);
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t blocks = (int64_t)a.batch * a.Hv;
  if (blocks == 0) return cudaSuccess;
  // 16-byte state accesses when every stored row is 128 floats and the pool is 16-byte aligned
  const bool vec = a.dk == 128 && a.dv == 128 && (reinterpret_cast<uintptr_t>(a.pool) & 15u) == 0;
  if (a.v_first) {
    if (vec)
      decode_kernel<true, true><<<(unsigned)blocks, kDecThreads, 0, stream>>>(a);
    else
      decode_kernel<true, false><<<(unsigned)blocks, kDecThreads, 0, stream>>>(a);
  } else {
    if (vec)
      decode_kernel<false, true><<<(unsigned)blocks, kDecThreads, 0, stream>>>(a);
    else
      decode_kernel<false, false><<<(unsigned)blocks, kDecThreads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace kda
