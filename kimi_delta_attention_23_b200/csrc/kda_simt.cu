// kda_simt.cu -- fp32 CUDA-core chunk kernel (any dk, w <= 128) and the exclusive affine scan.
//
// The chunk kernel evaluates the KDA recurrence 16 tokens at a time.  Inside a chunk with
// incoming state S0, log-gate prefix G_r = sum_{u<=r} g_u (per key channel) and
// Gamma_r = exp(G_r), the per-token step (decay, delta write from the decayed state,
// readout -- "nx_nofloat_kda.nx source", kda_forward) unrolls to
//
//   A_rs   = sum_i k_ri k_si exp(G_ri - G_si)    (s < r)      stable gated scores: every
//   P_rs   = sum_i q_ri k_si exp(G_ri - G_si)    (s <= r)     exponent is <= 0
//   Delta  = (I + diag(beta) A)^{-1} diag(beta) (V - (K o Gamma) S0)   forward substitution
//   O      = (Q o Gamma) S0 + P Delta
//   S_C    = Diag(Gamma_C) S0 + (K o exp(G_C - G))^T Delta
//
// (GStar Assignment 2, Learning path: P4 gate prefix scan, P6 triangular inverse, P8 stable
// scores, P9 the assembled chunked forward; "max.nn.state_space.kda_chunk": 16-token chunks.)
// The same kernel builds segment summaries: with the state started at I (width dk) and zero
// values it yields the transition M_i; started at 0 with the real values it yields U_i.
#include <cmath>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

constexpr int kSimtC = 16;
constexpr int kSimtThreads = 256;

size_t simt_smem_bytes(int dk, int w) {
  const int C = kSimtC;
  size_t floats = (size_t)dk * w + 6 * (size_t)C * dk + (size_t)C * w + 2 * C * C + C + dk;
  return floats * sizeof(float);
}

__global__ void __launch_bounds__(kSimtThreads) simt_chunk_kernel(SimtArgs a) {
  extern __shared__ float smem[];
  constexpr int C = kSimtC;
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int dk = a.dk, W = a.w;
  const int kh = h / (a.Hv / a.Hk);
  const bool safe = a.flags & KDA_GATE_SAFE, prob = a.flags & KDA_BETA_PROB;

  const int64_t t0 = a.cu[b], t1 = a.cu[b + 1];
  const int32_t slot = a.slots ? a.slots[b] : b;
  if (t0 < 0 || t1 < t0 || t1 > a.total_tokens || slot < 0 || slot >= a.max_slots) {
    if (tid == 0) report(a.status, KDA_ERR_DEVICE_CHECK);
    return;
  }

  float* S = smem;                     // [dk][W] working state, always row-major
  float* qq = S + (size_t)dk * W;      // [C][dk] q
  float* kk = qq + C * dk;             // [C][dk] k
  float* qg = kk + C * dk;             // [C][dk] q o Gamma
  float* kg = qg + C * dk;             // [C][dk] k o Gamma
  float* kp = kg + C * dk;             // [C][dk] k o exp(G_C - G)
  float* G = kp + C * dk;              // [C][dk] log-gate prefix
  float* D = G + C * dk;               // [C][W]  residual, then Delta
  float* A = D + C * W;                // [C][C]
  float* P = A + C * C;                // [C][C]
  float* bt = P + C * C;               // [C] beta
  float* gC = bt + C;                  // [dk] Gamma_C

  const size_t blk = (size_t)dk * W;
  const size_t blk_off = ((size_t)slot * a.Hv + h) * blk;
  if (a.init_mode == 0) {
    const float* src = a.state_in + blk_off;
    for (size_t e = tid; e < blk; e += kSimtThreads) {
      int i, j;
      if (a.v_first) { j = (int)(e / dk); i = (int)(e % dk); }
      else { i = (int)(e / W); j = (int)(e % W); }
      S[(size_t)i * W + j] = src[e];
    }
  } else {
    for (size_t e = tid; e < blk; e += kSimtThreads) {
      int i = (int)(e / W), j = (int)(e % W);
      S[e] = (a.init_mode == 2 && i == j) ? 1.0f : 0.0f;
    }
  }
  __syncthreads();

  const float al = a.a_log[h];
  for (int64_t c0 = t0; c0 < t1; c0 += C) {
    const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);
    for (int e = tid; e < C * dk; e += kSimtThreads) {
      const int r = e / dk, i = e % dk;
      float qv = 0.f, kv = 0.f, g = 0.f;
      if (r < L) {
        const int64_t t = c0 + r;
        const size_t qi = ((size_t)t * a.Hk + kh) * dk + i;
        qv = a.q ? load_in(a.q, qi, a.in_bf16) : 0.f;
        kv = load_in(a.k, qi, a.in_bf16);
        g = gate_f32(a.raw_gate[((size_t)t * a.Hv + h) * dk + i], al, a.dt_bias[(size_t)h * dk + i],
                     safe, a.lb);
      }
      qq[e] = qv;
      kk[e] = kv;
      G[e] = g;
    }
    if (tid < C) bt[tid] = tid < L ? beta_f32(a.beta[(size_t)(c0 + tid) * a.Hv + h], prob) : 0.f;
    __syncthreads();
    // padded rows carry g = 0, so the prefix stays flat past the sequence end
    for (int i = tid; i < dk; i += kSimtThreads) {
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += G[r * dk + i];
        G[r * dk + i] = acc;
      }
      gC[i] = expf(acc);
    }
    __syncthreads();
    for (int e = tid; e < C * dk; e += kSimtThreads) {
      const int i = e % dk;
      const float Gr = G[e], GC = G[(C - 1) * dk + i];
      const float gam = expf(Gr);
      qg[e] = qq[e] * gam;
      kg[e] = kk[e] * gam;
      kp[e] = kk[e] * expf(GC - Gr);
    }
    for (int e = tid; e < C * C; e += kSimtThreads) {
      const int r = e / C, s = e % C;
      float av = 0.f, pv = 0.f;
      if (s <= r) {
        for (int i = 0; i < dk; ++i) {
          const float w = kk[s * dk + i] * expf(G[r * dk + i] - G[s * dk + i]);
          av = fmaf(kk[r * dk + i], w, av);
          pv = fmaf(qq[r * dk + i], w, pv);
        }
      }
      A[e] = s < r ? av : 0.f;
      P[e] = pv;
    }
    __syncthreads();
    // residual R = V - (K o Gamma) S0
    for (int e = tid; e < C * W; e += kSimtThreads) {
      const int r = e / W, j = e % W;
      float acc = 0.f;
      if (r < L && !a.values_zero) acc = load_in(a.v, ((size_t)(c0 + r) * a.Hv + h) * a.dv_in + j, a.in_bf16);
      for (int i = 0; i < dk; ++i) acc = fmaf(-kg[r * dk + i], S[(size_t)i * W + j], acc);
      D[e] = acc;
    }
    __syncthreads();
    // Delta_r = beta_r (R_r - sum_{s<r} A_rs Delta_s), rows in order
    for (int r = 0; r < C; ++r) {
      for (int j = tid; j < W; j += kSimtThreads) {
        float acc = D[r * W + j];
        for (int s = 0; s < r; ++s) acc = fmaf(-A[r * C + s], D[s * W + j], acc);
        D[r * W + j] = bt[r] * acc;
      }
      __syncthreads();
    }
    if (a.out) {
      for (int e = tid; e < L * W; e += kSimtThreads) {
        const int r = e / W, j = e % W;
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc = fmaf(qg[r * dk + i], S[(size_t)i * W + j], acc);
        for (int s = 0; s <= r; ++s) acc = fmaf(P[r * C + s], D[s * W + j], acc);
        store_out(a.out, ((size_t)(c0 + r) * a.Hv + h) * W + j, acc, a.out_bf16);
      }
    }
    __syncthreads();
    for (size_t e = tid; e < blk; e += kSimtThreads) {
      const int i = (int)(e / W), j = (int)(e % W);
      float acc = gC[i] * S[e];
      for (int s = 0; s < C; ++s) acc = fmaf(kp[s * dk + i], D[s * W + j], acc);
      S[e] = acc;
    }
    __syncthreads();
  }

  float* dst = a.state_out + blk_off;
  for (size_t e = tid; e < blk; e += kSimtThreads) {
    int i, j;
    if (a.v_first) { j = (int)(e / dk); i = (int)(e % dk); }
    else { i = (int)(e / W); j = (int)(e % W); }
    dst[e] = S[(size_t)i * W + j];
  }
}

cudaError_t launch_simt_chunk(const SimtArgs& a, cudaStream_t stream) {
  const size_t smem = simt_smem_bytes(a.dk, a.w);
  cudaError_t err = cudaFuncSetAttribute(simt_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  if (a.batch == 0) return cudaSuccess;
  dim3 grid(a.Hv, a.batch);
  simt_chunk_kernel<<<grid, kSimtThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Exclusive affine scan ("KDA Context Parallelism", Incoming and outgoing states):
//   in_0 = S_initial;  out_i = M_i in_i + U_i;  in_{i+1} = out_i;  final = out_{N-1}.
// One block per (head, 16-column tile of the state); the segment loop is serial.
// ------------------------------------------------------------------------------------------
constexpr int kScanCols = 16;
constexpr int kScanThreads = 256;

// One block per (head, 16-column tile of the state).  Each step stages M_i (dk x dk) in shared
// memory with coalesced float4 loads; thread t then owns row t / 2 and eight of the sixteen
// columns, so every M element read from shared memory feeds eight independent accumulators.
__global__ void __launch_bounds__(kScanThreads) affine_scan_kernel(ScanArgs a) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, j0 = blockIdx.y * kScanCols, tid = threadIdx.x;
  const int dk = a.dk, dv = a.dv, H = a.H;
  const int nc = min(kScanCols, dv - j0);
  float* Ms = sm;                           // [dk][dk + 1]
  float* cur = Ms + dk * (dk + 1);          // [dk][kScanCols]
  float* nxt = cur + dk * kScanCols;        // [dk][kScanCols]
  const size_t st = (size_t)dk * dv;
  for (int e = tid; e < dk * kScanCols; e += kScanThreads) {
    const int i = e / kScanCols, jj = e % kScanCols;
    cur[e] = jj < nc ? a.initial[(size_t)h * st + state_off(i, j0 + jj, dk, dv, a.v_first)] : 0.f;
  }
  const int row = tid >> 1, c0 = (tid & 1) * 8;
  for (int s = 0; s < a.N; ++s) {
    const size_t base = ((size_t)s * H + h) * st;
    const float* Mg = a.M + ((size_t)s * H + h) * (size_t)dk * dk;
    __syncthreads();  // previous step's reads of Ms are done
    if ((dk & 3) == 0) {
      for (int e = tid; e < dk * dk / 4; e += kScanThreads) {
        const float4 m4 = reinterpret_cast<const float4*>(Mg)[e];
        const int i = (4 * e) / dk, l = (4 * e) % dk;
        float* d = Ms + i * (dk + 1) + l;
        d[0] = m4.x;
        d[1] = m4.y;
        d[2] = m4.z;
        d[3] = m4.w;
      }
    } else {
      for (int e = tid; e < dk * dk; e += kScanThreads) Ms[(e / dk) * (dk + 1) + e % dk] = Mg[e];
    }
    __syncthreads();
    for (int r = row; r < dk; r += kScanThreads / 2) {
      float acc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = 0.f;
      const float* mrow = Ms + r * (dk + 1);
      for (int l = 0; l < dk; ++l) {
        const float m = mrow[l];
        const float* cr = cur + l * kScanCols + c0;
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = fmaf(m, cr[u], acc[u]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int jj = c0 + u;
        if (jj >= nc) continue;
        const size_t o = base + state_off(r, j0 + jj, dk, dv, a.v_first);
        if (a.incoming) a.incoming[o] = cur[r * kScanCols + jj];
        const float v = acc[u] + a.U[o];
        nxt[r * kScanCols + jj] = v;
        if (a.outgoing) a.outgoing[o] = v;
      }
    }
    __syncthreads();
    float* t = cur;
    cur = nxt;
    nxt = t;
  }
  if (a.final_state) {
    __syncthreads();
    for (int e = tid; e < dk * kScanCols; e += kScanThreads) {
      const int i = e / kScanCols, jj = e % kScanCols;
      if (jj < nc) a.final_state[(size_t)h * st + state_off(i, j0 + jj, dk, dv, a.v_first)] = cur[e];
    }
  }
}

bool tiles128(int dk, int dv);
cudaError_t launch_affine_scan128(const ScanArgs& a, cudaStream_t stream);
__global__ void compose128_kernel(ComposeArgs a);

cudaError_t launch_affine_scan(const ScanArgs& a, cudaStream_t stream) {
  if (tiles128(a.dk, a.dv)) {
    return launch_affine_scan128(a, stream);
  }
  const size_t smem = ((size_t)a.dk * (a.dk + 1) + 2 * (size_t)a.dk * kScanCols) * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(affine_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid(a.H, (a.dv + kScanCols - 1) / kScanCols);
  affine_scan_kernel<<<grid, kScanThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Segments split into pieces (more chains for the segment build than segments): the pieces'
// boundaries, and each segment's summary rebuilt from its pieces' summaries by composing them
// in order ("KDA Context Parallelism", Theory: (M2, U2) o (M1, U1) = (M2 M1, M2 U1 + U2)).
// ------------------------------------------------------------------------------------------

// Piece p of segment i covers chunk-aligned tokens [s0 + 64 floor(nch p / k), ...) of the
// segment [s0, s1) (nch = its 64-token chunks); decreasing offsets stay decreasing.
__global__ void split_offsets_kernel(const int32_t* offs, int32_t N, int32_t k, int32_t* sub) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e > N * k) return;
  const int i = e / k, p = e % k;
  if (i == N) {
    sub[e] = offs[N];
    return;
  }
  const int64_t s0 = offs[i], s1 = offs[i + 1];
  const int64_t nch = s1 > s0 ? (s1 - s0 + 63) / 64 : 0;
  const int64_t b = s0 + 64 * ((nch * p) / k);
  sub[e] = (int32_t)(b < s1 ? b : (s1 > s0 ? s1 : s0));
}

cudaError_t launch_split_offsets(const int32_t* offs, int32_t N, int32_t k, int32_t* sub, cudaStream_t stream) {
  const int n = N * k + 1;
  split_offsets_kernel<<<(n + 255) / 256, 256, 0, stream>>>(offs, N, k, sub);
  return cudaGetLastError();
}

// One block per (segment, head, 16-column tile): tiles of M_i (dk columns) carry the product of
// the pieces' transitions from I; tiles of U_i (dv columns) carry the pieces' affine maps from
// 0.  The U tiles also copy the segment's incoming state (its first piece's) and outgoing state
// (the next segment's incoming state, or the final state), unless the pieces' incoming states
// are not given (inc == NULL: summaries only).
__global__ void __launch_bounds__(kScanThreads) compose_pieces_kernel(ComposeArgs a) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, seg = blockIdx.z, tid = threadIdx.x;
  const int dk = a.dk, dv = a.dv, H = a.H, k = a.k;
  const int nbm = (dk + kScanCols - 1) / kScanCols;
  const bool is_m = (int)blockIdx.y < nbm;
  const int j0 = (is_m ? (int)blockIdx.y : (int)blockIdx.y - nbm) * kScanCols;
  const int width = is_m ? dk : dv;
  const int nc = min(kScanCols, width - j0);
  float* Ms = sm;                   // [dk][dk + 1]
  float* cur = Ms + dk * (dk + 1);  // [dk][kScanCols]
  float* nxt = cur + dk * kScanCols;
  const size_t st = (size_t)dk * dv;
  for (int e = tid; e < dk * kScanCols; e += kScanThreads) {
    const int i = e / kScanCols, jj = e % kScanCols;
    cur[e] = (is_m && jj < nc && i == j0 + jj) ? 1.f : 0.f;
  }
  const int row = tid >> 1, c0 = (tid & 1) * 8;
  for (int p = 0; p < k; ++p) {
    const size_t piece = (size_t)seg * k + p;
    const float* Mg = a.M + (piece * H + h) * (size_t)dk * dk;
    __syncthreads();
    for (int e = tid; e < dk * dk; e += kScanThreads) Ms[(e / dk) * (dk + 1) + e % dk] = Mg[e];
    __syncthreads();
    for (int r = row; r < dk; r += kScanThreads / 2) {
      float acc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = 0.f;
      const float* mrow = Ms + r * (dk + 1);
      for (int l = 0; l < dk; ++l) {
        const float m = mrow[l];
        const float* cr = cur + l * kScanCols + c0;
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = fmaf(m, cr[u], acc[u]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int jj = c0 + u;
        if (jj >= nc) continue;
        nxt[r * kScanCols + jj] =
            is_m ? acc[u] : acc[u] + a.U[(piece * H + h) * st + state_off(r, j0 + jj, dk, dv, a.v_first)];
      }
    }
    __syncthreads();
    float* t = cur;
    cur = nxt;
    nxt = t;
  }
  for (int e = tid; e < dk * kScanCols; e += kScanThreads) {
    const int i = e / kScanCols, jj = e % kScanCols;
    if (jj >= nc) continue;
    if (is_m) {
      a.M_out[((size_t)seg * H + h) * (size_t)dk * dk + (size_t)i * dk + j0 + jj] = cur[e];
    } else {
      const size_t o = state_off(i, j0 + jj, dk, dv, a.v_first);
      a.U_out[((size_t)seg * H + h) * st + o] = cur[e];
      if (!a.inc) continue;
      a.incoming[((size_t)seg * H + h) * st + o] = a.inc[((size_t)seg * k * H + h) * st + o];
      a.outgoing[((size_t)seg * H + h) * st + o] =
          seg + 1 < a.N ? a.inc[((size_t)(seg + 1) * k * H + h) * st + o] : a.final_state[(size_t)h * st + o];
    }
  }
}

cudaError_t launch_compose_pieces(const ComposeArgs& a, cudaStream_t stream) {
  if (tiles128(a.dk, a.dv)) {
    const int smem = (128 * 132 + 2 * 128 * 40) * (int)sizeof(float);  // M, carried tile parts
    cudaError_t err = cudaFuncSetAttribute(compose128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    compose128_kernel<<<dim3(a.H, 4 + a.dv / 32, a.N), 256, smem, stream>>>(a);
    return cudaGetLastError();
  }
  const size_t smem = ((size_t)a.dk * (a.dk + 1) + 2 * (size_t)a.dk * kScanCols) * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(compose_pieces_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid(a.H, (a.dk + kScanCols - 1) / kScanCols + (a.dv + kScanCols - 1) / kScanCols, a.N);
  compose_pieces_kernel<<<grid, kScanThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// dk = 128 forms of the scan and of the composition: 128 x 32 tiles.  M is staged row-major in
// shared memory by 16-byte asynchronous copies (double-buffered along the scan).  The tile
// product runs on the tensor cores as tf32 mma.sync (m16n8k8) with the three-term split
// a b = a_hi b_hi + a_hi b_lo + a_lo b_hi (a_hi = a rounded to tf32, a_lo = the remainder, also
// rounded; the dropped a_lo b_lo is below fp32 rounding), so the products keep fp32 accuracy.
// Thread ownership is the MMA accumulator fragment: warp w owns rows 16 w + g and 16 w + g + 8
// (g = lane / 4), columns 8 n + 2 t and + 1 (t = lane % 4, n < 4) -- sixteen values.
// ------------------------------------------------------------------------------------------
constexpr int kT = 32;          // tile columns
constexpr int kLdM = 132;       // padded row of the staged M: 16-byte rows, conflict-free fragment reads
constexpr int kLdC = 40;        // padded row of the carried tile's two parts: conflict-free fragment reads
constexpr int kTileThreads = 256;

__device__ __forceinline__ void cp_async16_g2s(float* dst, const float* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_groups() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// M (128 x 128 fp32, row-major in global memory) into a padded shared tile
__device__ __forceinline__ void stage_m(float* Ms, const float* Mg) {
  for (int e = threadIdx.x; e < 128 * 32; e += kTileThreads) {
    const int r = e >> 5, c = (e & 31) * 4;
    cp_async16_g2s(Ms + r * kLdM + c, Mg + r * 128 + c);
  }
  cp_async_commit_group();
}

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t u;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(u) : "f"(x));
  return u;
}

// the carried 128 x 8 NT tile X (NT 8-column MMA tiles), as its tf32 high part (chi) and
// rounded remainder (clo), from this thread's fragment x[n][c]
template <int NT>
__device__ __forceinline__ void put_carried(float* chi, float* clo, const float (&x)[NT][4]) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = 16 * w + g + 8 * hh, c = 8 * n + 2 * t;
      const float a = x[n][2 * hh], b = x[n][2 * hh + 1];
      const float ah = __uint_as_float(tf32_rna(a)), bh = __uint_as_float(tf32_rna(b));
      *reinterpret_cast<float2*>(chi + r * kLdC + c) = make_float2(ah, bh);
      *reinterpret_cast<float2*>(clo + r * kLdC + c) =
          make_float2(__uint_as_float(tf32_rna(a - ah)), __uint_as_float(tf32_rna(b - bh)));
    }
}

// acc = Ms (128 x 128, row-major, stride kLdM) times X (128 x 8 NT, held as chi + clo)
template <int NT>
__device__ __forceinline__ void tile_product_tc(const float* Ms, const float* chi, const float* clo,
                                                float (&acc)[NT][4]) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[n][u] = 0.f;
  const float* a0p = Ms + (16 * w + g) * kLdM;
  const float* a1p = a0p + 8 * kLdM;
#pragma unroll 4
  for (int k0 = 0; k0 < 128; k0 += 8) {
    const float av[4] = {a0p[k0 + t], a1p[k0 + t], a0p[k0 + t + 4], a1p[k0 + t + 4]};
    uint32_t ah[4], al[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ah[i] = tf32_rna(av[i]);
      al[i] = tf32_rna(av[i] - __uint_as_float(ah[i]));
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int c = 8 * n + g;
      const uint32_t bh0 = __float_as_uint(chi[(k0 + t) * kLdC + c]), bh1 = __float_as_uint(chi[(k0 + t + 4) * kLdC + c]);
      const uint32_t bl0 = __float_as_uint(clo[(k0 + t) * kLdC + c]), bl1 = __float_as_uint(clo[(k0 + t + 4) * kLdC + c]);
      sm100::mma1688_tf32(acc[n], al[0], al[1], al[2], al[3], bh0, bh1);
      sm100::mma1688_tf32(acc[n], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
      sm100::mma1688_tf32(acc[n], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
    }
  }
}

// two consecutive columns j, j + 1 of row r of a state block in either layout
__device__ __forceinline__ float2 load_state2(const float* blk, int r, int j, int dv, int v_first) {
  if (!v_first) return *reinterpret_cast<const float2*>(blk + (size_t)r * dv + j);
  return make_float2(blk[(size_t)j * 128 + r], blk[(size_t)(j + 1) * 128 + r]);
}
__device__ __forceinline__ void store_state2(float* blk, int r, int j, int dv, int v_first, float2 x) {
  if (!v_first) {
    *reinterpret_cast<float2*>(blk + (size_t)r * dv + j) = x;
  } else {
    blk[(size_t)j * 128 + r] = x.x;
    blk[(size_t)(j + 1) * 128 + r] = x.y;
  }
}
// this thread's fragment of columns j0 .. j0 + 8 NT - 1 of a state block
template <int NT>
__device__ __forceinline__ void load_frag(float (&x)[NT][4], const float* blk, int j0, int dv, int v_first) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float2 v = load_state2(blk, 16 * w + g + 8 * hh, j0 + 8 * n + 2 * t, dv, v_first);
      x[n][2 * hh] = v.x;
      x[n][2 * hh + 1] = v.y;
    }
}
template <int NT>
__device__ __forceinline__ void store_frag(float* blk, const float (&x)[NT][4], int j0, int dv, int v_first) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
      store_state2(blk, 16 * w + g + 8 * hh, j0 + 8 * n + 2 * t, dv, v_first,
                   make_float2(x[n][2 * hh], x[n][2 * hh + 1]));
}

// the exclusive scan (as affine_scan_kernel) for dk = 128: one block per (head, 8 NT columns)
template <int NT>
__global__ void __launch_bounds__(kTileThreads, 1) affine_scan128_kernel(ScanArgs a) {
  extern __shared__ __align__(16) float smf[];
  float* Ms0 = smf;
  float* Ms1 = Ms0 + 128 * kLdM;
  float* chi = Ms1 + 128 * kLdM;  // [128][kLdC] the carried tile, tf32 high part
  float* clo = chi + 128 * kLdC;  // and remainder
  const int h = blockIdx.x, j0 = blockIdx.y * 8 * NT, H = a.H, dv = a.dv, vf = a.v_first;
  const size_t st = (size_t)128 * dv;
  if (a.N > 0) stage_m(Ms0, a.M + (size_t)h * 128 * 128);
  float x[NT][4];  // this thread's part of the carried state
  load_frag(x, a.initial + (size_t)h * st, j0, dv, vf);
  float un[NT][4];  // the next step's contribution, loaded one step ahead
  if (a.N > 0) load_frag(un, a.U + (size_t)h * st, j0, dv, vf);
  for (int s = 0; s < a.N; ++s) {
    float* Ms = (s & 1) ? Ms1 : Ms0;
    const size_t blk = ((size_t)s * H + h) * st;
    float u[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) u[n][c] = un[n][c];
    if (s + 1 < a.N) load_frag(un, a.U + ((size_t)(s + 1) * H + h) * st, j0, dv, vf);
    put_carried(chi, clo, x);
    if (a.incoming) store_frag(a.incoming + blk, x, j0, dv, vf);
    if (s + 1 < a.N) {
      stage_m((s & 1) ? Ms0 : Ms1, a.M + ((size_t)(s + 1) * H + h) * 128 * 128);
      cp_async_wait_groups<1>();
    } else {
      cp_async_wait_groups<0>();
    }
    __syncthreads();  // M_s staged, the carried tile complete
    float acc[NT][4];
    tile_product_tc(Ms, chi, clo, acc);
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) x[n][c] = acc[n][c] + u[n][c];
    if (a.outgoing) store_frag(a.outgoing + blk, x, j0, dv, vf);
    __syncthreads();  // every read of the carried tile and of M_s is done
  }
  if (a.final_state) store_frag(a.final_state + (size_t)h * st, x, j0, dv, vf);
}

// the composition (as compose_pieces_kernel) for dk = 128: one block per (head, 32 columns of
// M or of U, segment); the first piece's map is the starting tile
__global__ void __launch_bounds__(kTileThreads, 2) compose128_kernel(ComposeArgs a) {
  extern __shared__ __align__(16) float smf[];
  float* Ms = smf;
  float* chi = Ms + 128 * kLdM;
  float* clo = chi + 128 * kLdC;
  const int h = blockIdx.x, seg = blockIdx.z, H = a.H, dv = a.dv, vf = a.v_first, k = a.k;
  const int nbm = 128 / kT;
  const bool is_m = (int)blockIdx.y < nbm;
  const int j0 = (is_m ? (int)blockIdx.y : (int)blockIdx.y - nbm) * kT;
  const size_t st = (size_t)128 * dv;
  const size_t first = (size_t)seg * k;
  float x[4][4];
  if (is_m)
    load_frag(x, a.M + (first * H + h) * 128 * 128, j0, 128, 0);  // M is row-major [128][128]
  else
    load_frag(x, a.U + (first * H + h) * st, j0, dv, vf);
  for (int p = 1; p < k; ++p) {
    const size_t piece = first + p;
    stage_m(Ms, a.M + (piece * H + h) * 128 * 128);
    float u[4][4];
    put_carried(chi, clo, x);
    if (is_m) {
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) u[n][c] = 0.f;
    } else {
      load_frag(u, a.U + (piece * H + h) * st, j0, dv, vf);
    }
    cp_async_wait_groups<0>();
    __syncthreads();
    float acc[4][4];
    tile_product_tc(Ms, chi, clo, acc);
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) x[n][c] = acc[n][c] + u[n][c];
    __syncthreads();
  }
  const size_t ob = ((size_t)seg * H + h) * st;
  if (is_m) {
    store_frag(a.M_out + ((size_t)seg * H + h) * 128 * 128, x, j0, 128, 0);
  } else {
    store_frag(a.U_out + ob, x, j0, dv, vf);
    if (!a.inc) return;
    float y[4][4];
    load_frag(y, a.inc + (first * H + h) * st, j0, dv, vf);
    store_frag(a.incoming + ob, y, j0, dv, vf);
    const float* nxt = seg + 1 < a.N ? a.inc + ((size_t)(seg + 1) * k * H + h) * st : a.final_state + (size_t)h * st;
    load_frag(y, nxt, j0, dv, vf);
    store_frag(a.outgoing + ob, y, j0, dv, vf);
  }
}

bool tiles128(int dk, int dv) { return dk == 128 && dv % kT == 0 && dv <= 128; }

// whether 16-column tiles (twice the blocks of 32-column ones) still fit the SMs in one wave
bool narrow_tiles(int64_t blocks32) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return false;
  return 2 * blocks32 <= sms;
}

cudaError_t launch_affine_scan128(const ScanArgs& a, cudaStream_t stream) {
  const int smem = (2 * 128 * kLdM + 2 * 128 * kLdC) * (int)sizeof(float);  // M double buffer, carried tile parts
  if (narrow_tiles((int64_t)a.H * (a.dv / 32))) {
    cudaError_t err = cudaFuncSetAttribute(affine_scan128_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    affine_scan128_kernel<2><<<dim3(a.H, a.dv / 16), kTileThreads, smem, stream>>>(a);
  } else {
    cudaError_t err = cudaFuncSetAttribute(affine_scan128_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    affine_scan128_kernel<4><<<dim3(a.H, a.dv / kT), kTileThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// The exclusive scan in log depth ("KDA Context Parallelism", Compose segments in sequence
// order: the composition is associative, so the ordered prefix can be formed as a parallel
// prefix).  Hillis-Steele over the maps: level l (stride s = 2^l) replaces every prefix
// P_i (i >= s) by P_i o P_{i-s} = (M_i M_{i-s}, M_i U_{i-s} + U_i), so after ceil(log2 N) levels
// P_i = F_i o ... o F_0; one more pass applies every prefix to the initial state:
// outgoing_i = M_{0..i} S_init + U_{0..i}, incoming_{i+1} = outgoing_i, incoming_0 = S_init.
// Each level is a batch of 128 x 128 x 32 tile products (the same fp32-accurate tf32 split as the
// sequential scan's); the work grows to N log N products against the sequential scan's N, so it
// pays only where the sequential scan leaves the GPU idle: few heads, many segments.
// ------------------------------------------------------------------------------------------

// one level: block per (head, 32-column tile of M or of U, map i); prefixes below the stride are
// copied unchanged
__global__ void __launch_bounds__(kTileThreads, 2) scan_level128_kernel(ScanLevelArgs a) {
  extern __shared__ __align__(16) float smf[];
  float* Ms = smf;
  float* chi = Ms + 128 * kLdM;
  float* clo = chi + 128 * kLdC;
  const int h = blockIdx.x, i = blockIdx.z, H = a.H, dv = a.dv, vf = a.v_first, s = a.stride;
  const int nbm = 128 / kT;
  const bool is_m = (int)blockIdx.y < nbm;
  const int j0 = (is_m ? (int)blockIdx.y : (int)blockIdx.y - nbm) * kT;
  const size_t st = (size_t)128 * dv, mm = (size_t)128 * 128;
  const size_t bi = (size_t)i * H + h;
  float x[4][4];
  if (i < s) {
    if (is_m) {
      load_frag(x, a.M + bi * mm, j0, 128, 0);
      store_frag(a.M_out + bi * mm, x, j0, 128, 0);
    } else {
      load_frag(x, a.U + bi * st, j0, dv, vf);
      store_frag(a.U_out + bi * st, x, j0, dv, vf);
    }
    return;
  }
  const size_t be = (size_t)(i - s) * H + h;  // the earlier prefix
  stage_m(Ms, a.M + bi * mm);                 // the later prefix's transition, applied on the left
  if (is_m)
    load_frag(x, a.M + be * mm, j0, 128, 0);
  else
    load_frag(x, a.U + be * st, j0, dv, vf);
  put_carried(chi, clo, x);
  float u[4][4];
  if (is_m) {
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) u[n][c] = 0.f;
  } else {
    load_frag(u, a.U + bi * st, j0, dv, vf);
  }
  cp_async_wait_groups<0>();
  __syncthreads();
  float acc[4][4];
  tile_product_tc(Ms, chi, clo, acc);
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) x[n][c] = acc[n][c] + u[n][c];
  if (is_m)
    store_frag(a.M_out + bi * mm, x, j0, 128, 0);
  else
    store_frag(a.U_out + bi * st, x, j0, dv, vf);
}

// the prefixes applied to the initial state: block per (head, 32-column tile of the state, i)
__global__ void __launch_bounds__(kTileThreads, 2) scan_apply128_kernel(ScanArgs a) {
  extern __shared__ __align__(16) float smf[];
  float* Ms = smf;
  float* chi = Ms + 128 * kLdM;
  float* clo = chi + 128 * kLdC;
  const int h = blockIdx.x, j0 = blockIdx.y * kT, i = blockIdx.z, H = a.H, dv = a.dv, vf = a.v_first;
  const size_t st = (size_t)128 * dv;
  const size_t bi = (size_t)i * H + h;
  stage_m(Ms, a.M + bi * 128 * 128);
  float x[4][4], u[4][4];
  load_frag(x, a.initial + (size_t)h * st, j0, dv, vf);
  if (i == 0 && a.incoming) store_frag(a.incoming + (size_t)h * st, x, j0, dv, vf);
  put_carried(chi, clo, x);
  load_frag(u, a.U + bi * st, j0, dv, vf);
  cp_async_wait_groups<0>();
  __syncthreads();
  float acc[4][4];
  tile_product_tc(Ms, chi, clo, acc);
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) x[n][c] = acc[n][c] + u[n][c];
  if (a.outgoing) store_frag(a.outgoing + bi * st, x, j0, dv, vf);
  if (i + 1 < a.N && a.incoming) store_frag(a.incoming + (bi + H) * st, x, j0, dv, vf);
  if (i + 1 == a.N && a.final_state) store_frag(a.final_state + (size_t)h * st, x, j0, dv, vf);
}

size_t logdepth_scan_bytes(int N, int H, int dk, int dv) {
  if (!tiles128(dk, dv) || N < 1 || H < 1) return 0;
  return 2 * (size_t)N * H * ((size_t)128 * 128 + (size_t)128 * dv) * sizeof(float);
}

// whether the log-depth scan is expected to finish first: both scans are counted in rounds of
// tile products over the GPU (two blocks per SM); the sequential scan takes N rounds of at least
// one, the log-depth scan a round count per level from its blocks, plus the application to the
// initial state.  A level's round measured 2.3 times a sequential step on B200 (a level block
// stages its own M and both prefixes; a scan step's M is prefetched during the previous one):
// 1 head: 128 maps 0.21 ms against 0.40 ms, 1024 maps 1.88 ms against 3.13 ms; 4 heads, 128 maps:
// 0.68 ms against 0.40 ms; 32 heads, 128 maps: 5.06 ms against 0.54 ms.
bool logdepth_scan_preferred(int N, int H, int dv) {
  if (N < 4) return false;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess || sms <= 0)
    return false;
  const double slots = 2.0 * sms;
  const double seq_blocks = (double)H * (dv / kT);
  const double t_seq = (double)N * std::ceil(seq_blocks / slots);
  double t_log = 0.0;
  for (int s = 1; s < N; s *= 2) t_log += std::ceil((double)(N - s) * H * (4 + dv / kT) / slots);
  t_log += std::ceil((double)N * H * (dv / kT) / slots);
  return 2.3 * t_log < 0.9 * t_seq;
}

cudaError_t launch_affine_scan_logdepth(const ScanArgs& a, float* work, cudaStream_t stream) {
  const int smem = (128 * kLdM + 2 * 128 * kLdC) * (int)sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(scan_level128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(scan_apply128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const size_t mblk = (size_t)a.N * a.H * 128 * 128, ublk = (size_t)a.N * a.H * 128 * a.dv;
  float* bufM[2] = {work, work + mblk + ublk};
  float* bufU[2] = {work + mblk, work + 2 * mblk + ublk};
  ScanLevelArgs l{};
  l.M = a.M;
  l.U = a.U;
  l.N = a.N;
  l.H = a.H;
  l.dv = a.dv;
  l.v_first = a.v_first;
  int b = 0;
  for (int s = 1; s < a.N; s *= 2, b ^= 1) {
    l.stride = s;
    l.M_out = bufM[b];
    l.U_out = bufU[b];
    scan_level128_kernel<<<dim3(a.H, 4 + a.dv / kT, a.N), kTileThreads, smem, stream>>>(l);
    l.M = l.M_out;
    l.U = l.U_out;
  }
  ScanArgs p = a;
  p.M = l.M;
  p.U = l.U;
  scan_apply128_kernel<<<dim3(a.H, a.dv / kT, a.N), kTileThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// A varlen batch as pieces: every sequence cut into chunk-aligned pieces of at most piece_len
// tokens (an empty sequence keeps one empty piece), so that a prefill of few or uneven
// sequences has as many chains as the SMs need; the pieces are built, applied in order from
// each sequence's pool slot, and read out ("KDA Context Parallelism": any cut is a segment
// boundary).
// ------------------------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) plan_pieces_kernel(PlanArgs a) {
  __shared__ int s_bad;
  __shared__ int s_carry;
  __shared__ int s_warp[kPlanThreads / 32];
  __shared__ unsigned long long s_chunks;
  __shared__ int s_max_chunks;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) {
    s_bad = 0;
    s_carry = 0;
    s_chunks = 0;
    s_max_chunks = 0;
  }
  __syncthreads();
  for (int b = tid; b < a.batch; b += kPlanThreads) {
    const int64_t t0 = a.cu[b], t1 = a.cu[b + 1];
    const int32_t slot = a.slots ? a.slots[b] : b;
    if (t0 < 0 || t1 < t0 || t1 > a.total_tokens || slot < 0 || slot >= a.max_slots) {
      s_bad = 1;
    } else {
      const int nch = (int)((t1 - t0 + 63) / 64);
      atomicAdd(&s_chunks, (unsigned long long)nch);
      atomicMax(&s_max_chunks, nch);
    }
  }
  __syncthreads();
  // chunk steps on the SMs (one chain per SM): the plain schedule cannot beat its longest
  // sequence nor the total work; the pieces are no longer than piece_len, but a piece's chunk
  // carries two states and two readouts (taken as 1.25 chunk steps) and the scan and the apply
  // add about 12 chunk steps
  const double work = (double)s_chunks * a.num_heads / a.num_sms;
  const double plain = fmax((double)s_max_chunks, work);
  const double split = 1.25 * fmax((double)(a.piece_len / 64), work) + 12.0;
  if (s_bad || !(split < 0.9 * plain)) {  // the plain kernel runs instead (and reports what is wrong)
    if (tid == 0) *a.fallback = 1;
    return;
  }
  const int P = a.piece_len;
  for (int base = 0; base < a.batch; base += kPlanThreads) {
    const int b = base + tid;
    int n = 0;
    int64_t t0 = 0, len = 0;
    if (b < a.batch) {
      t0 = a.cu[b];
      len = a.cu[b + 1] - t0;
      n = len > 0 ? (int)((len + P - 1) / P) : 1;
    }
    // inclusive block scan of n
    int x = n;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) s_warp[w] = x;
    __syncthreads();
    if (w == 0) {
      int v = s_warp[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += y;
      }
      s_warp[lane] = v;
    }
    __syncthreads();
    const int incl = x + (w > 0 ? s_warp[w - 1] : 0);
    const int first = s_carry + incl - n;
    if (b < a.batch) {
      a.seq_first[b] = first;
      for (int j = 0; j < n && first + j < a.max_pieces; ++j) a.piece_offs[first + j] = (int32_t)(t0 + (int64_t)j * P);
    }
    __syncthreads();
    if (tid == kPlanThreads - 1) s_carry += incl;
    __syncthreads();
  }
  const int total = s_carry;
  if (total > a.max_pieces) {  // cannot happen for max_pieces >= batch + ceil(total_tokens / piece_len)
    if (tid == 0) *a.fallback = 1;
    return;
  }
  if (tid == 0) {
    a.seq_first[a.batch] = total;
    *a.fallback = 0;
  }
  const int32_t end = a.batch > 0 ? a.cu[a.batch] : 0;
  for (int i = total + tid; i <= a.max_pieces; i += kPlanThreads) a.piece_offs[i] = end;
}

cudaError_t launch_plan_pieces(const PlanArgs& a, cudaStream_t stream) {
  plan_pieces_kernel<<<1, kPlanThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

// one block per (head, 32 columns, sequence): the sequence's pieces applied in order to its
// pool state, each piece's incoming state recorded, the final state written back
template <int NT>
__global__ void __launch_bounds__(kTileThreads, 1) pool_scan128_kernel(PoolScanArgs a) {
  if (*a.fallback) return;
  extern __shared__ __align__(16) float smf[];
  float* Ms0 = smf;
  float* Ms1 = Ms0 + 128 * kLdM;
  float* chi = Ms1 + 128 * kLdM;
  float* clo = chi + 128 * kLdC;
  const int h = blockIdx.x, j0 = blockIdx.y * 8 * NT, b = blockIdx.z, H = a.H, dv = a.dv, vf = a.v_first;
  const size_t st = (size_t)128 * dv;
  const int p0 = a.seq_first[b], p1 = a.seq_first[b + 1];
  const int32_t slot = a.slots ? a.slots[b] : b;
  float* blk = a.pool + ((size_t)slot * H + h) * st;
  if (p1 > p0) stage_m(Ms0, a.M + ((size_t)p0 * H + h) * 128 * 128);
  float x[NT][4];
  load_frag(x, blk, j0, dv, vf);
  float un[NT][4];  // the next piece's contribution, loaded one step ahead
  if (p1 > p0) load_frag(un, a.U + ((size_t)p0 * H + h) * st, j0, dv, vf);
  for (int p = p0; p < p1; ++p) {
    const int s = p - p0;
    float* Ms = (s & 1) ? Ms1 : Ms0;
    const size_t pb = ((size_t)p * H + h) * st;
    float u[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) u[n][c] = un[n][c];
    if (p + 1 < p1) load_frag(un, a.U + ((size_t)(p + 1) * H + h) * st, j0, dv, vf);
    put_carried(chi, clo, x);
    store_frag(a.incoming + pb, x, j0, dv, vf);
    if (p + 1 < p1) {
      stage_m((s & 1) ? Ms0 : Ms1, a.M + ((size_t)(p + 1) * H + h) * 128 * 128);
      cp_async_wait_groups<1>();
    } else {
      cp_async_wait_groups<0>();
    }
    __syncthreads();
    float acc[NT][4];
    tile_product_tc(Ms, chi, clo, acc);
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) x[n][c] = acc[n][c] + u[n][c];
    __syncthreads();
  }
  store_frag(blk, x, j0, dv, vf);
}

cudaError_t launch_pool_scan(const PoolScanArgs& a, cudaStream_t stream) {
  const int smem = (2 * 128 * kLdM + 2 * 128 * kLdC) * (int)sizeof(float);
  if (a.batch == 0) return cudaSuccess;
  // the scan is bound per SM by its tile products: with blocks to spare for the SMs, 16-column
  // tiles spread the same products over twice the blocks
  if (narrow_tiles((int64_t)a.H * (a.dv / 32) * a.batch)) {
    cudaError_t err = cudaFuncSetAttribute(pool_scan128_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    pool_scan128_kernel<2><<<dim3(a.H, a.dv / 16, a.batch), kTileThreads, smem, stream>>>(a);
  } else {
    cudaError_t err = cudaFuncSetAttribute(pool_scan128_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    pool_scan128_kernel<4><<<dim3(a.H, a.dv / kT, a.batch), kTileThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace kda
