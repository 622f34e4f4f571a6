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
#include "kda_common.cuh"
#include "kda_internal.h"

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
// One block per (head, 32-column tile of the state); the segment loop is serial.
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

cudaError_t launch_affine_scan(const ScanArgs& a, cudaStream_t stream) {
  const size_t smem = ((size_t)a.dk * (a.dk + 1) + 2 * (size_t)a.dk * kScanCols) * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(affine_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid(a.H, (a.dv + kScanCols - 1) / kScanCols);
  affine_scan_kernel<<<grid, kScanThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
