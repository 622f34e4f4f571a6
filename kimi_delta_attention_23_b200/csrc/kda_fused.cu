// kda_fused.cu -- fused chunk-parallel KDA prefill for bf16 q/k/v, dk = dv = 128, on sm_100a.
//
// One CTA owns one (sequence, value head) chain and walks its 64-token chunks in order.  With
// S0 the state entering a chunk, positions r, s in [0, 64), per-channel decays a_t = exp(g_t)
// and Gamma_r = prod_{u<=r} a_u, the per-token step (decay, delta write predicting from the
// decayed state, readout: "nx_nofloat_kda.nx source", kda_forward) unrolls to
//
//   A_rs  = sum_i k_ri k_si prod_{u=s+1..r} a_ui          (s < r)     gated key scores
//   P_rs  = sum_i q_ri k_si prod_{u=s+1..r} a_ui          (s <= r)    gated query scores
//   T     = (I + diag(beta) A)^{-1} diag(beta)                         UT factor
//   X     = V - (K o Gamma) S0
//   Delta = T X
//   O     = (Q o Gamma) S0 + P Delta
//   S1    = Diag(Gamma_63) S0 + K'^T Delta,     K'_s = k_s o prod_{u>s} a_u
//
// (GStar Assignment 2, Learning path: P4 gate prefix scan, P6 triangular inverse, P8 stable
// score builder, P9 the assembled chunked forward; "max.nn.state_space.kda_chunk": chunk-
// parallel prefill mutating the state pool.)  Every factor above is a product of decays, so
// every operand is <= 1 in magnitude and nothing can overflow, whatever the gate.
//
// Two warp teams share the CTA (512 threads) and work one chunk apart:
//   * the key team (warps 0-7) does everything that does not touch the state.  It reads a
//     chunk's raw gates, keys and queries from global memory straight into registers (an L2
//     prefetch runs one or two chunks ahead), forms the decays, the 8x8 diagonal score blocks on CUDA
//     cores (a product recursion along the rows), the operand tiles, the off-diagonal scores
//     with mma.sync on operands scaled by a reference point that sits between rows and columns
//     (both factors <= 1), and the inverses of the 8x8 diagonal blocks;
//   * the state team (warps 8-15) combines those into T (16-blocks in fp32, then two tf32
//     mma.sync doubling levels) and runs the four products that touch S on tcgen05 with the
//     state transposed (dv = 128 rows = the 128 TMEM lanes): D1 = S^T [K o Gamma; Q o Gamma]^T,
//     D2 = X^T T^T, D1o += Delta^T P^T, S^T += Delta^T K'.  S^T stays in TMEM in fp32 across
//     chunks; a bf16 copy, also in TMEM, is the A operand of the next chunk's first product.
//     The team also decays the state, runs the epilogues (two warps per TMEM lane quadrant),
//     stages the outputs and issues V's tensor copies and the output stores.
// While the state team finishes chunk n, the key team is already on chunk n + 1.  They hand
// over through mbarriers: tiles ready and scores ready (key -> state); the inverse done and the
// products' completions, which free the shared tiles for the next chunk (state -> key).  Each
// team synchronises on its own named barrier; no barrier spans both teams in the chunk loop.
#include <cuda.h>
#include <string.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;          // chunk length
constexpr int D = 128;         // dk = dv
constexpr int kTeam = 256;     // threads per team
constexpr int kThreads = 2 * kTeam;  // key team: warps 0-7; state team: warps 8-15
constexpr int kKeyBar = 1, kStateBar = 2;  // the teams' named barriers
// registers per thread once the teams split; the two shares add up to the launch's 512 x 128.
// The build carries two states, so its state team has twice the epilogue work and gets more of
// them (measured: 184 / 72 there, 200 / 56 in the prefill; 8 fewer on either side costs more
// than 8 more on the other gains).
constexpr uint32_t kLaunchRegs = 128;
template <bool kBuild>
struct RegSplit {
  static constexpr uint32_t key = kBuild ? 184 : 200, state = kBuild ? 72 : 56;
  static_assert(kTeam * (key + state) == kThreads * kLaunchRegs, "register split");
};
// the state team's threads (index within the team) that issue the chunk's tensor-core products,
// one per group of products (each commits its own), and the one that issues copies and stores
constexpr int kIssueFirst = 192;   // D1 = S^T [K o Gamma ; Q o Gamma]^T          (team warp 6)
constexpr int kIssueDelta = 224;   // Delta = (V - (K o Gamma) S0) T             (team warp 7)
constexpr int kIssueRead = 128;    // readouts / outputs                          (team warp 4)
constexpr int kIssueUpdate = 160;  // state updates S += K'^T Delta               (team warp 5)
constexpr int kCopyThread = 160;   // V's tensor copies and the output stores
constexpr uint32_t kTmemCols = 512;  // D1 [0,128), S fp32 [128,256), S bf16 A operand [256,320)
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far beyond any legitimate wait

// shared-memory map (bytes from a 1024-aligned base); bf16 operand tiles use the K-major
// 128-byte swizzle layout (see sw_off)
constexpr int OFF_KQ = 0;                   // [K o Gamma ; Q o Gamma]   128 rows x 128 K     (key -> state)
constexpr int OFF_KPT = OFF_KQ + 32768;     // K'         64 rows x 128, the MN-major B operand K'^T
constexpr int OFF_X = OFF_KPT + 16384;      // X^T, then Delta^T   128 rows x 64 K; build: then the U readouts
constexpr int OFF_XM = OFF_X + 16384;       // build: X^T / Delta^T of the transition, then its readouts;
                                            // prefill: the staged outputs (bf16; fp32 from OFF_X on)
constexpr int OFF_V = OFF_XM + 16384;       // V as the MN-major A operand V^T (two 64-column halves, 8 KB
                                            // apart, 128B-swizzled by the tensor copy)
constexpr int OFF_T = OFF_V + 16384;        // T          64 rows x 64 K
constexpr int OFF_P = OFF_T + 8192;         // P          64 rows x 64 K, two buffers (chunk parity)
constexpr int OFF_KPI = OFF_P + 16384;      // K o pi     64 x 128 (rows scaled from their 16-block start)
constexpr int OFF_QPI = OFF_KPI + 16384;    // Q o pi
constexpr int OFF_KC = OFF_QPI + 16384;     // K o kappa  (columns scaled to their 16-block end)
constexpr int OFF_KPI8 = OFF_KC + 16384;    // 32 x 128: upper-half rows from the half start
constexpr int OFF_QPI8 = OFF_KPI8 + 8192;
constexpr int OFF_KK8 = OFF_QPI8 + 8192;    // 32 x 128: lower-half columns to the half end
constexpr int OFF_A = OFF_KK8 + 8192;       // fp32 [64][68] key scores
constexpr int OFF_TAU = OFF_A + 17408;      // fp32 [8][128] decay product of each 8-row block
constexpr int OFF_MP = OFF_TAU + 4096;      // bf16x2 [6][64] decay between 16-blocks of a pair
constexpr int OFF_BETA = OFF_MP + 1536;     // fp32 [2][64] beta (chunk parity)
constexpr int OFF_GC = OFF_BETA + 512;      // fp32 [2][128] Gamma of the last row (chunk parity)
constexpr int OFF_BAR = OFF_GC + 1024;      // mbarriers (+0..+71), TMEM base (+72), abort flag (+76),
                                            // the staged inputs' mbarrier (+80)
constexpr int kSmemBytes = OFF_BAR + 128;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for aligning the base to 1024
// Once the key team's scores of a chunk are done, the score tiles' region serves two users until
// the key team's next tiles: the state team's inverse works at its end, and the next chunk's raw
// gates and keys arrive at its start by tensor copies (the key team reads them there for its
// gates and in-block products)
constexpr int OFF_STG = OFF_KPI;            // raw gates, fp32 [64][128] (token rows)
constexpr int OFF_STG_K = OFF_STG + 32768;  // keys, bf16 [64][128]
constexpr int OFF_Y = OFF_A - 6144;         // fp32 inverse temporaries: [4][8][8] and [4][16][8], then
                                            // [32][32] after them
constexpr int OFF_XI = OFF_Y - 17408;       // fp32 [64][68] inverse
static_assert(OFF_STG_K + 16384 <= OFF_XI && OFF_XI >= OFF_KPI && OFF_XI % 1024 == 0,
              "staged inputs overlap the inverse's scratch");
constexpr int kLdA = 68;                    // row stride of the fp32 [64][*] arrays
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr float kLog2e = 1.4426950408889634f;

// byte offset of bf16 element (row, k) in a K-major 128B-swizzled tile with `rows` rows per
// 64-wide K block: 8-row atoms of 1024 bytes, 16-byte chunk c of row r stored at c ^ (r & 7)
__device__ __forceinline__ uint32_t sw_off(int row, int k, int rows) {
  const int kb = k >> 6, kin = k & 63;
  return (uint32_t)(kb * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 + ((((kin >> 3) ^ (row & 7))) << 4) +
                    ((kin & 7) << 1));
}

// T = X diag(beta) is written in bf16 as each block of the inverse X is completed; one entry, or
// two consecutive ones (s even), of the 64 x 64 tile (K-major, 128B swizzle)
__device__ __forceinline__ void put_t1(uint8_t* sm_t, int r, int s, float v) {
  *reinterpret_cast<__nv_bfloat16*>(sm_t + sw_off(r, s, 64)) = __float2bfloat16_rn(v);
}
__device__ __forceinline__ void put_t2(uint8_t* sm_t, int r, int s, float v0, float v1) {
  *reinterpret_cast<uint32_t*>(sm_t + sw_off(r, s, 64)) = pack_bf16(v0, v1);
}

__device__ __forceinline__ uint2 pack4(float a, float b, float c, float d) {
  return make_uint2(pack_bf16(a, b), pack_bf16(c, d));
}

// two fp32 products in one instruction (each rounded to nearest, as two multiplies would be)
__device__ __forceinline__ float2 mul_f32x2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
// a . b over four channels held as two pairs (pairwise: (a0 b0 + a2 b2) + (a1 b1 + a3 b3))
__device__ __forceinline__ float dot4(float2 a01, float2 a23, float2 b01, float2 b23) {
  const float2 t = fma_f32x2(a23, b23, mul_f32x2(a01, b01));
  return t.x + t.y;
}
__device__ __forceinline__ uint2 pack4(float2 lo, float2 hi) {
  return make_uint2(pack_bf16(lo.x, lo.y), pack_bf16(hi.x, hi.y));
}

// two bf16 products in one instruction (each rounded to nearest)
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t x, uint32_t y) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(x), "r"(y));
  return d;
}

// slot -> (row, column) of the 8x8 diagonal-block scores, entry = row * 8 + column: slots 0..27
// are A (row > column), slots 28..63 are P -- 28..31 its diagonal rows 0..3, 32..59 its strictly
// lower part in A's order, 60..63 its diagonal rows 4..7 (slot i and i + 32 are partners of the
// reduction's first level)
__constant__ unsigned char kDiagPair[64] = {
    8,  16, 17, 24, 25, 26, 32, 33, 34, 35, 40, 41, 42, 43, 44, 48, 49, 50, 51, 52, 53, 56,
    57, 58, 59, 60, 61, 62, 0,  9,  18, 27, 8,  16, 17, 24, 25, 26, 32, 33, 34, 35, 40, 41,
    42, 43, 44, 48, 49, 50, 51, 52, 53, 56, 57, 58, 59, 60, 61, 62, 36, 45, 54, 63};

}  // namespace

// Tensor maps of the four token-major inputs, each viewed as [tokens][heads][128] with a box of
// 64 tokens x 1 head x 128 channels: V arrives by one tensor copy per chunk, the others are
// prefetched into L2 through theirs (the key team then reads them with plain loads).
struct InputMaps {
  CUtensorMap raw, k, q, v;
  CUtensorMap out, out2;  // bf16 outputs (readouts in the build), written by tensor stores
};

// kBuild = false: prefill (state from the pool, readout, state back to the pool).
// kBuild = true: segment build -- two states share every key-side product: the transition M
// (started at I, zero values) and the contribution U (started at 0, real values); no readout.
// kRead: the query side is present (scores P, Q o Gamma) and readouts are produced -- always
// in prefill; in the build, the readouts of both states (local outputs of the segment).
template <bool kBuild, bool kRead>
__global__ void __launch_bounds__(kThreads, 1) fused_chunk_kernel(const FusedArgs a, const __grid_constant__ InputMaps tm) {
  if (a.gate_flag && *a.gate_flag != a.gate_run_if) return;  // this launch is not the one that runs
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-aligned base, offset from the shared array itself so that every pointer derived from it
  // stays in the shared window (32-bit shared addressing instead of generic pointers)
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool key_team = warp < 8;
  const int h = blockIdx.x;
  int b = blockIdx.y;
  if constexpr (!kBuild) {
    // longest sequences first: blocks start in the order of blockIdx.y, and a batch's time is
    // bound by when its longest chains start, so block row y takes the sequence of rank y in
    // decreasing length (ties by index) -- for batches of at most kTeam sequences; the
    // lengths go through the score scratch, which no chunk has touched yet
    if (a.batch > 1 && a.batch <= kTeam) {
      int* s_len = reinterpret_cast<int*>(sm + OFF_A);
      volatile int* s_pick = reinterpret_cast<volatile int*>(sm + OFF_A + 4 * kTeam);
      for (int s = tid; s < a.batch; s += kThreads) s_len[s] = a.cu[s + 1] - a.cu[s];
      if (tid == 0) *s_pick = b;
      __syncthreads();
      if (tid < a.batch) {
        const int ls = s_len[tid];
        int rank = 0;
        for (int s2 = 0; s2 < a.batch; ++s2) {
          const int l2 = s_len[s2];
          rank += (l2 > ls || (l2 == ls && s2 < tid)) ? 1 : 0;
        }
        if (rank == (int)blockIdx.y) *s_pick = tid;
      }
      __syncthreads();
      b = *s_pick;
      __syncthreads();  // every read of the scratch and of the pick is done
    }
  }
  const int kh = h / (a.Hv / a.Hk);
  const bool safe = a.flags & KDA_GATE_SAFE, prob = a.flags & KDA_BETA_PROB;

  const int t0 = a.cu[b], t1 = a.cu[b + 1];  // token offsets (int32 like cu_seqlens)
  const int32_t slot = a.slots ? a.slots[b] : b;
  if (t0 < 0 || t1 < t0 || t1 > a.total_tokens || slot < 0 || slot >= a.max_slots) {
    if (tid == 0) report(a.status, KDA_ERR_DEVICE_CHECK);
    return;
  }

  const uint32_t sbase = smem_addr(sm);
  // bar0..bar4: completions of the chunk's product groups (bar3: the issuing threads' final
  // commits when a chunk loop is abandoned); bar_v: V's tensor copy; bar_tiles, bar_scores:
  // the key team's operand tiles and scores of a chunk are in place; bar_inv: the state team's
  // inverse of a chunk is done (sA and the inverse's scratch in the score tiles are free); bar_stg:
  // a chunk's raw gates and keys have been copied in
  const uint32_t bar0 = sbase + OFF_BAR, bar1 = bar0 + 8, bar2 = bar0 + 16, bar3 = bar0 + 24, bar4 = bar0 + 32;
  const uint32_t bar_v = bar0 + 40, bar_tiles = bar0 + 48, bar_scores = bar0 + 56, bar_inv = bar0 + 64;
  const uint32_t bar_stg = bar0 + 80;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 72);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + OFF_BAR + 76);
  float* sA = reinterpret_cast<float*>(sm + OFF_A);
  float* sTau = reinterpret_cast<float*>(sm + OFF_TAU);
  uint32_t* sMp = reinterpret_cast<uint32_t*>(sm + OFF_MP);
  float* sBeta = reinterpret_cast<float*>(sm + OFF_BETA);
  float* sGC = reinterpret_cast<float*>(sm + OFF_GC);

  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar1, 1);
    mbar_init(bar2, kBuild ? 2 : 1);  // build: one commit per state
    mbar_init(bar3, 4);
    mbar_init(bar4, kBuild ? 2 : 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_tiles, 1);
    mbar_init(bar_scores, 1);
    mbar_init(bar_inv, 1);
    mbar_init(bar_stg, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_addr(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // TMEM columns.  prefill: D1 [0,128) (X/Delta part, then O part), S fp32 [128,256), S bf16
  // [256,320), Delta^T bf16 [320,352) (the A operand of the output product and the update).
  // build: D1 of M [0,64) and of U [64,128), S_M [128,256), S_U [256,384), bf16 copies [384,448)
  // and [448,512).
  const uint32_t tmD1 = tmem, tmS = tmem + 128, tmSb = kBuild ? tmem + 384 : tmem + 256;
  const uint32_t tmDb = tmem + 320;
  const uint32_t tmD1u = tmem + 64, tmSu = tmem + 256, tmSbu = tmem + 448;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  constexpr bool qb = kRead;
  const bool has_v = kBuild || !a.values_zero;
  const size_t blk_off = ((size_t)slot * a.Hv + h) * (size_t)(D * D);
  const float* in_blk = a.state_in ? a.state_in + blk_off : nullptr;
  float* out_blk = a.state_out + blk_off;
  auto rows_of = [&](int c0n) { return (t1 - c0n) < C ? (t1 - c0n) : C; };

  if (!key_team) {
    // ---- the incoming state: S^T into TMEM (fp32) and its bf16 copy, the A operand of the first
    // chunk's first product; thread -> state row j (its TMEM lane), columns split between the two
    // warps of a quadrant
    const int sw = warp - 8;
    const int j = (sw & 3) * 32 + lane, ehalf = sw >> 2;
#pragma unroll 1
    for (int i0 = 64 * ehalf; i0 < 64 * ehalf + 64; i0 += 16) {
      float v[16];
      if (kBuild || a.init_mode != 0) {
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = ((kBuild || a.init_mode == 2) && i0 + u == j) ? 1.f : 0.f;
      } else if (a.v_first) {
        const float4* p = reinterpret_cast<const float4*>(in_blk + (size_t)j * D + i0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float4 f = p[q];
          v[4 * q] = f.x;
          v[4 * q + 1] = f.y;
          v[4 * q + 2] = f.z;
          v[4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = in_blk[(size_t)(i0 + u) * D + j];
      }
      tmem_st16(tmS + lane_base + i0, v);
      uint32_t pk[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) pk[q] = pack_bf16(v[2 * q], v[2 * q + 1]);
      tmem_st8u(tmSb + lane_base + i0 / 2, pk);
      if constexpr (kBuild) {  // the contribution starts at zero
        float z[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) z[u] = 0.f;
        const uint32_t zp[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        tmem_st16(tmSu + lane_base + i0, z);
        tmem_st8u(tmSbu + lane_base + i0 / 2, zp);
      }
    }
    tmem_wait_st();
  } else {
    // P's upper triangle (both buffers) must read as zero (A's upper triangle is never read as A);
    // no chunk writes there, so it is cleared once; likewise T's upper triangle: the inverse
    // writes only entries s <= r
    if constexpr (kRead)
      for (int e = tid; e < 2 * 8192 / 16; e += kTeam) reinterpret_cast<uint4*>(sm + OFF_P)[e] = make_uint4(0, 0, 0, 0);
    for (int e = tid; e < 8192 / 16; e += kTeam) reinterpret_cast<uint4*>(sm + OFF_T)[e] = make_uint4(0, 0, 0, 0);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();

  bool aborted = false;
  if (key_team) {
    regs_increase<RegSplit<kBuild>::key>();
    // ================================================================ key team
    // mapping: warp kw owns rows 8 kw .. 8 kw + 7 of a chunk, lane owns channels 4 lane .. + 3
    const int kw = warp;
    const int ch = lane * 4;
    const float4 dtb = *reinterpret_cast<const float4*>(a.dt_bias + (size_t)h * D + ch);
    const float cexp = expf(a.a_log[h]);
    const float alpha_floor = safe ? expf(a.lb) : 0.f;
    const int b16 = kw >> 1, upper = kw & 1;
    const size_t kq_stride = (size_t)a.Hk * D;
    const __nv_bfloat16* q_base = reinterpret_cast<const __nv_bfloat16*>(qb ? a.q : a.k) + (size_t)kh * D + ch;
    // A chunk's raw gates and keys arrive in shared memory by tensor copies, issued once the
    // previous chunk's scores are done (the copies then run under its state tiles); the queries
    // of this thread's rows and channels are read straight into registers.  Rows past the
    // sequence's end read as zero (keys, queries) or are never used (gates).  An L2 prefetch of
    // a later chunk's inputs runs ahead of both.
    uint2 k2[8], q2[8];
    float beta_raw = 0.f;  // beta of one row (lanes 0..7)
    auto issue_stage = [&](int c0n) {  // one thread
      mbar_arrive_expect_tx(bar_stg, 32768u + 16384u);
      tma_load_3d(sbase + OFF_STG, &tm.raw, 0, h, c0n, bar_stg);
      tma_load_3d(sbase + OFF_STG_K, &tm.k, 0, kh, c0n, bar_stg);
    };
    auto read_k = [&](int L) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int row = kw * 8 + r;
        k2[r] = row < L ? *reinterpret_cast<const uint2*>(sm + OFF_STG_K + (row * D + ch) * 2) : make_uint2(0u, 0u);
      }
    };
    auto load_q = [&](int c0n) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int t = c0n + kw * 8 + r;
        q2[r] = (qb && t < t1) ? __ldg(reinterpret_cast<const uint2*>(q_base + (size_t)t * kq_stride))
                               : make_uint2(0u, 0u);
      }
    };
    auto load_beta = [&](int c0n) {
      const int t = c0n + kw * 8 + lane;
      if (lane < 8 && t < t1) beta_raw = __ldg(a.beta + (size_t)t * a.Hv + h);
    };
    // the inputs of the chunk at c0n into L2 ahead of the plain loads above
    auto prefetch_l2 = [&](int c0n) {
      if (tid == 0 && c0n < t1) {
        tma_prefetch_l2_3d(&tm.raw, 0, h, c0n);
        tma_prefetch_l2_3d(&tm.k, 0, kh, c0n);
        if (qb) tma_prefetch_l2_3d(&tm.q, 0, kh, c0n);
      }
    };
    // L2 prefetch distance in chunks (measured: the prefill 1.90 -> 1.80 ms with one chunk on the
    // 64 x 2048-token batch; the segment build 4.79 -> 4.90 ms, so it keeps two)
    constexpr int kAhead = kBuild ? 2 : 1;
    bool stg_pending = false;  // a staging copy issued whose completion was not yet observed
    uint32_t stg_parity = 0;   // parity of the next completion on bar_stg
    if (t1 > t0) {
      if (kAhead > 1) prefetch_l2(t0 + C);
      if (tid == 0) issue_stage(t0);
      stg_pending = true;
    }
    uint32_t ci = 0;  // chunk index
#pragma unroll 1
    for (int c0 = t0; c0 < t1; c0 += C, ++ci) {
      const int L = rows_of(c0);
      const uint32_t par = ci & 1u;
      uint8_t* sP = sm + OFF_P + par * 8192;
      float* sBetaC = sBeta + par * 64;
      // this chunk's beta and queries, read into registers: the gates hide their latency
      // (measured: with the keys staged, the benchmark step 4.635 -> 4.585 ms against issuing the
      // build's queries after the gates)
      load_beta(c0);
      load_q(c0);
      prefetch_l2(c0 + kAhead * C);
      // this chunk's staged raw gates and keys
      if (!mbar_wait_bounded(bar_stg, stg_parity, kWaitLimitNs)) {
        *s_abort = 1;
        report(a.status, KDA_ERR_DEVICE_TIMEOUT);
      }
      stg_pending = false;
      stg_parity ^= 1u;

      // ---- gates of this chunk: alpha = exp(g), 1 past the sequence end
      float al[8][4];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int row = kw * 8 + r;
#pragma unroll
        for (int c = 0; c < 4; ++c) al[r][c] = 1.f;
        if (row < L) {
          const float4 raw = *reinterpret_cast<const float4*>(sm + OFF_STG + (row * D + ch) * 4);
          // softplus(x) in log2 units, log2(1 + 2^(x log2 e)), then alpha = exp(-exp(a_log)
          // softplus(x)) = 2^(-c sp2); the limits come out right on both sides (x large: the power
          // overflows to inf and alpha = 0; x very negative: it flushes to 0 and alpha = 1).  In the
          // build the plain arithmetic runs on channel pairs (the special functions one value at
          // a time); the prefill keeps one value at a time, which measured faster there.  The
          // roundings are the same either way.
          if constexpr (kBuild) {
#pragma unroll
            for (int c = 0; c < 4; c += 2) {
              const float2 x = add_f32x2(c ? make_float2(raw.z, raw.w) : make_float2(raw.x, raw.y),
                                         c ? make_float2(dtb.z, dtb.w) : make_float2(dtb.x, dtb.y));
              const float2 xl = mul_f32x2(x, make_float2(kLog2e, kLog2e));
              const float2 e = add_f32x2(make_float2(1.f, 1.f), make_float2(fast_ex2(xl.x), fast_ex2(xl.y)));
              const float2 y = mul_f32x2(make_float2(-cexp, -cexp), make_float2(fast_lg2(e.x), fast_lg2(e.y)));
              const float a0 = fast_ex2(y.x), a1 = fast_ex2(y.y);
              al[r][c] = safe ? fmaxf(a0, alpha_floor) : a0;
              al[r][c + 1] = safe ? fmaxf(a1, alpha_floor) : a1;
            }
          } else {
            const float xs[4] = {raw.x + dtb.x, raw.y + dtb.y, raw.z + dtb.z, raw.w + dtb.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float sp2 = fast_lg2(1.f + fast_ex2(xs[c] * kLog2e));
              const float al_c = fast_ex2(-cexp * sp2);
              al[r][c] = safe ? fmaxf(al_c, alpha_floor) : al_c;
            }
          }
        }
      }
      if (lane < 8) {
        const int row = kw * 8 + lane;
        sBetaC[row] = row < L ? beta_f32(beta_raw, prob) : 0.f;
      }

      read_k(L);
      // ---- part 1: in-block products.  k and q of my rows stay packed in registers (two bf16
      // per word) and are widened where they are used: widening is one instruction per value,
      // and the fp32 copies would hold 64 more registers through part 1 and the tiles
      auto klo = [&](int r) { return unpack_bf16(k2[r].x); };
      auto khi = [&](int r) { return unpack_bf16(k2[r].y); };
      auto qlo = [&](int r) { return unpack_bf16(q2[r].x); };
      auto qhi = [&](int r) { return unpack_bf16(q2[r].y); };
      // diagonal 8x8 blocks on CUDA cores: partial sums over my 4 channels of
      //   A_rs (r > s, slots 0..27) and P_rs (r >= s, slots 28..63), then a butterfly
      //   reduce-scatter over the 32 lanes leaves slots 2*lane and 2*lane+1 in this lane
      //   (build without queries: A only, 32 slots, slot lane in this lane).  A goes to the lower triangles of
      //   sA's diagonal blocks (read only by this team's 8x8 block inverses), P to this chunk's
      //   P buffer (last read by the products of the chunk before the previous one).
      if constexpr (!kRead) {
        float acc[32];
#pragma unroll
        for (int i = 28; i < 32; ++i) acc[i] = 0.f;
        // rows outer: w[s] = k_s o prod_{u=s+1..r} a_u is carried along the rows (the same
        // products in the same order as a column-by-column recursion), so only the current
        // row's k is widened at a time
        float2 w01[8], w23[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float2 k01 = klo(r), k23 = khi(r);
#pragma unroll
          for (int s = 0; s < r; ++s) {
            w01[s] = mul_f32x2(w01[s], make_float2(al[r][0], al[r][1]));
            w23[s] = mul_f32x2(w23[s], make_float2(al[r][2], al[r][3]));
            acc[r * (r - 1) / 2 + s] = dot4(k01, k23, w01[s], w23[s]);
          }
          w01[r] = k01;
          w23[r] = k23;
        }
#pragma unroll
        for (int half = 16; half >= 1; half >>= 1) {
          const bool hi = (lane & half) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float send = hi ? acc[i] : acc[i + half];
            const float keep = hi ? acc[i + half] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
          }
        }
        if (lane < 28) {
          const int rs = kDiagPair[lane], r = rs >> 3, sc = rs & 7;
          sA[(kw * 8 + r) * kLdA + kw * 8 + sc] = acc[0];
        }
      } else {
        // 64 slots: 0..27 A_rs (r > s), 28..31 P_rr (r < 4), then their partners of the first
        // butterfly level, 32..59 P_rs (r > s, in A's order) and 60..63 P_rr (r >= 4).  That first
        // level (slot i with slot i + 32, lanes 16 apart) runs row by row as soon as both partners
        // exist, so 32 partial sums are live instead of 64; the additions are the same.
        // Rows outer: w[s] = k_s o prod_{u=s+1..r} a_u is carried along the rows (the same
        // products in the same order as a column-by-column recursion), so only the current row's
        // k and q are widened at a time.
        const bool hi16 = (lane & 16) != 0;
        float red[32], pdiag[4];
        float2 w01[8], w23[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float2 k01 = klo(r), k23 = khi(r), q01 = qlo(r), q23 = qhi(r);
#pragma unroll
          for (int s = 0; s < r; ++s) {
            w01[s] = mul_f32x2(w01[s], make_float2(al[r][0], al[r][1]));
            w23[s] = mul_f32x2(w23[s], make_float2(al[r][2], al[r][3]));
            const float av = dot4(k01, k23, w01[s], w23[s]);
            const float pv = dot4(q01, q23, w01[s], w23[s]);
            red[r * (r - 1) / 2 + s] = (hi16 ? pv : av) + __shfl_xor_sync(0xffffffffu, hi16 ? av : pv, 16);
          }
          const float pd = dot4(q01, q23, k01, k23);
          if (r < 4) {
            pdiag[r] = pd;
          } else {
            red[28 + r - 4] = (hi16 ? pd : pdiag[r - 4]) + __shfl_xor_sync(0xffffffffu, hi16 ? pdiag[r - 4] : pd, 16);
          }
          w01[r] = k01;
          w23[r] = k23;
        }
        // the remaining levels over the 32 slots: lanes end with slots 2 lane and 2 lane + 1
#pragma unroll
        for (int half = 16; half >= 2; half >>= 1) {
          const int bit = half >> 1;  // 8, 4, 2, 1
          const bool hi = (lane & bit) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float send = hi ? red[i] : red[i + half];
            const float keep = hi ? red[i + half] : red[i];
            red[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = 2 * lane + u;
          const int rs = kDiagPair[idx], r = rs >> 3, sc = rs & 7;
          if (idx < 28) {
            sA[(kw * 8 + r) * kLdA + kw * 8 + sc] = red[u];
          } else {
            *reinterpret_cast<__nv_bfloat16*>(sP + sw_off(kw * 8 + r, kw * 8 + sc, 64)) = __float2bfloat16_rn(red[u]);
          }
        }
      }
      // in-block products: p8 inclusive prefix from the block start, s8 exclusive suffix (formed
      // once for the score tiles and once more, after the scores, for the state tiles: the
      // decays stay in registers, the products would hold twice as many through the scores)
      auto block_products = [&](float (&p8)[8][4], float (&s8)[8][4]) {
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          float2 acc = make_float2(1.f, 1.f);
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            acc = mul_f32x2(acc, make_float2(al[r][c], al[r][c + 1]));
            p8[r][c] = acc.x;
            p8[r][c + 1] = acc.y;
          }
          acc = make_float2(1.f, 1.f);
#pragma unroll
          for (int r = 7; r >= 0; --r) {
            s8[r][c] = acc.x;
            s8[r][c + 1] = acc.y;
            acc = mul_f32x2(acc, make_float2(al[r][c], al[r][c + 1]));
          }
        }
      };
      {
        float p8[8][4], s8[8][4];
        block_products(p8, s8);
        *reinterpret_cast<float4*>(sTau + kw * D + ch) = make_float4(p8[7][0], p8[7][1], p8[7][2], p8[7][3]);

        // the state team's inverse of the previous chunk must be done before this chunk rewrites
        // sA and the score tiles (the inverse's scratch); one thread waits, the team barrier
        // passes the outcome on
        bool bad = false;
        if (ci > 0 && tid == 0) {
          bad = !mbar_wait_bounded(bar_inv, par ^ 1u, kWaitLimitNs);
          if (bad) {
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          }
        }
        if (group_sync_any(kKeyBar, kTeam, bad || *s_abort != 0)) {  // (1) block products visible
          aborted = true;
          break;
        }

        // the 16-block-level factors: the decay of the other 8-block of my 16-block
        float prevb[4], nextb[4];
        {
          const float4 t4 = *reinterpret_cast<const float4*>(sTau + (kw ^ 1) * D + ch);
          prevb[0] = nextb[0] = t4.x;
          prevb[1] = nextb[1] = t4.y;
          prevb[2] = nextb[2] = t4.z;
          prevb[3] = nextb[3] = t4.w;
        }
        // decay between the two 16-blocks of each pair (both blocks excluded); pairs in the order
        // (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
        if (kw == 0) {
          float t16a[4], t16b[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float* tv = sTau + ch + c;
            t16a[c] = tv[2 * D] * tv[3 * D];  // 16-block 1
            t16b[c] = tv[4 * D] * tv[5 * D];  // 16-block 2
          }
          // bf16 pairs of channels (the scale of a bf16 operand pair in the score products)
          const uint2 one = pack4(1.f, 1.f, 1.f, 1.f);
          uint2* mp2 = reinterpret_cast<uint2*>(sMp + ch / 2);
          mp2[0 * 32] = one;
          mp2[1 * 32] = pack4(t16a[0], t16a[1], t16a[2], t16a[3]);
          mp2[2 * 32] = one;
          mp2[3 * 32] = pack4(t16a[0] * t16b[0], t16a[1] * t16b[1], t16a[2] * t16b[2], t16a[3] * t16b[3]);
          mp2[4 * 32] = pack4(t16b[0], t16b[1], t16b[2], t16b[3]);
          mp2[5 * 32] = one;
        }
        // score tiles.  The block-local products are formed once per row -- kp = k o p8 (prefix
        // from the block start), qp = q o p8, ks = k o s8 (suffix to the block end) -- and every
        // tile is one of them, possibly scaled once more: K o pi = kp (o prevb in an upper half),
        // K o kappa = ks (o nextb in a lower half), the 8-level halves kp / qp (upper) and ks
        // (lower).  (channel pairs multiplied two at a time)
        const float2 pb01 = make_float2(prevb[0], prevb[1]), pb23 = make_float2(prevb[2], prevb[3]);
        const float2 nb01 = make_float2(nextb[0], nextb[1]), nb23 = make_float2(nextb[2], nextb[3]);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = kw * 8 + r;
          const float2 p01 = make_float2(p8[r][0], p8[r][1]), p23 = make_float2(p8[r][2], p8[r][3]);
          const float2 s01 = make_float2(s8[r][0], s8[r][1]), s23 = make_float2(s8[r][2], s8[r][3]);
          const float2 k01 = klo(r), k23 = khi(r);
          const float2 kp01 = mul_f32x2(k01, p01), kp23 = mul_f32x2(k23, p23);
          const float2 ks01 = mul_f32x2(k01, s01), ks23 = mul_f32x2(k23, s23);
          float2 qp01 = make_float2(0.f, 0.f), qp23 = qp01;
          if constexpr (kRead) {
            qp01 = mul_f32x2(qlo(r), p01);
            qp23 = mul_f32x2(qhi(r), p23);
          }
          const int r32 = b16 * 8 + r;
          if (upper) {
            *reinterpret_cast<uint2*>(sm + OFF_KPI + sw_off(row, ch, 64)) =
                pack4(mul_f32x2(kp01, pb01), mul_f32x2(kp23, pb23));
            *reinterpret_cast<uint2*>(sm + OFF_KPI8 + sw_off(r32, ch, 32)) = pack4(kp01, kp23);
            if constexpr (kRead) {
              *reinterpret_cast<uint2*>(sm + OFF_QPI + sw_off(row, ch, 64)) =
                  pack4(mul_f32x2(qp01, pb01), mul_f32x2(qp23, pb23));
              *reinterpret_cast<uint2*>(sm + OFF_QPI8 + sw_off(r32, ch, 32)) = pack4(qp01, qp23);
            }
            *reinterpret_cast<uint2*>(sm + OFF_KC + sw_off(row, ch, 64)) = pack4(ks01, ks23);
          } else {
            *reinterpret_cast<uint2*>(sm + OFF_KPI + sw_off(row, ch, 64)) = pack4(kp01, kp23);
            if constexpr (kRead)
              *reinterpret_cast<uint2*>(sm + OFF_QPI + sw_off(row, ch, 64)) = pack4(qp01, qp23);
            *reinterpret_cast<uint2*>(sm + OFF_KC + sw_off(row, ch, 64)) =
                pack4(mul_f32x2(ks01, nb01), mul_f32x2(ks23, nb23));
            *reinterpret_cast<uint2*>(sm + OFF_KK8 + sw_off(r32, ch, 32)) = pack4(ks01, ks23);
          }
        }
      }
      group_sync(kKeyBar, kTeam);  // (2) score tiles, pair decays and diagonal scores in place


      // ---- part 2: off-diagonal scores on mma.sync
      {
        const int g = lane >> 2, t = lane & 3, m = lane >> 3;
        if (kw < 6) {
          // pairs (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
          const int pa = kw < 1 ? 1 : (kw < 3 ? 2 : 3), pb = kw - pa * (pa - 1) / 2;
          float accA[2][4] = {}, accP[2][4] = {};
          const uint32_t* mp = sMp + kw * (D / 2);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t ak0, ak1, ak2, ak3, aq0, aq1, aq2, aq3, b00, b01, b10, b11;
            const int ar = 16 * pa + (m & 1) * 8 + (lane & 7), akc = 2 * kk + (m >> 1);
            ldsm_x4(sbase + OFF_KPI + sw_off(ar, akc * 8, 64), ak0, ak1, ak2, ak3);
            if constexpr (kRead) ldsm_x4(sbase + OFF_QPI + sw_off(ar, akc * 8, 64), aq0, aq1, aq2, aq3);
            const int br = 16 * pb + (m >> 1) * 8 + (lane & 7), bkc = 2 * kk + (m & 1);
            ldsm_x4(sbase + OFF_KC + sw_off(br, bkc * 8, 64), b00, b01, b10, b11);
            if (pa - pb > 1) {  // adjacent 16-blocks have nothing between them
              // channels 16 kk + 2 t, + 1 and 16 kk + 2 t + 8, + 9
              const uint32_t m01 = mp[8 * kk + t], m89 = mp[8 * kk + t + 4];
              b00 = mul_bf16x2(b00, m01);
              b10 = mul_bf16x2(b10, m01);
              b01 = mul_bf16x2(b01, m89);
              b11 = mul_bf16x2(b11, m89);
            }
            mma16816(accA[0], ak0, ak1, ak2, ak3, b00, b01);
            mma16816(accA[1], ak0, ak1, ak2, ak3, b10, b11);
            if constexpr (kRead) {
              mma16816(accP[0], aq0, aq1, aq2, aq3, b00, b01);
              mma16816(accP[1], aq0, aq1, aq2, aq3, b10, b11);
            }
          }
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              const int r = 16 * pa + g + 8 * hlf, s = 16 * pb + 8 * nt + 2 * t;
              sA[r * kLdA + s] = accA[nt][2 * hlf];
              sA[r * kLdA + s + 1] = accA[nt][2 * hlf + 1];
              if constexpr (kRead)
                *reinterpret_cast<uint32_t*>(sP + sw_off(r, s, 64)) = pack_bf16(accP[nt][2 * hlf], accP[nt][2 * hlf + 1]);
            }
          }
          if (kw == 0 || kw == 2) {
            // the inverses of the diagonal 8x8 blocks, X = (I + diag(beta) A_blk)^{-1} (unit lower
            // triangular), on the two warps whose score pairs are adjacent (the lightest): four
            // blocks per warp, lane -> (block, column j) runs the forward substitution of column j;
            // the strictly lower part goes to the block's upper triangle of sA (never read as A),
            // transposed
            const int j = lane & 7, base = 8 * ((kw >> 1) * 4 + (lane >> 3));
            float lb[8][8], bb[8];  // the block's strictly lower scores and its betas, loaded up front
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              bb[r] = sBetaC[base + r];
#pragma unroll
              for (int c = 0; c < r; ++c) lb[r][c] = sA[(base + r) * kLdA + base + c];
            }
            float x[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              float acc = 0.f;
#pragma unroll
              for (int c = 0; c < r; ++c) acc = fmaf(lb[r][c], x[c], acc);
              x[r] = r < j ? 0.f : (r == j ? 1.f : -bb[r] * acc);
            }
#pragma unroll
            for (int r = 1; r < 8; ++r)
              if (r > j) sA[(base + j) * kLdA + base + r] = x[r];
          }
        } else {
          // rows 8..15 x columns 0..7 inside each 16-block, reference point between the halves
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            const int bb = 2 * (kw - 6) + q;
            float accA[4] = {}, accP[4] = {};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              uint32_t ak0, ak1, ak2, ak3, aq0, aq1, aq2, aq3, b0, b1;
              const int ar = 8 * bb + (lane & 7), akc = 2 * kk + (m >> 1);
              ldsm_x4(sbase + OFF_KPI8 + sw_off(ar, akc * 8, 32), ak0, ak1, ak2, ak3);
              if constexpr (kRead) ldsm_x4(sbase + OFF_QPI8 + sw_off(ar, akc * 8, 32), aq0, aq1, aq2, aq3);
              const int br = 8 * bb + (lane & 7), bkc = 2 * kk + ((lane >> 3) & 1);
              ldsm_x2(sbase + OFF_KK8 + sw_off(br, bkc * 8, 32), b0, b1);
              mma16816(accA, ak0, ak1, ak2, ak3, b0, b1);
              if constexpr (kRead) mma16816(accP, aq0, aq1, aq2, aq3, b0, b1);
            }
            const int r = 16 * bb + 8 + g, s = 16 * bb + 2 * t;
            sA[r * kLdA + s] = accA[2];
            sA[r * kLdA + s + 1] = accA[3];
            if constexpr (kRead)
              *reinterpret_cast<uint32_t*>(sP + sw_off(r, s, 64)) = pack_bf16(accP[2], accP[3]);
          }
        }
      }
      fence_async_smem();          // P is read by the tensor cores
      group_sync(kKeyBar, kTeam);  // (3) A, P and the 8x8 block inverses complete
      // the score tiles have been read: the next chunk's raw gates and keys may come in (every
      // thread's reads were ordered before the copies by its proxy fence and the barrier)
      if (tid == 0) {
        // (the test hook withholds the first chunk's signal: the state team's bounded wait then
        // gives up and both teams leave through the abort flag)
        if (!((a.flags & KDA_DEBUG_WITHHOLD_HANDOFF) && ci == 0)) mbar_arrive(bar_scores);
        if (c0 + C < t1) issue_stage(c0 + C);
      }
      stg_pending = c0 + C < t1;

      // ---- prefill: the state side's tiles.  K o Gamma and Q o Gamma were read only by the previous
      // chunk's first product, which completed before its inverse signalled (observed at (1)), so
      // they are written at once.  K' waits for the previous chunk's state update, and the wait
      // also covers its output product: it read the score tile P of that chunk's parity, which
      // the next chunk's in-block products rewrite before their first barrier.
      if constexpr (!kBuild) {
        float p8[8][4], s8[8][4];
        block_products(p8, s8);
        float pre[4], suf[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pre[c] = 1.f;
          suf[c] = 1.f;
        }
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const float4 t4 = *reinterpret_cast<const float4*>(sTau + w * D + ch);
          const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (w < kw) pre[c] *= tv[c];
            if (w > kw) suf[c] *= tv[c];
          }
        }
        if (kw == 0) {
          *reinterpret_cast<float4*>(sGC + par * 128 + ch) =
              make_float4(p8[7][0] * suf[0], p8[7][1] * suf[1], p8[7][2] * suf[2], p8[7][3] * suf[3]);
        }
        const float2 pre01 = make_float2(pre[0], pre[1]), pre23 = make_float2(pre[2], pre[3]);
        const float2 suf01 = make_float2(suf[0], suf[1]), suf23 = make_float2(suf[2], suf[3]);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = kw * 8 + r;
          const float2 p01 = make_float2(p8[r][0], p8[r][1]), p23 = make_float2(p8[r][2], p8[r][3]);
          const float2 kp01 = mul_f32x2(klo(r), p01), kp23 = mul_f32x2(khi(r), p23);
          const float2 qp01 = mul_f32x2(qlo(r), p01), qp23 = mul_f32x2(qhi(r), p23);
          *reinterpret_cast<uint2*>(sm + OFF_KQ + sw_off(row, ch, 128)) =
              pack4(mul_f32x2(kp01, pre01), mul_f32x2(kp23, pre23));
          *reinterpret_cast<uint2*>(sm + OFF_KQ + sw_off(64 + row, ch, 128)) =
              pack4(mul_f32x2(qp01, pre01), mul_f32x2(qp23, pre23));
        }
        bool bad = false;
        if (ci > 0 && tid == 0) {
          bad = !mbar_wait_bounded(bar4, par ^ 1u, kWaitLimitNs) || !mbar_wait_bounded(bar2, par ^ 1u, kWaitLimitNs);
          if (bad) {
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          }
        }
        if (group_sync_any(kKeyBar, kTeam, bad || *s_abort != 0)) {  // (4)
          aborted = true;
          break;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = kw * 8 + r;
          const float2 s01 = make_float2(s8[r][0], s8[r][1]), s23 = make_float2(s8[r][2], s8[r][3]);
          const float2 ks01 = mul_f32x2(klo(r), s01), ks23 = mul_f32x2(khi(r), s23);
          *reinterpret_cast<uint2*>(sm + OFF_KPT + sw_off(row, ch, 64)) =
              pack4(mul_f32x2(ks01, suf01), mul_f32x2(ks23, suf23));
        }
        fence_async_smem();  // the state tiles are read by the tensor cores
        group_sync(kKeyBar, kTeam);  // (5) state tiles in place (and every read of sTau done)
        if (tid == 0) mbar_arrive(bar_tiles);
      } else
      // ---- the state side's tiles, once the previous chunk's products that read them completed:
      // its state updates (K') and its readout / output products (the K o Gamma and Q o Gamma
      // tile).  This is the only place the key team waits on those products, so its gates,
      // in-block products and scores of this chunk ran under them.
      {
        bool bad = false;
        if (ci > 0 && tid == 0) {
          bad = !mbar_wait_bounded(bar4, par ^ 1u, kWaitLimitNs) ||
                (kRead && !mbar_wait_bounded(bar2, par ^ 1u, kWaitLimitNs));
          if (bad) {
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          }
        }
        if (group_sync_any(kKeyBar, kTeam, bad || *s_abort != 0)) {  // (4)
          aborted = true;
          break;
        }
        float p8[8][4], s8[8][4];
        block_products(p8, s8);
        // chunk-level factors: the decay from the chunk start to my block (pre) and from my block
        // to the chunk end (suf)
        float pre[4], suf[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pre[c] = 1.f;
          suf[c] = 1.f;
        }
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const float4 t4 = *reinterpret_cast<const float4*>(sTau + w * D + ch);
          const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (w < kw) pre[c] *= tv[c];
            if (w > kw) suf[c] *= tv[c];
          }
        }
        if (kw == 0) {
          *reinterpret_cast<float4*>(sGC + par * 128 + ch) =
              make_float4(p8[7][0] * suf[0], p8[7][1] * suf[1], p8[7][2] * suf[2], p8[7][3] * suf[3]);
        }
        // K o Gamma = kp o pre, Q o Gamma = qp o pre, K' = ks o suf
        const float2 pre01 = make_float2(pre[0], pre[1]), pre23 = make_float2(pre[2], pre[3]);
        const float2 suf01 = make_float2(suf[0], suf[1]), suf23 = make_float2(suf[2], suf[3]);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = kw * 8 + r;
          const float2 p01 = make_float2(p8[r][0], p8[r][1]), p23 = make_float2(p8[r][2], p8[r][3]);
          const float2 s01 = make_float2(s8[r][0], s8[r][1]), s23 = make_float2(s8[r][2], s8[r][3]);
          const float2 k01 = klo(r), k23 = khi(r);
          const float2 kp01 = mul_f32x2(k01, p01), kp23 = mul_f32x2(k23, p23);
          const float2 ks01 = mul_f32x2(k01, s01), ks23 = mul_f32x2(k23, s23);
          *reinterpret_cast<uint2*>(sm + OFF_KQ + sw_off(row, ch, 128)) =
              pack4(mul_f32x2(kp01, pre01), mul_f32x2(kp23, pre23));
          if constexpr (kRead) {
            const float2 qp01 = mul_f32x2(qlo(r), p01), qp23 = mul_f32x2(qhi(r), p23);
            *reinterpret_cast<uint2*>(sm + OFF_KQ + sw_off(64 + row, ch, 128)) =
                pack4(mul_f32x2(qp01, pre01), mul_f32x2(qp23, pre23));
          }
          // K' = K o (decay to the chunk end), token rows like the other tiles: the update reads
          // it as the MN-major B operand K'^T
          *reinterpret_cast<uint2*>(sm + OFF_KPT + sw_off(row, ch, 64)) =
              pack4(mul_f32x2(ks01, suf01), mul_f32x2(ks23, suf23));
        }
        fence_async_smem();  // the state tiles are read by the tensor cores
        group_sync(kKeyBar, kTeam);  // (5) state tiles in place (and every read of sTau done)
        if (tid == 0) mbar_arrive(bar_tiles);
      }
    }
    if (stg_pending) mbar_wait_bounded(bar_stg, stg_parity, kWaitLimitNs);  // a copy still in flight
    regs_decrease<kLaunchRegs>();  // back to the launch's share before the teams join
  } else {
    regs_decrease<RegSplit<kBuild>::state>();
    // ================================================================ state team
    // mapping: team warp sw, team thread st; epilogue row ej (its TMEM lane) and column half ehalf
    const int sw = warp - 8, st = tid - kTeam;
    const int ej = (sw & 3) * 32 + lane, ehalf = sw >> 2;
    auto issue_prefetch_v = [&](int c0n) {
      if (has_v) {
        mbar_arrive_expect_tx(bar_v, 16384u);
        tma_load_3d(sbase + OFF_V, &tm.v, 0, h, (int)c0n, bar_v);
        tma_load_3d(sbase + OFF_V + 8192, &tm.v, 64, h, (int)c0n, bar_v);
      }
    };
    bool v_pending = false;   // V copy issued whose completion was not yet observed
    uint32_t v_parity = 0;    // parity of the next completion on bar_v
    if (t1 > t0) {
      if (st == kCopyThread) issue_prefetch_v(t0);
      v_pending = has_v;
    }
    uint32_t ci = 0;
#pragma unroll 1
    for (int c0 = t0; c0 < t1; c0 += C, ++ci) {
      const int L = rows_of(c0);
      const uint32_t par = ci & 1u;
      const uint32_t pofs = OFF_P + par * 8192;
      const float* sBetaC = sBeta + par * 64;
      const float* sGCc = sGC + par * 128;

      // the first product(s), once the key team's tiles are in place (the bf16 state copies, this
      // team's, landed at the end of the previous chunk); one thread
      auto issue_first = [&]() {
        if (!mbar_wait_bounded(bar_tiles, par, kWaitLimitNs)) {
          *s_abort = 1;
          report(a.status, KDA_ERR_DEVICE_TIMEOUT);
        } else {
          tc_fence_after();
          if constexpr (!kBuild) {
            // D1 = S^T [K o Gamma ; Q o Gamma]^T   (M = 128, N = 128, K = 128)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_bf16_ts(tmD1, tmSb + 8 * kk, desc_sw128(sbase + OFF_KQ + koff), idesc_bf16_f32(128), kk > 0);
            }
          } else {
            // D1_M = -S_M^T (K o Gamma)^T and D1_U = -S_U^T (K o Gamma)^T   (N = 64 each, K = 128; the
            // instruction negates K o Gamma, so the epilogue stores Y^T as it comes)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
              constexpr uint32_t idn = idesc_bf16_f32(64, false, false, true);
              mma_bf16_ts(tmD1, tmSb + 8 * kk, desc_sw128(sbase + OFF_KQ + koff), idn, kk > 0);
              mma_bf16_ts(tmD1u, tmSbu + 8 * kk, desc_sw128(sbase + OFF_KQ + koff), idn, kk > 0);
            }
          }
          mma_commit(bar0);
        }
      };
      // The build issues them here; the prefill inside the inverse's first level, where its
      // epilogue runs (measured: the prefill 1.705 -> 1.67 ms on the 64 x 2048-token batch; the
      // build slower, 4.62 -> 4.89 ms on the benchmark step, as its later products then meet the
      // key team's tile stores)
      if (kBuild && st == kIssueFirst) issue_first();
      // the previous chunk's staged outputs have been read by their tensor store (the staging
      // tiles are rewritten below)
      if (st == kCopyThread) bulk_wait_read_all();
      // ---- the key team's scores of this chunk are in place
      bool bad = false;
      if (st == 0) {
        bad = !mbar_wait_bounded(bar_scores, par, kWaitLimitNs);
        if (bad) {
          *s_abort = 1;
          report(a.status, KDA_ERR_DEVICE_TIMEOUT);
        }
      }
      if (group_sync_any(kStateBar, kTeam, bad || *s_abort != 0)) {
        aborted = true;
        break;
      }

      // ---- T = (I + diag(beta) A)^{-1} diag(beta)
      // X = (I + L)^{-1}, L = diag(beta) A strictly lower.  Diagonal 8-blocks by forward
      // substitution (the key team, during its scores), 16-blocks from them in fp32; then two
      // doubling levels on tf32 mma.sync -- X10 and X32 from the 16-blocks, then the lower-left
      // 32-block from the 32-blocks -- each as X_ab = -X_aa (L_ab X_bb).  T is rounded to bf16
      // afterwards, so tf32 products suffice.
      {
        float* Xi = reinterpret_cast<float*>(sm + OFF_XI);
        float* Yb = reinterpret_cast<float*>(sm + OFF_Y);  // per-warp 16x8 tiles, then [32][32]
        {
          // the 16-blocks from their 8-blocks a = 2m, b = 2m + 1 (inverted by the key team, stored
          // transposed above the diagonal of sA): X_ba = -X_bb (L_ba X_aa); thread -> (16-block m,
          // row i, column j) of the 8 x 8 products
          const int m = st >> 6, i = (st >> 3) & 7, j = st & 7;
          const int ra = 16 * m, rb8 = 16 * m + 8;
          auto xblk = [&](int base, int r, int c) {  // unit lower triangular 8-block inverse
            return r == c ? 1.f : (c < r ? sA[(base + c) * kLdA + base + r] : 0.f);
          };
          float y = 0.f;
#pragma unroll
          for (int l = 0; l < 8; ++l) y = fmaf(sA[(rb8 + i) * kLdA + ra + l], xblk(ra, l, j), y);
          Yb[st] = sBetaC[rb8 + i] * y;  // (L_ba X_aa)[i][j]
          group_sync(kStateBar, kTeam);
          float xv = 0.f;
#pragma unroll
          for (int l = 0; l < 8; ++l) xv = fmaf(xblk(rb8, i, l), Yb[m * 64 + l * 8 + j], xv);
          const float xa = xblk(ra, i, j), xb = xblk(rb8, i, j);
          Xi[(rb8 + i) * kLdA + ra + j] = -xv;
          Xi[(ra + i) * kLdA + ra + j] = xa;
          Xi[(rb8 + i) * kLdA + rb8 + j] = xb;
          Xi[(ra + i) * kLdA + rb8 + j] = 0.f;
          // this 16-block of T = X diag(beta) (its upper triangle stays zero from the launch)
          put_t1(sm + OFF_T, rb8 + i, ra + j, -xv * sBetaC[ra + j]);
          if (j <= i) {
            put_t1(sm + OFF_T, ra + i, ra + j, xa * sBetaC[ra + j]);
            put_t1(sm + OFF_T, rb8 + i, rb8 + j, xb * sBetaC[rb8 + j]);
          }
        }
        group_sync(kStateBar, kTeam);
        const int g = lane >> 2, t = lane & 3;
        auto lval = [&](int r, int c) { return sBetaC[r] * sA[r * kLdA + c]; };
        if (sw >= 4) {
          // team warps 4..7 have no part in the first doubling level: they run the first
          // product's epilogue; warp -> TMEM lane quadrant sw % 4, all 64 columns.  Y^T[j][r] =
          // -((K o Gamma) S0)^T into the X tile(s) (in the build the products computed it negated;
          // the prefill's one N = 128 product negates here); V enters in the next product
          if (!kBuild && st == kIssueFirst) issue_first();
          __syncwarp();
          if (!mbar_wait_bounded(bar0, par, kWaitLimitNs)) {
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          } else {
            tc_fence_after();
#pragma unroll 1
            for (int stt = 0; stt < (kBuild ? 2 : 1); ++stt) {
#pragma unroll 1
              for (int r0 = 0; r0 < 64; r0 += 32) {
                float d[32];
                tmem_ld16n<2>((stt ? tmD1u : tmD1) + lane_base + r0, d);
                tmem_wait_ld();
                const uint32_t xoff = (kBuild && stt == 0) ? OFF_XM : OFF_X;
#pragma unroll
                for (int u = 0; u < 32; u += 8)
                  *reinterpret_cast<uint4*>(sm + xoff + sw_off(ej, r0 + u, 128)) =
                      kBuild ? make_uint4(pack_bf16(d[u], d[u + 1]), pack_bf16(d[u + 2], d[u + 3]),
                                          pack_bf16(d[u + 4], d[u + 5]), pack_bf16(d[u + 6], d[u + 7]))
                             : make_uint4(pack_bf16(-d[u], -d[u + 1]), pack_bf16(-d[u + 2], -d[u + 3]),
                                          pack_bf16(-d[u + 4], -d[u + 5]), pack_bf16(-d[u + 6], -d[u + 7]));
              }
            }
          }
          fence_async_smem();
          tc_fence_before();
        } else {
          // level 1: warp -> (problem, 8-column tile); problem 0 = X10, problem 1 = X32
          const int ra = (sw >> 1) ? 3 : 1, cb = 16 * (ra - 1), R0 = 16 * ra, n0 = 8 * (sw & 1);
          float* yt = Yb + sw * 128;  // 16 x 8 tile of Y, row-major
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int k0 = 8 * ks;
            mma1688_tf32(acc, to_tf32(lval(R0 + g, cb + k0 + t)), to_tf32(lval(R0 + g + 8, cb + k0 + t)),
                         to_tf32(lval(R0 + g, cb + k0 + t + 4)), to_tf32(lval(R0 + g + 8, cb + k0 + t + 4)),
                         to_tf32(Xi[(cb + k0 + t) * kLdA + cb + n0 + g]),
                         to_tf32(Xi[(cb + k0 + t + 4) * kLdA + cb + n0 + g]));
          }
          yt[g * 8 + 2 * t] = acc[0];
          yt[g * 8 + 2 * t + 1] = acc[1];
          yt[(g + 8) * 8 + 2 * t] = acc[2];
          yt[(g + 8) * 8 + 2 * t + 1] = acc[3];
          __syncwarp();
          float xo[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int k0 = 8 * ks;
            mma1688_tf32(xo, to_tf32(Xi[(R0 + g) * kLdA + R0 + k0 + t]), to_tf32(Xi[(R0 + g + 8) * kLdA + R0 + k0 + t]),
                         to_tf32(Xi[(R0 + g) * kLdA + R0 + k0 + t + 4]),
                         to_tf32(Xi[(R0 + g + 8) * kLdA + R0 + k0 + t + 4]), to_tf32(yt[(k0 + t) * 8 + g]),
                         to_tf32(yt[(k0 + t + 4) * 8 + g]));
          }
          Xi[(R0 + g) * kLdA + cb + n0 + 2 * t] = -xo[0];
          Xi[(R0 + g) * kLdA + cb + n0 + 2 * t + 1] = -xo[1];
          Xi[(R0 + g + 8) * kLdA + cb + n0 + 2 * t] = -xo[2];
          Xi[(R0 + g + 8) * kLdA + cb + n0 + 2 * t + 1] = -xo[3];
          const int s0 = cb + n0 + 2 * t;
          const float b0 = sBetaC[s0], b1 = sBetaC[s0 + 1];
          put_t2(sm + OFF_T, R0 + g, s0, -xo[0] * b0, -xo[1] * b1);
          put_t2(sm + OFF_T, R0 + g + 8, s0, -xo[2] * b0, -xo[3] * b1);
        }
        group_sync(kStateBar, kTeam);
        {
          // level 2: Y = L[32:64, 0:32] X[0:32, 0:32]; X[32:64, 0:32] = -X[32:64, 32:64] Y
          // warp -> (16-row tile mt, 8-column tile nt); X[0:16, 16:32] and X[32:48, 48:64] are zero
          float* Y2 = Yb + 512;
          const int mt = sw >> 2, nt = sw & 3, R0 = 32 + 16 * mt, n0 = 8 * nt;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const int k0 = 8 * ks;
            if (nt >= 2 && ks < 2) continue;
            mma1688_tf32(acc, to_tf32(lval(R0 + g, k0 + t)), to_tf32(lval(R0 + g + 8, k0 + t)),
                         to_tf32(lval(R0 + g, k0 + t + 4)), to_tf32(lval(R0 + g + 8, k0 + t + 4)),
                         to_tf32(Xi[(k0 + t) * kLdA + n0 + g]), to_tf32(Xi[(k0 + t + 4) * kLdA + n0 + g]));
          }
          const int yr = 16 * mt;
          Y2[(yr + g) * 32 + n0 + 2 * t] = acc[0];
          Y2[(yr + g) * 32 + n0 + 2 * t + 1] = acc[1];
          Y2[(yr + g + 8) * 32 + n0 + 2 * t] = acc[2];
          Y2[(yr + g + 8) * 32 + n0 + 2 * t + 1] = acc[3];
          group_sync(kStateBar, kTeam);
          float xo[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const int k0 = 8 * ks;
            if (mt == 0 && ks >= 2) continue;
            mma1688_tf32(xo, to_tf32(Xi[(R0 + g) * kLdA + 32 + k0 + t]), to_tf32(Xi[(R0 + g + 8) * kLdA + 32 + k0 + t]),
                         to_tf32(Xi[(R0 + g) * kLdA + 32 + k0 + t + 4]),
                         to_tf32(Xi[(R0 + g + 8) * kLdA + 32 + k0 + t + 4]), to_tf32(Y2[(k0 + t) * 32 + n0 + g]),
                         to_tf32(Y2[(k0 + t + 4) * 32 + n0 + g]));
          }
          // the last block of X: only T is needed from here on
          const int s0 = n0 + 2 * t;
          const float b0 = sBetaC[s0], b1 = sBetaC[s0 + 1];
          put_t2(sm + OFF_T, R0 + g, s0, -xo[0] * b0, -xo[1] * b1);
          put_t2(sm + OFF_T, R0 + g + 8, s0, -xo[2] * b0, -xo[3] * b1);
        }
      }
      fence_async_smem();  // T (and the first epilogue's X tiles) are read by the tensor cores
      if (group_sync_any(kStateBar, kTeam, *s_abort != 0)) {  // (4) every operand of this chunk is in place
        aborted = true;
        break;
      }
      if (st == 0) mbar_arrive(bar_inv);  // sA and the score tiles are the key team's again

      if constexpr (!kBuild) {
        // ============================ prefill state side (the first product's epilogue ran
        // during the inverse)
        // D1[:, 0:64] = V^T T^T + Y^T T^T = (V - (K o Gamma) S0)^T T^T = Delta^T   (N = 64, K = 64)
        if (st == kIssueDelta) {
          tc_fence_after();
          if (has_v && !mbar_wait_bounded(bar_v, v_parity, kWaitLimitNs)) {  // this chunk's V has landed
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          }
          if (!a.values_zero) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmD1, desc_sw128_mn(sbase + OFF_V + kk * 2048, 8192), desc_sw128(sbase + OFF_T + kk * 32),
                       idesc_bf16_f32(64, true), kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmD1, desc_sw128(sbase + OFF_X + kk * 32), desc_sw128(sbase + OFF_T + kk * 32), idesc_bf16_f32(64),
                     (kk > 0) || !a.values_zero);
          mma_commit(bar1);
        }
        {
          // decay the state columns while the second product runs (it reads neither state copy):
          // S^T[j][i] *= Gamma_63[i]
#pragma unroll 1
          for (int i0 = 64 * ehalf; i0 < 64 * ehalf + 64; i0 += 32) {
            float sv[32];
            tmem_ld32(tmS + lane_base + i0, sv);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
              const float4 gv = *reinterpret_cast<const float4*>(sGCc + i0 + u);
              sv[u] *= gv.x;
              sv[u + 1] *= gv.y;
              sv[u + 2] *= gv.z;
              sv[u + 3] *= gv.w;
            }
            tmem_st32(tmS + lane_base + i0, sv);
          }
          if (!mbar_wait_bounded(bar1, par, kWaitLimitNs)) {
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          } else {
            tc_fence_after();
            // Delta^T stays in TMEM as bf16 (two tokens per column), the A operand of the two
            // products below: no shared-memory round trip for it (measured: see the products)
            float d[32];
            tmem_ld16n<2>(tmD1 + lane_base + 32 * ehalf, d);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) pk[u] = pack_bf16(d[2 * u], d[2 * u + 1]);
            tmem_st16u(tmDb + lane_base + 16 * ehalf, pk);
          }
          tmem_wait_st();
          fence_async_smem();
          tc_fence_before();
        }
        if (group_sync_any(kStateBar, kTeam, *s_abort != 0)) {
          aborted = true;
          break;
        }
        // the V tile is free now that the second product completed (and its copy was observed)
        if (has_v) {
          v_pending = false;
          v_parity ^= 1u;
        }
        if (c0 + C < t1) {
          if (st == kCopyThread) issue_prefetch_v(c0 + C);
          v_pending = has_v;
        }

        // D1[:, 64:128] += Delta^T P^T ;  S^T += Delta^T K'   (accumulate; two issuing threads; A is
        // Delta^T in TMEM, 8 columns per 16 tokens)
        if (st == kIssueRead) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmD1 + 64, tmDb + 8 * kk, desc_sw128(sbase + pofs + kk * 32), idesc_bf16_f32(64), 1);
          mma_commit(bar2);
        }
        if (st == kIssueUpdate) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmS, tmDb + 8 * kk, desc_sw128_mn(sbase + OFF_KPT + kk * 2048, 8192),
                        idesc_bf16_f32(128, false, true), 1);
          mma_commit(bar4);
        }
        {
          // the outputs are staged while the state update still runs: bf16 in the XM tile (no
          // product reads it in the prefill); fp32 from the X tile on (free once the second
          // product completed), after the update too
          const bool out_done = mbar_wait_bounded(bar2, par, kWaitLimitNs);
          const bool upd_done = out_done && (a.out_bf16 || !a.out || mbar_wait_bounded(bar4, par, kWaitLimitNs));
          if (out_done && upd_done) {
            tc_fence_after();
            if (a.out && a.out_bf16) {
              // two token-row [64][64 channels] halves with the 128-byte swizzle, written by
              // transposing matrix stores from a 16 x 256-bit TMEM load (as the build's readouts)
              const int q4 = warp & 3, jm = lane >> 3, rr = lane & 7;
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[16];
                tmem_ld16x256b_x4(tmD1 + 64 + ((uint32_t)(32 * q4 + 16 * hh) << 16) + 32 * ehalf, r);
                tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                  const int tok = 32 * ehalf + 16 * k2 + 8 * (jm >> 1) + rr;
                  const int chn = 32 * q4 + 16 * hh + 8 * (jm & 1);
                  const uint32_t addr =
                      sbase + OFF_XM + (chn >> 6) * 8192 + tok * 128 + ((((chn & 63) >> 3) ^ (tok & 7)) << 4);
                  const uint32_t* v = r + 8 * k2;
                  stsm_x4_trans(addr, pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                                pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                                pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                                pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
                }
              }
            } else if (a.out) {
              float d[32];
              tmem_ld16n<2>(tmD1 + lane_base + 64 + 32 * ehalf, d);
              tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 32; ++u) reinterpret_cast<float*>(sm + OFF_X)[(32 * ehalf + u) * D + ej] = d[u];
            }
          }
          if (!out_done || !upd_done || !mbar_wait_bounded(bar4, par, kWaitLimitNs)) {
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          } else {
            tc_fence_after();
            // bf16 copy of the new state for the next chunk, into the TMEM A operand
#pragma unroll 1
            for (int i0 = 64 * ehalf; i0 < 64 * ehalf + 64; i0 += 32) {
              float sv[32];
              tmem_ld32(tmS + lane_base + i0, sv);
              tmem_wait_ld();
              uint32_t pk[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) pk[u] = pack_bf16(sv[2 * u], sv[2 * u + 1]);
              tmem_st16u(tmSb + lane_base + i0 / 2, pk);
            }
          }
          tmem_wait_st();
          fence_async_smem();
          tc_fence_before();
        }
        if (group_sync_any(kStateBar, kTeam, *s_abort != 0)) {
          aborted = true;
          break;
        }
        // flush the staged output rows of this chunk: a full chunk of a bf16 output leaves through
        // two tensor stores, a 64-channel half each (the source is read before the next chunk's
        // staging); otherwise row by row, so that no row of the next sequence is touched
        if (!a.out) {
        } else if (a.out_bf16 && L == C) {
          if (st == kCopyThread) {
            tma_store_3d(&tm.out, sbase + OFF_XM, 0, h, (int)c0);
            tma_store_3d(&tm.out, sbase + OFF_XM + 8192, 64, h, (int)c0);
            bulk_commit();
          }
        } else if (a.out_bf16) {
          for (int e = st; e < C * 16; e += kTeam) {
            const int row = e >> 4, cc = e & 15;
            if (row < L)
              *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ((size_t)(c0 + row) * a.Hv + h) * D +
                                        cc * 8) =
                  *reinterpret_cast<const uint4*>(sm + OFF_XM + (cc >> 3) * 8192 + row * 128 + (((cc & 7) ^ (row & 7)) << 4));
          }
        } else {
          for (int e = st; e < C * 32; e += kTeam) {
            const int row = e >> 5, cc = e & 31;
            if (row < L)
              *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ((size_t)(c0 + row) * a.Hv + h) * D + cc * 4) =
                  *reinterpret_cast<const float4*>(sm + OFF_X + row * 512 + cc * 16);
          }
        }
      } else {
        // ============================ segment build state side: both states (the first products'
        // epilogues ran during the inverse)
        // Delta_M^T = Y_M^T T^T ;  Delta_U^T = V^T T^T + Y_U^T T^T
        if (st == kIssueDelta) {
          tc_fence_after();
          if (!mbar_wait_bounded(bar_v, v_parity, kWaitLimitNs)) {  // this chunk's V has landed
            *s_abort = 1;
            report(a.status, KDA_ERR_DEVICE_TIMEOUT);
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmD1, desc_sw128(sbase + OFF_XM + kk * 32), desc_sw128(sbase + OFF_T + kk * 32),
                     idesc_bf16_f32(64), kk > 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmD1u, desc_sw128_mn(sbase + OFF_V + kk * 2048, 8192), desc_sw128(sbase + OFF_T + kk * 32),
                     idesc_bf16_f32(64, true), kk > 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmD1u, desc_sw128(sbase + OFF_X + kk * 32), desc_sw128(sbase + OFF_T + kk * 32),
                     idesc_bf16_f32(64), 1);
          mma_commit(bar1);
        }
        // decay both states while the second products run (they read neither state):
        // S^T[j][i] *= Gamma_63[i]
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          const uint32_t col = (q & 1 ? tmSu : tmS) + 64 * ehalf + 32 * (q >> 1);
          float sv[32];
          tmem_ld32(col + lane_base, sv);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            const float4 gv = *reinterpret_cast<const float4*>(sGCc + 64 * ehalf + 32 * (q >> 1) + u);
            sv[u] *= gv.x;
            sv[u + 1] *= gv.y;
            sv[u + 2] *= gv.z;
            sv[u + 3] *= gv.w;
          }
          tmem_st32(col + lane_base, sv);
        }
        if (!mbar_wait_bounded(bar1, par, kWaitLimitNs)) {
          *s_abort = 1;
          report(a.status, KDA_ERR_DEVICE_TIMEOUT);
        } else {
          tc_fence_after();
#pragma unroll 1
          for (int stt = 0; stt < 2; ++stt) {
            float d[32];
            tmem_ld16n<2>((stt ? tmD1u : tmD1) + lane_base + 32 * ehalf, d);
            tmem_wait_ld();
            const uint32_t xoff = stt ? OFF_X : OFF_XM;
#pragma unroll
            for (int r0 = 0; r0 < 32; r0 += 8)
              *reinterpret_cast<uint4*>(sm + xoff + sw_off(ej, 32 * ehalf + r0, 128)) =
                  make_uint4(pack_bf16(d[r0], d[r0 + 1]), pack_bf16(d[r0 + 2], d[r0 + 3]),
                             pack_bf16(d[r0 + 4], d[r0 + 5]), pack_bf16(d[r0 + 6], d[r0 + 7]));
          }
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        if (group_sync_any(kStateBar, kTeam, *s_abort != 0)) {
          aborted = true;
          break;
        }
        // the V tile is free now that the second products completed (and its copy was observed)
        v_pending = false;
        v_parity ^= 1u;
        if (c0 + C < t1) {
          if (st == kCopyThread) issue_prefetch_v(c0 + C);
          v_pending = true;
        }

        // [readouts: D_st = S_st,0^T (Q o Gamma)^T + Delta_st^T P^T -- the bf16 copies still hold the
        //  chunk's incoming states]   S_M^T += Delta_M^T K' ;  S_U^T += Delta_U^T K'
        // one issuing thread per state for each group (team warps 4 / 6 the readouts of M / U,
        // 5 / 7 their updates); bar2 and bar4 count the two commits of their group
        if (kRead && (st == kIssueRead || st == kIssueFirst)) {
          tc_fence_after();
          if constexpr (kRead) {
            const int sti = st == kIssueFirst ? 1 : 0;
            const uint32_t dcol = sti ? tmD1u : tmD1, acol = sti ? tmSbu : tmSb;
            const uint32_t xoff = sti ? OFF_X : OFF_XM;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32 + 8192;  // rows 64..127: Q o Gamma
              mma_bf16_ts(dcol, acol + 8 * kk, desc_sw128(sbase + OFF_KQ + koff), idesc_bf16_f32(64), kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(dcol, desc_sw128(sbase + xoff + kk * 32), desc_sw128(sbase + pofs + kk * 32),
                       idesc_bf16_f32(64), 1);
            mma_commit(bar2);
          }
        }
        if (st == kIssueUpdate || st == kIssueDelta) {
          tc_fence_after();
          const bool u = st == kIssueDelta;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(u ? tmSu : tmS, desc_sw128(sbase + (u ? OFF_X : OFF_XM) + kk * 32),
                     desc_sw128_mn(sbase + OFF_KPT + kk * 2048, 8192), idesc_bf16_f32(128, false, true), 1);
          mma_commit(bar4);
        }
        // the readouts are staged in the X tiles once both product groups (which read them) have
        // completed: row-major bf16, the transition's in XM, the contribution's in X
        const bool read_done = !kRead || mbar_wait_bounded(bar2, par, kWaitLimitNs);
        const bool upd_done = read_done && mbar_wait_bounded(bar4, par, kWaitLimitNs);
        if (!read_done || !upd_done) {
          *s_abort = 1;
          report(a.status, KDA_ERR_DEVICE_TIMEOUT);
        } else {
          tc_fence_after();
          if constexpr (kRead) {
            // staged for the tensor stores as two token-row [64][64 channels] bf16 halves with the
            // 128-byte swizzle: a 16 x 256-bit TMEM load hands each thread two adjacent tokens of
            // two channels, and transposing matrix stores write them as 8 x 8 blocks of token rows
            // (8 channels, 16 bytes each)
            const int q4 = warp & 3, jm = lane >> 3, rr = lane & 7;
#pragma unroll 1
            for (int stt = 0; stt < 2; ++stt) {
              const uint32_t stage = sbase + (stt ? OFF_X : OFF_XM);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                uint32_t r[16];
                tmem_ld16x256b_x4((stt ? tmD1u : tmD1) + ((uint32_t)(32 * q4 + 16 * hh) << 16) + 32 * ehalf, r);
                tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                  // matrix jm: tokens 32 ehalf + 16 k2 + 8 (jm / 2) .., channels 32 q4 + 16 hh + 8 (jm % 2) ..;
                  // this lane addresses its token row rr
                  const int tok = 32 * ehalf + 16 * k2 + 8 * (jm >> 1) + rr;
                  const int chn = 32 * q4 + 16 * hh + 8 * (jm & 1);
                  const uint32_t addr =
                      stage + (chn >> 6) * 8192 + tok * 128 + ((((chn & 63) >> 3) ^ (tok & 7)) << 4);
                  const uint32_t* v = r + 8 * k2;
                  stsm_x4_trans(addr, pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                                pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                                pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                                pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
                }
              }
            }
          }
          // bf16 copies of both new states for the next chunk's first products
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            const int i0 = 64 * ehalf + 32 * (q >> 1);
            float sv[32];
            tmem_ld32((q & 1 ? tmSu : tmS) + lane_base + i0, sv);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) pk[u] = pack_bf16(sv[2 * u], sv[2 * u + 1]);
            tmem_st16u((q & 1 ? tmSbu : tmSb) + lane_base + i0 / 2, pk);
          }
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        if (group_sync_any(kStateBar, kTeam, *s_abort != 0)) {
          aborted = true;
          break;
        }
        if constexpr (kRead) {
          // full chunks leave through four tensor stores, a 64-channel half each (sources read before
          // the next chunk's first epilogue rewrites them)
          if (L == C) {
            if (st == kCopyThread) {
              const int y = a.readout_hm ? (int)c0 : h, z = a.readout_hm ? h : (int)c0;
              tma_store_3d(&tm.out, sbase + OFF_XM, 0, y, z);
              tma_store_3d(&tm.out, sbase + OFF_XM + 8192, 64, y, z);
              tma_store_3d(&tm.out2, sbase + OFF_X, 0, y, z);
              tma_store_3d(&tm.out2, sbase + OFF_X + 8192, 64, y, z);
              bulk_commit();
            }
          } else {
            for (int e = st; e < 2 * C * 16; e += kTeam) {
              const int sti = e >> 10, row = (e >> 4) & 63, cc = e & 15;
              if (row < L)
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(sti ? a.out2 : a.out) +
                                          (a.readout_hm ? (size_t)h * a.total_tokens + c0 + row
                                                        : (size_t)(c0 + row) * a.Hv + h) * D + cc * 8) =
                    *reinterpret_cast<const uint4*>(sm + (sti ? OFF_X : OFF_XM) + (cc >> 3) * 8192 + row * 128 +
                                                    (((cc & 7) ^ (row & 7)) << 4));
            }
          }
        }
      }
    }

    if (!aborted) {
      // final state(s): the pool slot (prefill), or M and U of this segment (build); row j, columns
      // split between the two warps of a quadrant
      tc_fence_after();
#pragma unroll 1
      for (int sti = 0; sti < (kBuild ? 2 : 1); ++sti) {
        float* dst = sti ? a.state_out2 + blk_off : out_blk;
        const bool vf = (kBuild && sti == 0) ? false : (a.v_first != 0);
        const uint32_t tcol = sti ? tmSu : tmS;
#pragma unroll 1
        for (int i0 = 64 * ehalf; i0 < 64 * ehalf + 64; i0 += 16) {
          float sv[16];
          tmem_ld16(tcol + lane_base + i0, sv);
          tmem_wait_ld();
          if (vf) {
            float4* p = reinterpret_cast<float4*>(dst + (size_t)ej * D + i0);
#pragma unroll
            for (int q = 0; q < 4; ++q) p[q] = make_float4(sv[4 * q], sv[4 * q + 1], sv[4 * q + 2], sv[4 * q + 3]);
          } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) dst[(size_t)(i0 + u) * D + ej] = sv[u];
          }
        }
      }
    }
    tmem_wait_st();  // the last bf16 state copies
    if (v_pending) mbar_wait_bounded(bar_v, v_parity, kWaitLimitNs);  // a copy still in flight
    if (st == kCopyThread) bulk_wait_all();                             // output tensor stores
    if (aborted && (st == kIssueFirst || st == kIssueDelta || st == kIssueRead || st == kIssueUpdate)) {
      // let any MMA still in flight finish before the tensor memory is released (bar3 counts the
      // four issuing threads' commits)
      mma_commit(bar3);
      mbar_wait_bounded(bar3, 0, kWaitLimitNs);
    }
    regs_increase<kLaunchRegs>();  // back to the launch's share before the teams join
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) tmem_dealloc(tmem, kTmemCols);
}

bool fused_available() { return true; }

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [tokens][heads][128] row-major; box = box_x channels x 1 head x 64 tokens
// head_major: [heads][tokens][128] instead, coordinates (channel, token, head), box = box_x
// channels x 64 tokens x 1 head
bool encode_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t esize, int64_t tokens,
                 int heads, uint32_t box_x = D, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE,
                 bool head_major = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)(head_major ? tokens : heads),
                              (cuuint64_t)(head_major ? heads : tokens)};
  const cuuint64_t strides[2] = {(cuuint64_t)D * esize,
                                 (cuuint64_t)(head_major ? tokens : heads) * D * esize};
  const cuuint32_t box[3] = {box_x, head_major ? (cuuint32_t)C : 1u, head_major ? 1u : (cuuint32_t)C};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool encode_token_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t esize, int64_t tokens,
                       int heads, uint32_t box_x, CUtensorMapSwizzle swz, bool head_major) {
  return encode_rows(m, base, dt, esize, tokens, heads, box_x, swz, head_major);
}

cudaError_t launch_fused_chunk(const FusedArgs& a, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(fused_chunk_kernel<false, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(fused_chunk_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemAlloc);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(fused_chunk_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemAlloc);
  if (err != cudaSuccess) return err;
  if (a.batch == 0) return cudaSuccess;
  InputMaps tm;
  memset(&tm, 0, sizeof(tm));
  // with no tokens at all the maps are never used (every sequence is empty)
  const int64_t rows = a.total_tokens;
  const bool ok = rows == 0 || encode_rows(&tm.raw, a.raw_gate, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, a.Hv) &&
                  encode_rows(&tm.k, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, a.Hk) &&
                  encode_rows(&tm.q, a.q ? a.q : a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, a.Hk) &&
                  encode_rows(&tm.v, a.v ? a.v : a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, a.Hv, 64,
                              CU_TENSOR_MAP_SWIZZLE_128B);
  // bf16 outputs (the prefill output, or both readouts of the build) leave through tensor stores,
  // staged as 64-channel halves with the 128-byte swizzle
  const uint32_t out_box = 64u;
  const CUtensorMapSwizzle out_swz = CU_TENSOR_MAP_SWIZZLE_128B;
  const bool out_ok = rows == 0 || !a.out || !a.out_bf16 ||
                      (encode_rows(&tm.out, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, a.Hv, out_box, out_swz,
                                   a.build && a.readout_hm) &&
                       (!a.out2 || encode_rows(&tm.out2, a.out2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, a.Hv,
                                               out_box, out_swz, a.build && a.readout_hm)));
  if (!ok || !out_ok) return cudaErrorInvalidValue;
  dim3 grid(a.Hv, a.batch);
  if (a.build && a.out)
    fused_chunk_kernel<true, true><<<grid, kThreads, kSmemAlloc, stream>>>(a, tm);
  else if (a.build)
    fused_chunk_kernel<true, false><<<grid, kThreads, kSmemAlloc, stream>>>(a, tm);
  else
    fused_chunk_kernel<false, true><<<grid, kThreads, kSmemAlloc, stream>>>(a, tm);
  return cudaGetLastError();
}

}  // namespace kda
