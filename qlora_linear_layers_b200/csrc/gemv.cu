// Decode-sized QLoRA forward (M <= 16 tokens): HBM-bound NF4 GEMV on the
// warp-level tensor-core path.
//
// Page "QLoRA Explained", section "Why it is ever worth paying": a step reads
// every weight at least once, and when few tokens share that read the layer
// waits on memory -- NF4 reads a quarter of the bf16 bytes.  This kernel's job
// is to stream the packed codes at HBM rate.
//
// Design:
//  * A warp owns 16 weight rows (the 16-row operand of mma.m16n8k16) and a
//    slice of the contraction; tokens are the 8-column operand (two tiles for
//    M <= 16).
//  * Inside each 64-wide NF4 block the contraction order is permuted the same
//    way for both operands, so that lane (g, c) holds weight bytes
//    [8c, 8c+8) of rows g and g+8 (two 8-byte loads) and the activations
//    k in [16c, 16c+16) of its token (two 16-byte loads); the sum is unchanged.
//  * A code byte (two weights) becomes a bf16 pair through a 256-entry table
//    of the unscaled NF4 values, replicated per bank so the 32 lanes never
//    conflict.  The block scale multiplies the block's fp32 partial product:
//    Y = sum_b a^_b (sum_{k in b} q[c_k] x_k) -- the real-valued layer with the
//    table rounded to bf16 instead of the scaled weights (both within the
//    layer's tolerance of the exact dequantised weights).
//  * The rank-r rows of A ride along as r/16 extra bf16 row tiles of the same
//    pass, so T = X A^T comes out of the same read of X.
//  * Slices write fp32 partials; one epilogue kernel sums them in slice order,
//    reduces T, adds s (T B^T) in fp32 and writes Y (and T when asked).

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.h"

namespace qnf4 {

namespace {

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kWarps = 8;
constexpr int kMaxBps = 64;                      // NF4 blocks per warp item (bounded)

struct GemvArgs {
  const uint8_t* packed;
  const float* absmax;
  const int8_t* qabsmax;
  const float* dq_scale;
  const float* dq_mean;
  const __nv_bfloat16* X;     // [M, K]
  const __nv_bfloat16* A;     // [r, K]  adapter factor (extra bf16 rows)
  float* part;                // [splits, M, N + r]
  int M, N, K, r;
  int splits, blocks_per_split;
  float q[16];
};

template <bool DQ>
__global__ void __launch_bounds__(kWarps * 32)
k_qlora_gemv(const GemvArgs p) {
  extern __shared__ __align__(16) uint8_t gsm[];
  uint32_t* tbl = reinterpret_cast<uint32_t*>(gsm);            // [256 * 32]: entry e, lane l at e*32 + l
  float* inv127 = reinterpret_cast<float*>(gsm + 256 * 32 * 4);  // [256]

  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const int e = i >> 5;
    tbl[i] = pack_bf16x2(p.q[e >> 4], p.q[e & 15]);   // element 2j (high nibble) low half
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) inv127[i] = __fdiv_rn((float)(i - 127), 127.0f);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t* tb = tbl + lane;
  const float mu = DQ ? __ldg(p.dq_mean) : 0.0f;
  const int wtiles = (p.N + 15) / 16;             // NF4 row tiles
  const int rowtiles = wtiles + (p.r + 15) / 16;  // + bf16 rows of A
  const int NE = p.N + p.r;
  const int nb = p.K / 64;
  const int64_t items = (int64_t)rowtiles * p.splits;
  const int64_t kb_per_row = p.K / 64;

  for (int64_t it = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); it < items;
       it += (int64_t)gridDim.x * kWarps) {
    const int sp = (int)(it / rowtiles);           // slice-major: concurrent warps share X
    const int rt = (int)(it % rowtiles);
    const int b0 = sp * p.blocks_per_split;
    const int b1 = min(nb, b0 + p.blocks_per_split);
    const int t0 = g, t1 = 8 + g;                 // this lane's tokens in the two 8-token tiles
    const bool v0 = t0 < p.M, v1 = t1 < p.M;
    const __nv_bfloat16* x0 = p.X + (int64_t)(v0 ? t0 : 0) * p.K + 16 * c;
    const __nv_bfloat16* x1 = p.X + (int64_t)(v1 ? t1 : 0) * p.K + 16 * c;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int r0;

    if (rt < wtiles) {
      // ---- NF4 rows
      r0 = rt * 16;
      const int rg = min(r0 + g, p.N - 1), rh = min(r0 + g + 8, p.N - 1);
      const uint8_t* pg = p.packed + (int64_t)rg * (p.K / 2) + 8 * c;
      const uint8_t* ph = p.packed + (int64_t)rh * (p.K / 2) + 8 * c;
      for (int b = b0; b < b1; ++b) {
        const uint2 wg = __ldcs(reinterpret_cast<const uint2*>(pg + b * 32));
        const uint2 wh = __ldcs(reinterpret_cast<const uint2*>(ph + b * 32));
        uint4 xa0 = make_uint4(0, 0, 0, 0), xa1 = xa0, xb0 = xa0, xb1 = xa0;
        if (v0) { xa0 = __ldg(reinterpret_cast<const uint4*>(x0 + b * 64)); xa1 = __ldg(reinterpret_cast<const uint4*>(x0 + b * 64) + 1); }
        if (v1) { xb0 = __ldg(reinterpret_cast<const uint4*>(x1 + b * 64)); xb1 = __ldg(reinterpret_cast<const uint4*>(x1 + b * 64) + 1); }
        float ag, ah;
        {
          const int64_t bg = (int64_t)rg * kb_per_row + b, bh = (int64_t)rh * kb_per_row + b;
          if (DQ) {
            ag = __fadd_rn(__fmul_rn(inv127[__ldg(p.qabsmax + bg) + 127], __ldg(p.dq_scale + (bg >> 8))), mu);
            ah = __fadd_rn(__fmul_rn(inv127[__ldg(p.qabsmax + bh) + 127], __ldg(p.dq_scale + (bh >> 8))), mu);
          } else {
            ag = __ldg(p.absmax + bg);
            ah = __ldg(p.absmax + bh);
          }
        }
        const uint32_t bytes_g[2] = {wg.x, wg.y}, bytes_h[2] = {wh.x, wh.y};
        const uint32_t xw0[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
        const uint32_t xw1[8] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w};
        float cb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          // bytes 2s and 2s+1 of this lane's 8 bytes (physical pairs 8c+2s, 8c+2s+1)
          const uint32_t eg0 = (bytes_g[s >> 1] >> (16 * (s & 1))) & 0xFF;
          const uint32_t eg1 = (bytes_g[s >> 1] >> (16 * (s & 1) + 8)) & 0xFF;
          const uint32_t eh0 = (bytes_h[s >> 1] >> (16 * (s & 1))) & 0xFF;
          const uint32_t eh1 = (bytes_h[s >> 1] >> (16 * (s & 1) + 8)) & 0xFF;
          const uint32_t a0 = tb[eg0 * 32], a1 = tb[eh0 * 32], a2 = tb[eg1 * 32], a3 = tb[eh1 * 32];
          mma16816(cb[0], a0, a1, a2, a3, xw0[2 * s], xw0[2 * s + 1]);
          mma16816(cb[1], a0, a1, a2, a3, xw1[2 * s], xw1[2 * s + 1]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          acc[nt][0] = fmaf(ag, cb[nt][0], acc[nt][0]);
          acc[nt][1] = fmaf(ag, cb[nt][1], acc[nt][1]);
          acc[nt][2] = fmaf(ah, cb[nt][2], acc[nt][2]);
          acc[nt][3] = fmaf(ah, cb[nt][3], acc[nt][3]);
        }
      }
    } else {
      // ---- bf16 rows of A: T[m, j] = sum_k X[m, k] A[j, k]
      const int j0 = (rt - wtiles) * 16;
      r0 = p.N + j0;
      const bool jgv = j0 + g < p.r, jhv = j0 + g + 8 < p.r;   // rows past r read as zero
      const __nv_bfloat16* ag4 = p.A + (int64_t)(jgv ? j0 + g : 0) * p.K + 16 * c;
      const __nv_bfloat16* ah4 = p.A + (int64_t)(jhv ? j0 + g + 8 : 0) * p.K + 16 * c;
      for (int b = b0; b < b1; ++b) {
        uint4 ga = make_uint4(0, 0, 0, 0), gb = ga, ha = ga, hb = ga;
        if (jgv) { ga = __ldg(reinterpret_cast<const uint4*>(ag4 + b * 64)); gb = __ldg(reinterpret_cast<const uint4*>(ag4 + b * 64) + 1); }
        if (jhv) { ha = __ldg(reinterpret_cast<const uint4*>(ah4 + b * 64)); hb = __ldg(reinterpret_cast<const uint4*>(ah4 + b * 64) + 1); }
        uint4 xa0 = make_uint4(0, 0, 0, 0), xa1 = xa0, xb0 = xa0, xb1 = xa0;
        if (v0) { xa0 = __ldg(reinterpret_cast<const uint4*>(x0 + b * 64)); xa1 = __ldg(reinterpret_cast<const uint4*>(x0 + b * 64) + 1); }
        if (v1) { xb0 = __ldg(reinterpret_cast<const uint4*>(x1 + b * 64)); xb1 = __ldg(reinterpret_cast<const uint4*>(x1 + b * 64) + 1); }
        const uint32_t gw[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        const uint32_t hw[8] = {ha.x, ha.y, ha.z, ha.w, hb.x, hb.y, hb.z, hb.w};
        const uint32_t xw0[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
        const uint32_t xw1[8] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          mma16816(acc[0], gw[2 * s], hw[2 * s], gw[2 * s + 1], hw[2 * s + 1], xw0[2 * s], xw0[2 * s + 1]);
          mma16816(acc[1], gw[2 * s], hw[2 * s], gw[2 * s + 1], hw[2 * s + 1], xw1[2 * s], xw1[2 * s + 1]);
        }
      }
    }
    // fragment: acc[nt][0..1] = row g, tokens nt*8 + 2c, +1; acc[nt][2..3] = row g+8
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = nt * 8 + 2 * c + (i & 1);
        const int row = r0 + g + ((i & 2) ? 8 : 0);
        const int lim = (rt < wtiles) ? p.N : NE;
        if (tok < p.M && row < lim)
          p.part[((int64_t)sp * p.M + tok) * NE + row] = acc[nt][i];
      }
  }
}

// Y[m, n] = RNbf16( sum_slices part[.][m][n] + sum_j RNbf16(s T[m, j]) B[n, j] )
// with T[m, j] = sum_slices part[.][m][N + j] (slices summed in order; every
// CTA reduces T into shared memory, CTA 0 also writes T_save = RNbf16(T)).
// The adapter product runs on mma.m16n8k16: a warp owns 16 output features
// (rows of B) and both 8-token tiles.
__global__ void __launch_bounds__(256)
k_gemv_epilogue(const float* __restrict__ part, int splits, int M, int N, int r, float s,
                const __nv_bfloat16* __restrict__ B, __nv_bfloat16* __restrict__ Y,
                __nv_bfloat16* __restrict__ T_save) {
  __shared__ __align__(16) uint32_t sT[kDecodeMaxTokens][64 + 4];   // bf16 pairs of s*T (r <= 128)
  const int NE = N + r;
  const int64_t plane = (int64_t)M * NE;
  for (int e = threadIdx.x; e < kDecodeMaxTokens * 64; e += blockDim.x) {
    const int m = e / 64, jp = e % 64;            // token, pair of adapter columns
    float t0 = 0.f, t1 = 0.f;
    if (m < M && 2 * jp < r) {
      for (int k = 0; k < splits; ++k) {
        const float* src = part + k * plane + (int64_t)m * NE + N + 2 * jp;
        t0 = __fadd_rn(t0, src[0]);
        t1 = __fadd_rn(t1, src[1]);
      }
      if (T_save && blockIdx.x == 0)
        *reinterpret_cast<uint32_t*>(T_save + (int64_t)m * r + 2 * jp) = pack_bf16x2(t0, t1);
    }
    sT[m][jp] = pack_bf16x2(__fmul_rn(s, t0), __fmul_rn(s, t1));
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = (blockIdx.x * 8 + warp) * 16;
  if (n0 >= N) return;
  const int ng = min(n0 + g, N - 1), nh = min(n0 + g + 8, N - 1);
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int j0 = 0; j0 < r; j0 += 16) {
    // A = B rows (row-major, j contiguous); B operand = s*T, column j, token
    const uint32_t a0 = *reinterpret_cast<const uint32_t*>(B + (int64_t)ng * r + j0 + 2 * c);
    const uint32_t a1 = *reinterpret_cast<const uint32_t*>(B + (int64_t)nh * r + j0 + 2 * c);
    const uint32_t a2 = (j0 + 8 < r) ? *reinterpret_cast<const uint32_t*>(B + (int64_t)ng * r + j0 + 8 + 2 * c) : 0u;
    const uint32_t a3 = (j0 + 8 < r) ? *reinterpret_cast<const uint32_t*>(B + (int64_t)nh * r + j0 + 8 + 2 * c) : 0u;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const uint32_t b0 = sT[nt * 8 + g][j0 / 2 + c];
      const uint32_t b1 = sT[nt * 8 + g][j0 / 2 + 4 + c];
      mma16816(acc[nt], a0, a1, a2, a3, b0, b1);
    }
  }
  // fragment: acc[nt][0..1] = feature n0+g, tokens nt*8 + 2c, +1; [2..3] = feature n0+g+8
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = nt * 8 + 2 * c + (i & 1);
      const int n = n0 + g + ((i & 2) ? 8 : 0);
      if (tok >= M || n >= N) continue;
      float a = 0.f;
      for (int k = 0; k < splits; ++k) a = __fadd_rn(a, part[k * plane + (int64_t)tok * NE + n]);
      Y[(int64_t)tok * N + n] = __float2bfloat16_rn(a + acc[nt][i]);
    }
}

}  // namespace

// Contraction slices of the decode GEMV: enough 16-row warp items to fill the
// GPU about four times over (fixed target, so sizes and summation order
// depend only on the shapes).
int gemv_splits(int N, int K) {
  const int rowtiles = (N + 15) / 16;
  const int nb = K / 64;
  const int maxs = std::max(1, nb / 8);
  int s = std::min(std::max(1, (4736 + rowtiles - 1) / rowtiles), maxs);
  s = std::max(s, (nb + kMaxBps - 1) / kMaxBps);     // a warp item walks <= kMaxBps blocks
  const int bps = (nb + s - 1) / s;
  return (nb + bps - 1) / bps;
}

size_t gemv_workspace_bytes(int M, int N, int K, int r) {
  return (size_t)gemv_splits(N, K) * M * (N + r) * 4;
}

int launch_qlora_gemv(const nf4_weight* w, const void* X, int M, const void* A, const void* B,
                      int r, float s, void* Y, void* T_save, float* part, const float* q,
                      cudaStream_t st, int num_sms) {
  GemvArgs a{};
  a.packed = w->packed; a.absmax = w->absmax; a.qabsmax = w->qabsmax;
  a.dq_scale = w->dq_scale; a.dq_mean = w->dq_mean;
  a.X = (const __nv_bfloat16*)X; a.A = (const __nv_bfloat16*)A;
  a.part = part;
  a.M = M; a.N = (int)w->rows; a.K = (int)w->cols; a.r = r;
  a.splits = gemv_splits(a.N, a.K);
  const int nb = a.K / 64;
  a.blocks_per_split = (nb + a.splits - 1) / a.splits;
  for (int i = 0; i < 16; ++i) a.q[i] = q[i];
  const int64_t items = (int64_t)((a.N + 15) / 16 + (r + 15) / 16) * a.splits;
  const int grid = (int)std::min<int64_t>((items + kWarps - 1) / kWarps, (int64_t)num_sms * 4);
  constexpr int smem = 256 * 32 * 4 + 256 * 4;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_qlora_gemv<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaFuncSetAttribute(k_qlora_gemv<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    attr = true;
  }
  if (w->double_quant) k_qlora_gemv<true><<<grid, kWarps * 32, smem, st>>>(a);
  else k_qlora_gemv<false><<<grid, kWarps * 32, smem, st>>>(a);
  const int eb = std::max(1, (a.N + 127) / 128);
  k_gemv_epilogue<<<eb, 256, 0, st>>>(part, a.splits, M, a.N, r, s, (const __nv_bfloat16*)B,
                                      (__nv_bfloat16*)Y, (__nv_bfloat16*)T_save);
  return 2;
}

}  // namespace qnf4
