// Merge the adapter into the dequantised base weight, one HBM pass:
//
//   W_merged[n, k] = RNbf16( RN32( w'[n, k] + RN32(s * sum_j B[n, j] A[j, k]) ) )
//   w' = RNbf16(RN32(q[code] * a^))            (the values nf4_dequantize writes)
//
// Page "QLoRA Explained", section "Why a 16-bit adapter will not fold into a
// 4-bit base": a bf16 adapter product cannot be added to 4-bit codes, so the
// base is expanded to 16 bits first and the product added there; page "LoRA
// vs QLoRA", section "How LoRA Works": the effective weight is
// W + (alpha/r) B A, computed once.
//
// A CTA writes a 128-row x 128-column tile.  The rank-r product (a dense
// contraction of depth r <= 128) runs on the warp-level tensor cores: each
// warp owns 16 rows, its A fragments are the rows of B (read from global, L2
// resident), its B fragments the tile's columns of A (staged once per CTA in
// shared memory, transposed by ldmatrix).  The epilogue reads the tile's
// codes (a warp reads its 16 rows' 64 code bytes each), forms the block
// scales, dequantises and adds -- the 4-bit codes and the bf16 output are the
// only HBM traffic of any size.

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "gemm.h"

namespace qnf4 {

namespace {

constexpr int kTile = 128;                 // rows and columns per CTA
constexpr int kAPitch = kTile + 8;         // bf16 per staged row of A (pad: conflict-free ldmatrix)

__device__ __forceinline__ void mma16816_acc(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two 8x8 bf16 matrices from shared memory, transposed (the k16 x n8 B
// fragment of mma.m16n8k16 from a [k][n] row-major tile).
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1) : "r"(addr));
}

template <bool DQ>
__global__ void __launch_bounds__(256)
k_qlora_merge(const uint8_t* __restrict__ packed, int N, int K, const float* __restrict__ absmax,
              const int8_t* __restrict__ qabsmax, const float* __restrict__ dq_scale,
              const float* __restrict__ dq_mean, const __nv_bfloat16* __restrict__ A,
              const __nv_bfloat16* __restrict__ B, int r, float s, __nv_bfloat16* __restrict__ Wm,
              CodeTables tb, int dq_type) {
  __shared__ __align__(16) uint16_t sA[128][kAPitch];    // rows j < r16 of A, the tile's columns
  __shared__ float s_q[16];
  __shared__ float s_inv127[256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int k0 = blockIdx.x * kTile, n0 = blockIdx.y * kTile;
  const int r16 = r < 16 ? 16 : r;                       // depth padded to the MMA's k16
  if (tid < 16) s_q[tid] = tb.q[tid];
  s_inv127[tid] = dq_code_value(tid, dq_type);             // entry c + 128: any code byte
  for (int i = tid; i < r16 * (kTile / 8); i += 256) {
    const int j = i / (kTile / 8), ch = i % (kTile / 8);
    const int k = k0 + ch * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < r && k < K) v = __ldg(reinterpret_cast<const uint4*>(A + (int64_t)j * K + k));
    *reinterpret_cast<uint4*>(&sA[j][ch * 8]) = v;
  }

  // this warp's rows: n0 + 16 warp + g (+8); clamp reads past N (never stored)
  const int ra = min(n0 + 16 * warp + g, N - 1), rb = min(n0 + 16 * warp + g + 8, N - 1);
  // codes of both rows for the tile's 128 columns (64 bytes each), issued early
  // (a 16-byte load holds 32 columns; a last tile of 64 columns reads two)
  uint4 ca[4], cb[4];
  const int nld = min(4, (K - k0) / 32);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ca[i] = i < nld ? __ldg(reinterpret_cast<const uint4*>(packed + ((int64_t)ra * K + k0) / 2) + i)
                    : make_uint4(0u, 0u, 0u, 0u);
    cb[i] = i < nld ? __ldg(reinterpret_cast<const uint4*>(packed + ((int64_t)rb * K + k0) / 2) + i)
                    : make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  float acc[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  for (int kk = 0; kk < r16; kk += 16) {
    // A fragment = rows of B: (g, kk + 2c..), (g+8, ..), (g, kk + 8 + 2c..), (g+8, ..)
    const int j0 = kk + 2 * c, j1 = kk + 8 + 2 * c;
    const uint32_t a0 = j0 < r ? __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)ra * r + j0)) : 0u;
    const uint32_t a1 = j0 < r ? __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)rb * r + j0)) : 0u;
    const uint32_t a2 = j1 < r ? __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)ra * r + j1)) : 0u;
    const uint32_t a3 = j1 < r ? __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)rb * r + j1)) : 0u;
    // B fragments: rows kk..kk+15 of the staged A, columns 8t..8t+7
    const uint32_t row_addr = smem_u32(&sA[kk + (lane & 15)][0]);
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      uint32_t b0, b1;
      ldsm_x2_t(row_addr + t * 16, b0, b1);
      mma16816_acc(acc[t], a0, a1, a2, a3, b0, b1);
    }
  }

  // block scales of both rows, both 64-column blocks of the tile
  const int kb = K / 64;
  float sc[2][2];
  const float mu = DQ ? dq_mean[0] : 0.0f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int rr = h ? rb : ra;
#pragma unroll
    for (int bq = 0; bq < 2; ++bq) {
      const int64_t blk = (int64_t)rr * kb + min(k0 / 64 + bq, kb - 1);
      sc[h][bq] = DQ ? __fadd_rn(__fmul_rn(s_inv127[qabsmax[blk] + 128], __ldg(dq_scale + (blk >> 8))), mu)
                     : __ldg(absmax + blk);
    }
  }
  const uint32_t wa[16] = {ca[0].x, ca[0].y, ca[0].z, ca[0].w, ca[1].x, ca[1].y, ca[1].z, ca[1].w,
                           ca[2].x, ca[2].y, ca[2].z, ca[2].w, ca[3].x, ca[3].y, ca[3].z, ca[3].w};
  const uint32_t wb[16] = {cb[0].x, cb[0].y, cb[0].z, cb[0].w, cb[1].x, cb[1].y, cb[1].z, cb[1].w,
                           cb[2].x, cb[2].y, cb[2].z, cb[2].w, cb[3].x, cb[3].y, cb[3].z, cb[3].w};
  // the tile is staged in shared memory (the staged A is no longer needed),
  // then written with 16-byte stores, whole rows per half-warp
  __syncthreads();
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    // columns 8t + 2c and 8t + 2c + 1 share code byte 4t + c (byte c of word t)
    const int bq = t >> 3;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t byte = ((h ? wb[t] : wa[t]) >> (8 * c)) & 0xFFu;
      const float a = sc[h][bq];
      const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_q[byte >> 4], a)));
      const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_q[byte & 15], a)));
      const float m0 = __fadd_rn(w0, __fmul_rn(s, acc[t][2 * h]));
      const float m1 = __fadd_rn(w1, __fmul_rn(s, acc[t][2 * h + 1]));
      *reinterpret_cast<uint32_t*>(&sA[16 * warp + g + 8 * h][8 * t + 2 * c]) = pack_bf16x2(m0, m1);
    }
  }
  __syncthreads();
  for (int i = tid; i < kTile * (kTile / 8); i += 256) {
    const int row = i / (kTile / 8), ch = i % (kTile / 8);
    const int n = n0 + row, k = k0 + ch * 8;
    if (n < N && k < K)
      *reinterpret_cast<uint4*>(Wm + (int64_t)n * K + k) = *reinterpret_cast<const uint4*>(&sA[row][ch * 8]);
  }
}

// Y[M, K] += D * c * (Bm A): the adapter term of dX under LoRA dropout (Bm =
// s U padded to ldb columns).  Same tiling and tensor-core product as the
// merge; the epilogue adds into the bf16 Y in place.  The keep bits of a
// row's 8-column group come from one Philox block, computed once per quad of
// lanes (lane c of the quad for groups c, c + 4, c + 8, c + 12) and shared by
// shuffle.
template <bool DROP>
__global__ void __launch_bounds__(256)
k_rank_add(const __nv_bfloat16* __restrict__ Bm, int ldb, const __nv_bfloat16* __restrict__ A, int r,
           int M, int K, __nv_bfloat16* __restrict__ Y, Dropout drop) {
  __shared__ __align__(16) uint16_t sA[128][kAPitch];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int k0 = blockIdx.x * kTile, m0 = blockIdx.y * kTile;
  const int r16 = r < 16 ? 16 : r;
  for (int i = tid; i < r16 * (kTile / 8); i += 256) {
    const int j = i / (kTile / 8), ch = i % (kTile / 8);
    const int k = k0 + ch * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < r && k < K) v = __ldg(reinterpret_cast<const uint4*>(A + (int64_t)j * K + k));
    *reinterpret_cast<uint4*>(&sA[j][ch * 8]) = v;
  }
  const int ma = m0 + 16 * warp + g, mb = ma + 8;
  const int ra = min(ma, M - 1), rb = min(mb, M - 1);
  // keep bits of this lane's four 8-column groups, rows ma and mb
  uint32_t kb[2][4] = {{0xFFu, 0xFFu, 0xFFu, 0xFFu}, {0xFFu, 0xFFu, 0xFFu, 0xFFu}};
  if (DROP) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = k0 + 8 * (c + 4 * i);
        const int m = h ? rb : ra;
        kb[h][i] = k < K ? dropout_keep8(((uint64_t)m * (uint64_t)K + (uint64_t)k) >> 3, drop.seed, drop.thr) : 0u;
      }
  }
  __syncthreads();

  float acc[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  for (int kk = 0; kk < r16; kk += 16) {
    const int j0 = kk + 2 * c, j1 = kk + 8 + 2 * c;
    const uint32_t a0 = j0 < r ? __ldg(reinterpret_cast<const uint32_t*>(Bm + (int64_t)ra * ldb + j0)) : 0u;
    const uint32_t a1 = j0 < r ? __ldg(reinterpret_cast<const uint32_t*>(Bm + (int64_t)rb * ldb + j0)) : 0u;
    const uint32_t a2 = j1 < r ? __ldg(reinterpret_cast<const uint32_t*>(Bm + (int64_t)ra * ldb + j1)) : 0u;
    const uint32_t a3 = j1 < r ? __ldg(reinterpret_cast<const uint32_t*>(Bm + (int64_t)rb * ldb + j1)) : 0u;
    const uint32_t row_addr = smem_u32(&sA[kk + (lane & 15)][0]);
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      uint32_t b0, b1;
      ldsm_x2_t(row_addr + t * 16, b0, b1);
      mma16816_acc(acc[t], a0, a1, a2, a3, b0, b1);
    }
  }

  const float cs = DROP ? drop.scale : 1.0f;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const int k = k0 + 8 * t + 2 * c;
    // the group's keep bits from lane (g, t % 4) of this quad; columns 2c, 2c + 1
    uint32_t bits[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t b = DROP ? __shfl_sync(0xffffffffu, kb[h][t >> 2], (lane & ~3) | (t & 3)) : 0xFFu;
      bits[h] = b >> (2 * c);
    }
    if (k >= K) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = h ? mb : ma;
      if (m >= M) continue;
      uint32_t* yp = reinterpret_cast<uint32_t*>(Y + (int64_t)m * K + k);
      const uint32_t y = *yp;
      const float d0 = (bits[h] & 1u) ? __fmul_rn(cs, acc[t][2 * h]) : 0.0f;
      const float d1 = (bits[h] & 2u) ? __fmul_rn(cs, acc[t][2 * h + 1]) : 0.0f;
      *yp = pack_bf16x2(__fadd_rn(bf16_lo(y), d0), __fadd_rn(bf16_hi(y), d1));
    }
  }
}

}  // namespace

void launch_rank_add(const void* Bm, int ldb, const void* A, int r, int M, int K, void* Y,
                     const Dropout& drop, cudaStream_t st) {
  const dim3 grid((unsigned)((K + kTile - 1) / kTile), (unsigned)((M + kTile - 1) / kTile));
  if (drop.on)
    k_rank_add<true><<<grid, 256, 0, st>>>((const __nv_bfloat16*)Bm, ldb, (const __nv_bfloat16*)A, r, M, K,
                                           (__nv_bfloat16*)Y, drop);
  else
    k_rank_add<false><<<grid, 256, 0, st>>>((const __nv_bfloat16*)Bm, ldb, (const __nv_bfloat16*)A, r, M, K,
                                            (__nv_bfloat16*)Y, drop);
}

void launch_merge(const nf4_weight* w, const void* A, const void* B, int r, float s, void* out,
                  cudaStream_t st) {
  const dim3 grid((unsigned)((w->cols + kTile - 1) / kTile), (unsigned)((w->rows + kTile - 1) / kTile));
  const CodeTables& tb = host_tables(w->quant_type);
  if (w->double_quant)
    k_qlora_merge<true><<<grid, 256, 0, st>>>(w->packed, (int)w->rows, (int)w->cols, nullptr, w->qabsmax,
                                              w->dq_scale, w->dq_mean, (const __nv_bfloat16*)A,
                                              (const __nv_bfloat16*)B, r, s, (__nv_bfloat16*)out, tb, w->double_quant);
  else
    k_qlora_merge<false><<<grid, 256, 0, st>>>(w->packed, (int)w->rows, (int)w->cols, w->absmax, nullptr,
                                               nullptr, nullptr, (const __nv_bfloat16*)A,
                                               (const __nv_bfloat16*)B, r, s, (__nv_bfloat16*)out, tb, 0);
}

}  // namespace qnf4
