// Skinny adapter products of the QLoRA layer (rank r <= 128).
//
// Page "LoRA vs QLoRA", section "How LoRA Works: Low-Rank Adapters": the
// adapter adds (alpha/r) B A to the frozen weight; applied to a batch this is
// s (X A^T) B^T.  T = X A^T has only r columns, so it is computed once per
// layer call by this kernel (it reads X once: HBM-bound) and enters the big
// GEMM as r/64 extra K steps.  These skinny products use the warp-level
// mma.sync tensor-core path with ldmatrix from XOR-swizzled shared memory.

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.h"

namespace qnf4 {

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(saddr), "l"(g), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of element (row, k) in a [rows][64] bf16 tile whose 16-byte
// chunks are XOR-swizzled by row (conflict-free ldmatrix).
__device__ __forceinline__ uint32_t swz64(int row, int k) {
  return (uint32_t)(row * 128 + ((((k >> 3) ^ (row & 7))) << 4) + ((k & 7) << 1));
}

// ===========================================================================
// T = X A^T : CTA = 64 tokens x RP adapter columns, 4 warps x 16 tokens.
// ===========================================================================
template <int RP>
__global__ void __launch_bounds__(128)
k_lora_down(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ A, int M,
            int K, int r, float s, __nv_bfloat16* __restrict__ sT, __nv_bfloat16* __restrict__ Tsave) {
  constexpr int TM = 64, KC = 64, STG = 3;
  constexpr int XB = TM * KC * 2, AB = RP * KC * 2;
  extern __shared__ __align__(128) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * TM;
  const int nkc = K / KC;

  auto load_stage = [&](int kc, int stg) {
    uint8_t* xs = sm + stg * (XB + AB);
    uint8_t* as = xs + XB;
    for (int c = tid; c < TM * 8; c += 128) {
      const int row = c >> 3, ch = c & 7;
      const int m = m0 + row;
      const __nv_bfloat16* g = X + (int64_t)(m < M ? m : 0) * K + kc * KC + ch * 8;
      cp_async16(smem_u32(xs) + swz64(row, ch * 8), g, m < M ? 16 : 0);
    }
    for (int c = tid; c < RP * 8; c += 128) {
      const int row = c >> 3, ch = c & 7;
      const __nv_bfloat16* g = A + (int64_t)(row < r ? row : 0) * K + kc * KC + ch * 8;
      cp_async16(smem_u32(as) + swz64(row, ch * 8), g, row < r ? 16 : 0);
    }
  };

  float acc[RP / 8][4];
#pragma unroll
  for (int t = 0; t < RP / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

#pragma unroll
  for (int i = 0; i < STG - 1; ++i) {
    if (i < nkc) load_stage(i, i);
    cp_async_commit();
  }
  for (int kc = 0; kc < nkc; ++kc) {
    cp_async_wait<STG - 2>();
    __syncthreads();
    if (kc + STG - 1 < nkc) load_stage(kc + STG - 1, (kc + STG - 1) % STG);
    cp_async_commit();
    const uint8_t* xs = sm + (kc % STG) * (XB + AB);
    const uint8_t* as = xs + XB;
#pragma unroll
    for (int k16 = 0; k16 < KC / 16; ++k16) {
      uint32_t a0, a1, a2, a3;
      {
        const int row = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int k = k16 * 16 + 8 * (lane >> 4);
        ldsm_x4(smem_u32(xs) + swz64(row, k), a0, a1, a2, a3);
      }
#pragma unroll
      for (int pr = 0; pr < RP / 16; ++pr) {
        uint32_t b0, b1, b2, b3;
        const int row = pr * 16 + (lane & 7) + 8 * (lane >> 4);
        const int k = k16 * 16 + 8 * ((lane >> 3) & 1);
        ldsm_x4(smem_u32(as) + swz64(row, k), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * pr], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * pr + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
  for (int t = 0; t < RP / 8; ++t) {
    const int col = t * 8 + c2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + warp * 16 + g + 8 * h;
      if (m >= M) continue;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      *reinterpret_cast<uint32_t*>(sT + (int64_t)m * RP + col) =
          pack_bf16x2(__fmul_rn(s, v0), __fmul_rn(s, v1));
      if (Tsave && col < r)
        *reinterpret_cast<uint32_t*>(Tsave + (int64_t)m * r + col) = pack_bf16x2(v0, v1);
    }
  }
}

void launch_lora_down(const void* X, const void* A, int M, int K, int r, int RP, float s,
                      void* sT_pad, void* T_save, cudaStream_t st) {
  const int grid = (M + 63) / 64;
  if (RP == 64) {
    constexpr int smem = 3 * (64 * 64 * 2 + 64 * 64 * 2);
    k_lora_down<64><<<grid, 128, smem, st>>>((const __nv_bfloat16*)X, (const __nv_bfloat16*)A, M,
                                             K, r, s, (__nv_bfloat16*)sT_pad, (__nv_bfloat16*)T_save);
  } else {
    constexpr int smem = 3 * (64 * 64 * 2 + 128 * 64 * 2);
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(k_lora_down<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      attr = true;
    }
    k_lora_down<128><<<grid, 128, smem, st>>>((const __nv_bfloat16*)X, (const __nv_bfloat16*)A, M,
                                              K, r, s, (__nv_bfloat16*)sT_pad, (__nv_bfloat16*)T_save);
  }
}

// ===========================================================================
// Zero-padded copy of a narrow matrix: out[rows, RP] = in[rows, r] | 0.
// ===========================================================================
__global__ void k_pad_cols(const __nv_bfloat16* __restrict__ in, int64_t rows, int r, int RP,
                           __nv_bfloat16* __restrict__ out) {
  const int64_t total = rows * RP;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / RP;
    const int c = (int)(i % RP);
    out[i] = c < r ? in[row * r + c] : __float2bfloat16_rn(0.0f);
  }
}

void launch_pad_cols(const void* B, int rows, int r, int RP, void* Bpad, cudaStream_t st) {
  const int64_t total = (int64_t)rows * RP;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, 148 * 8);
  k_pad_cols<<<grid, 256, 0, st>>>((const __nv_bfloat16*)B, rows, r, RP, (__nv_bfloat16*)Bpad);
}

}  // namespace qnf4
