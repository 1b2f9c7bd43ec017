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

// Byte offset of element (row, col) in a [rows][W] bf16 tile (W = 64 or 128)
// whose 16-byte chunks are XOR-swizzled by row.
template <int W>
__device__ __forceinline__ uint32_t swzw(int row, int col) {
  return (uint32_t)(row * W * 2 + ((((col >> 3) ^ (row & 7))) << 4) + ((col & 7) << 1));
}

// ===========================================================================
// Skinny product  S[M, RP] = Z[M, L] * R   (R = A^T or B; rank <= 128)
//   BT = false: R[l, j] = A[j, l]   (A is [r, L], L contiguous)   -> T = X A^T
//   BT = true : R[l, j] = B[l, j]   (B is [L, r], r contiguous)   -> U = dY B
// CTA = 128 rows of Z x RP columns (8 warps x 16 rows) over one slice of the
// contraction (blockIdx.y of `splits`), so that small token counts still
// spread over the GPU.  One slice: the CTA writes
//   Ss[M, RP] = RNbf16(s * S) (zero beyond r), Sraw[M, r] = RNbf16(S);
// several: fp32 partials part[split][M][RP], summed in order by
// k_skinny_reduce.
// ===========================================================================
template <int RP, bool BT, bool DROP>
__global__ void __launch_bounds__(256)
k_lora_skinny(const __nv_bfloat16* __restrict__ Z, const __nv_bfloat16* __restrict__ R, int M,
              int L, int r, float s, int chunks_per_split, __nv_bfloat16* __restrict__ Ss,
              __nv_bfloat16* __restrict__ Sraw, float* __restrict__ part, Dropout drop) {
  constexpr int TM = 128, KC = 64, STG = 3;
  constexpr int XB = TM * KC * 2, AB = RP * KC * 2;
  extern __shared__ __align__(128) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * TM;
  const int nkc_all = (L + KC - 1) / KC;
  const int kc0 = blockIdx.y * chunks_per_split;
  const int nkc = min(nkc_all - kc0, chunks_per_split);

  auto load_stage = [&](int kc, int stg) {
    uint8_t* xs = sm + stg * (XB + AB);
    uint8_t* as = xs + XB;
    for (int c = tid; c < TM * 8; c += 256) {
      const int row = c >> 3, ch = c & 7;
      const int m = m0 + row, l = kc * KC + ch * 8;
      const bool ok = m < M && l < L;
      cp_async16(smem_u32(xs) + swz64(row, ch * 8), ok ? (const void*)(Z + (int64_t)m * L + l) : (const void*)Z,
                 ok ? 16 : 0);
    }
    if (!BT) {
      for (int c = tid; c < RP * 8; c += 256) {
        const int row = c >> 3, ch = c & 7;            // row = j, chunk along l
        const int l = kc * KC + ch * 8;
        const bool ok = row < r && l < L;
        cp_async16(smem_u32(as) + swz64(row, ch * 8), ok ? (const void*)(R + (int64_t)row * L + l) : (const void*)R,
                   ok ? 16 : 0);
      }
    } else {
      for (int c = tid; c < KC * (RP / 8); c += 256) {
        const int row = c / (RP / 8), ch = c % (RP / 8);   // row = l, chunk along j
        const int l = kc * KC + row;
        const bool ok = l < L && ch * 8 < r;
        cp_async16(smem_u32(as) + swzw<RP>(row, ch * 8), ok ? (const void*)(R + (int64_t)l * r + ch * 8) : (const void*)R,
                   ok ? 16 : 0);
      }
    }
  };

  float acc[RP / 8][4];
#pragma unroll
  for (int t = 0; t < RP / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

#pragma unroll
  for (int i = 0; i < STG - 1; ++i) {
    if (i < nkc) load_stage(kc0 + i, i);
    cp_async_commit();
  }
  for (int kc = 0; kc < nkc; ++kc) {
    cp_async_wait<STG - 2>();
    __syncthreads();
    if (kc + STG - 1 < nkc) load_stage(kc0 + kc + STG - 1, (kc + STG - 1) % STG);
    cp_async_commit();
    const uint8_t* xs = sm + (kc % STG) * (XB + AB);
    const uint8_t* as = xs + XB;
    if (DROP) {
      // LoRA dropout on this stage's rows of Z (the adapter input X)
      uint8_t* xw = sm + (kc % STG) * (XB + AB);
      for (int ci = tid; ci < TM * 8; ci += 256) {
        const int row = ci >> 3, ch = ci & 7;
        const int m = m0 + row, l = (kc0 + kc) * KC + ch * 8;
        if (m < M && l < L) {
          uint4* q = reinterpret_cast<uint4*>(xw + swz64(row, ch * 8));
          *q = dropout8(*q, dropout_keep8(((uint64_t)m * (uint64_t)L + (uint64_t)l) >> 3, drop.seed, drop.thr),
                        drop.scale);
        }
      }
      __syncthreads();
    }
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
        if (!BT) {
          const int row = pr * 16 + (lane & 7) + 8 * (lane >> 4);
          const int k = k16 * 16 + 8 * ((lane >> 3) & 1);
          ldsm_x4(smem_u32(as) + swz64(row, k), b0, b1, b2, b3);
        } else {
          const int row = k16 * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
          const int col = pr * 16 + 8 * (lane >> 4);
          ldsm_x4_t(smem_u32(as) + swzw<RP>(row, col), b0, b1, b2, b3);
        }
        mma_bf16_16816(acc[2 * pr], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * pr + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  const int g = lane >> 2, c2 = (lane & 3) * 2;
  const bool direct = gridDim.y == 1;
#pragma unroll
  for (int t = 0; t < RP / 8; ++t) {
    const int col = t * 8 + c2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + warp * 16 + g + 8 * h;
      if (m >= M) continue;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      if (!direct) {
        *reinterpret_cast<float2*>(part + ((int64_t)blockIdx.y * M + m) * RP + col) = make_float2(v0, v1);
        continue;
      }
      if (Ss)
        *reinterpret_cast<uint32_t*>(Ss + (int64_t)m * RP + col) =
            pack_bf16x2(__fmul_rn(s, v0), __fmul_rn(s, v1));
      if (Sraw && col < r)
        *reinterpret_cast<uint32_t*>(Sraw + (int64_t)m * r + col) = pack_bf16x2(v0, v1);
    }
  }
}

// Sum the contraction slices in order and write Ss / Sraw as above.
__global__ void k_skinny_reduce(const float* __restrict__ part, int splits, int M, int RP, int r,
                                float s, __nv_bfloat16* __restrict__ Ss, __nv_bfloat16* __restrict__ Sraw) {
  const int64_t total = (int64_t)M * RP / 2;
  const int64_t plane = (int64_t)M * RP;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = 2 * e;
    float a0 = 0.f, a1 = 0.f;
    for (int k = 0; k < splits; ++k) {
      const float2 v = *reinterpret_cast<const float2*>(part + k * plane + i);
      a0 = __fadd_rn(a0, v.x);
      a1 = __fadd_rn(a1, v.y);
    }
    const int64_t m = i / RP;
    const int col = (int)(i % RP);
    if (Ss) *reinterpret_cast<uint32_t*>(Ss + i) = pack_bf16x2(__fmul_rn(s, a0), __fmul_rn(s, a1));
    if (Sraw && col < r) *reinterpret_cast<uint32_t*>(Sraw + m * r + col) = pack_bf16x2(a0, a1);
  }
}

// Number of contraction slices for an M x L skinny product: about one full
// wave of CTAs on a B200 (148 SMs x 3 resident CTAs), whatever the device, so
// that the workspace size and summation order depend only on the shapes.
constexpr int kOneWave = 148 * 3;
int skinny_splits(int M, int L) {
  const int tiles = (M + 127) / 128;
  const int nkc = (L + 63) / 64;
  int splits = std::min(std::max(1, kOneWave / tiles), nkc);
  const int cps = (nkc + splits - 1) / splits;
  return (nkc + cps - 1) / cps;
}

size_t skinny_workspace_bytes(int M, int L, int RP) {
  const int sp = skinny_splits(M, L);
  return sp > 1 ? (size_t)sp * M * RP * 4 : 0;
}

template <int RP, bool BT, bool DROP>
static void launch_skinny_t(const void* Z, const void* R, int M, int L, int r, float s, void* Ss,
                            void* Sraw, float* part, const Dropout& drop, cudaStream_t st) {
  constexpr int smem = 3 * (128 * 64 * 2 + RP * 64 * 2);
  static std::atomic<unsigned long long> attr_devs{0};
  set_smem_attr_once(k_lora_skinny<RP, BT, DROP>, smem, attr_devs);
  const int splits = skinny_splits(M, L);
  const int nkc = (L + 63) / 64;
  const int cps = (nkc + splits - 1) / splits;
  const dim3 grid((M + 127) / 128, splits);
  k_lora_skinny<RP, BT, DROP><<<grid, 256, smem, st>>>(
      (const __nv_bfloat16*)Z, (const __nv_bfloat16*)R, M, L, r, s, cps, (__nv_bfloat16*)Ss,
      (__nv_bfloat16*)Sraw, part, drop);
}

template <int RP, bool BT>
static void launch_skinny(const void* Z, const void* R, int M, int L, int r, float s, void* Ss,
                          void* Sraw, float* part, const Dropout& drop, cudaStream_t st) {
  if (drop.on) launch_skinny_t<RP, BT, true>(Z, R, M, L, r, s, Ss, Sraw, part, drop, st);
  else launch_skinny_t<RP, BT, false>(Z, R, M, L, r, s, Ss, Sraw, part, drop, st);
  const int splits = skinny_splits(M, L);
  if (splits > 1) {
    const int64_t total = (int64_t)M * RP / 2;
    const int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 8);
    k_skinny_reduce<<<blocks, 256, 0, st>>>(part, splits, M, RP, r, s, (__nv_bfloat16*)Ss,
                                            (__nv_bfloat16*)Sraw);
  }
}

// Returns the number of kernels launched.
int launch_lora_down(const void* X, const void* A, int M, int K, int r, int RP, float s,
                     void* sT_pad, void* T_save, float* part, cudaStream_t st, const Dropout* drop) {
  const Dropout d = drop ? *drop : Dropout{0, 0, 1.0f, 0};
  if (RP == 64) launch_skinny<64, false>(X, A, M, K, r, s, sT_pad, T_save, part, d, st);
  else launch_skinny<128, false>(X, A, M, K, r, s, sT_pad, T_save, part, d, st);
  return skinny_splits(M, K) > 1 ? 2 : 1;
}

int launch_lora_u(const void* dY, const void* B, int M, int N, int r, int RP, float s,
                  void* sU_pad, float* part, cudaStream_t st) {
  const Dropout d{0, 0, 1.0f, 0};
  if (RP == 64) launch_skinny<64, true>(dY, B, M, N, r, s, sU_pad, nullptr, part, d, st);
  else launch_skinny<128, true>(dY, B, M, N, r, s, sU_pad, nullptr, part, d, st);
  return skinny_splits(M, N) > 1 ? 2 : 1;
}

// ===========================================================================
// Split-M reduction products  C = P^T Q  over the token dimension:
//   partial[chunk][TR-tile rows][TC-tile cols] = sum_{m in chunk} P[m, i] Q[m, c]
// P is [M, Rdim] (Rdim contiguous), Q is [M, Cdim] (Cdim contiguous), both bf16.
// dA = s U^T X uses P = sU, Q = X;  dB = s dY^T T uses P = dY, Q = T.
// 8 warps, each 32 x 32 of the tile; operands via ldmatrix.trans.
// ===========================================================================
template <int TR, int TC, bool DROPQ>
__global__ void __launch_bounds__(256)
k_atb_partial(const __nv_bfloat16* __restrict__ P, int ldp, int Rdim,
              const __nv_bfloat16* __restrict__ Q, int ldq, int Cdim, int M, int rows_per_chunk,
              float* __restrict__ part, int Rpad, int Cpad, Dropout drop) {
  constexpr int MC = 32, STG = 3;
  constexpr int PB = MC * TR * 2, QB = MC * TC * 2;
  constexpr int WC = TC / 32;                       // warps along columns
  extern __shared__ __align__(128) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wr = warp / WC, wc = warp % WC;
  const int i0 = blockIdx.x * TR, c0 = blockIdx.y * TC;
  const int mbeg = blockIdx.z * rows_per_chunk;
  const int mend = min(M, mbeg + rows_per_chunk);
  const int nst = (mend - mbeg + MC - 1) / MC;

  auto load_stage = [&](int it, int stg) {
    uint8_t* ps = sm + stg * (PB + QB);
    uint8_t* qs = ps + PB;
    const int mb = mbeg + it * MC;
    for (int c = tid; c < MC * (TR / 8); c += 256) {
      const int row = c / (TR / 8), ch = c % (TR / 8);
      const int m = mb + row, i = i0 + ch * 8;
      const bool ok = m < mend && i < Rdim;
      cp_async16(smem_u32(ps) + swzw<TR>(row, ch * 8), ok ? (const void*)(P + (int64_t)m * ldp + i) : (const void*)P,
                 ok ? 16 : 0);
    }
    for (int c = tid; c < MC * (TC / 8); c += 256) {
      const int row = c / (TC / 8), ch = c % (TC / 8);
      const int m = mb + row, cc = c0 + ch * 8;
      const bool ok = m < mend && cc < Cdim;
      cp_async16(smem_u32(qs) + swzw<TC>(row, ch * 8), ok ? (const void*)(Q + (int64_t)m * ldq + cc) : (const void*)Q,
                 ok ? 16 : 0);
    }
  };

  float acc[2][4][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = acc[a][b][2] = acc[a][b][3] = 0.f;

#pragma unroll
  for (int i = 0; i < STG - 1; ++i) {
    if (i < nst) load_stage(i, i);
    cp_async_commit();
  }
  for (int it = 0; it < nst; ++it) {
    cp_async_wait<STG - 2>();
    __syncthreads();
    if (it + STG - 1 < nst) load_stage(it + STG - 1, (it + STG - 1) % STG);
    cp_async_commit();
    const uint8_t* ps = sm + (it % STG) * (PB + QB);
    const uint8_t* qs = ps + PB;
    if (DROPQ) {
      // LoRA dropout on this stage's rows of Q (the adapter input X)
      uint8_t* qw = sm + (it % STG) * (PB + QB) + PB;
      const int mb = mbeg + it * MC;
      for (int ci = tid; ci < MC * (TC / 8); ci += 256) {
        const int row = ci / (TC / 8), ch = ci % (TC / 8);
        const int m = mb + row, cc = c0 + ch * 8;
        if (m < mend && cc < Cdim) {
          uint4* q = reinterpret_cast<uint4*>(qw + swzw<TC>(row, ch * 8));
          *q = dropout8(*q, dropout_keep8(((uint64_t)m * (uint64_t)ldq + (uint64_t)cc) >> 3, drop.seed, drop.thr),
                        drop.scale);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int k16 = 0; k16 < MC / 16; ++k16) {
      uint32_t af[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        // A = P^T: rows i, cols m.  Stored P[m][i]: .trans gives the fragment.
        const int m = k16 * 16 + (lane & 7) + 8 * (lane >> 4);
        const int i = wr * 32 + a * 16 + 8 * ((lane >> 3) & 1);
        ldsm_x4_t(smem_u32(ps) + swzw<TR>(m, i), af[a][0], af[a][1], af[a][2], af[a][3]);
      }
#pragma unroll
      for (int bp = 0; bp < 2; ++bp) {
        // B = Q: k = m, n = c.  Stored Q[m][c]: .trans gives the fragment.
        uint32_t b0, b1, b2, b3;
        const int m = k16 * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = wc * 32 + bp * 16 + 8 * (lane >> 4);
        ldsm_x4_t(smem_u32(qs) + swzw<TC>(m, c), b0, b1, b2, b3);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          mma_bf16_16816(acc[a][2 * bp], af[a][0], af[a][1], af[a][2], af[a][3], b0, b1);
          mma_bf16_16816(acc[a][2 * bp + 1], af[a][0], af[a][1], af[a][2], af[a][3], b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();

  float* out = part + (int64_t)blockIdx.z * Rpad * Cpad;
  const int g = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = i0 + wr * 32 + a * 16 + g + 8 * h;
        const int c = c0 + wc * 32 + b * 8 + cq;
        *reinterpret_cast<float2*>(out + (int64_t)i * Cpad + c) =
            make_float2(acc[a][b][2 * h], acc[a][b][2 * h + 1]);
      }
}

// out[i, c] = RNbf16(s * sum_{chunk = 0..n-1} part[chunk][i][c]) for i < Rdim, c < Cdim,
// summed in chunk order (deterministic).
__global__ void k_reduce_partials(const float* __restrict__ part, int nchunks, int Rpad, int Cpad,
                                  int Rdim, int Cdim, float s, __nv_bfloat16* __restrict__ out) {
  const int64_t total = (int64_t)Rdim * Cdim;
  const int64_t plane = (int64_t)Rpad * Cpad;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / Cdim, c = e % Cdim;
    const float* p = part + i * Cpad + c;
    float acc = 0.f;
    for (int k = 0; k < nchunks; ++k) acc = __fadd_rn(acc, p[k * plane]);
    out[e] = __float2bfloat16_rn(__fmul_rn(s, acc));
  }
}

// Split count of the token dimension: about one full wave of CTAs on a B200
// (148 SMs x 3 resident CTAs) whatever the device, so that workspace size and
// summation order depend only on the shapes.
int atb_chunks(int tiles, int M) {
  int want = std::max(1, kOneWave / tiles);
  int maxc = std::max(1, (M + 31) / 32);
  return std::min(want, maxc);
}

// C[Rdim, Cdim] = s * P^T Q over M rows, bf16 out.  `part` must hold
// chunks * Rpad * Cpad floats (see atb_workspace_floats).
void launch_atb(const void* P, int ldp, int Rdim, const void* Q, int ldq, int Cdim, int M, float s,
                void* out, float* part, int num_sms, cudaStream_t st, const Dropout* dropq) {
  const Dropout d = dropq ? *dropq : Dropout{0, 0, 1.0f, 0};
  const bool tall = Rdim >= Cdim;                  // choose the tile shape by aspect
  const int TR = tall ? 128 : 64, TC = tall ? 64 : 128;
  const int gr = (Rdim + TR - 1) / TR, gc = (Cdim + TC - 1) / TC;
  const int Rpad = gr * TR, Cpad = gc * TC;
  const int chunks = atb_chunks(gr * gc, M);
  const int rows_per_chunk = (((M + chunks - 1) / chunks) + 31) / 32 * 32;
  const int nch = (M + rows_per_chunk - 1) / rows_per_chunk;
  const dim3 grid(gr, gc, nch);
  constexpr int smem = 3 * (32 * 128 * 2 + 32 * 64 * 2);
  auto run = [&](auto kern) {
    kern<<<grid, 256, smem, st>>>((const __nv_bfloat16*)P, ldp, Rdim, (const __nv_bfloat16*)Q, ldq, Cdim,
                                  M, rows_per_chunk, part, Rpad, Cpad, d);
  };
  if (tall) {
    if (d.on) run(k_atb_partial<128, 64, true>);
    else run(k_atb_partial<128, 64, false>);
  } else {
    if (d.on) run(k_atb_partial<64, 128, true>);
    else run(k_atb_partial<64, 128, false>);
  }
  const int64_t total = (int64_t)Rdim * Cdim;
  const int rb = (int)std::min<int64_t>((total + 255) / 256, (int64_t)num_sms * 8);
  k_reduce_partials<<<std::max(rb, 1), 256, 0, st>>>(part, nch, Rpad, Cpad, Rdim, Cdim, s,
                                                     (__nv_bfloat16*)out);
}

size_t atb_workspace_floats(int Rdim, int Cdim, int M) {
  const bool tall = Rdim >= Cdim;
  const int TR = tall ? 128 : 64, TC = tall ? 64 : 128;
  const int gr = (Rdim + TR - 1) / TR, gc = (Cdim + TC - 1) / TC;
  const int chunks = atb_chunks(gr * gc, M);
  const int rows_per_chunk = (((M + chunks - 1) / chunks) + 31) / 32 * 32;
  const int nch = (M + rows_per_chunk - 1) / rows_per_chunk;
  return (size_t)nch * gr * TR * gc * TC;
}

// ===========================================================================
// Dequantise-transpose: Wt[k, n] = deq(W)[n, k], bf16, same values as
// nf4_dequantize.  CTA tile 64 rows (n) x 128 columns (k) = 2 NF4 blocks per
// row; 256 threads, each dequantises 32 weights into shared memory, then the
// tile is written out transposed with 16-byte stores.
// ===========================================================================
// Dequantise-transpose: Wt[k, n] = deq(W)[n, k], bf16, same values as
// nf4_dequantize.  CTA tile 64 rows (n) x 128 columns (k) = 2 NF4 blocks per
// row; thread (p, q) expands rows 2p and 2p + 1, columns [16q, 16q + 16), and
// stores each column's pair of rows as one 32-bit word of the transposed tile
// in shared memory (a warp's 32 words are consecutive: no bank conflicts);
// the CTA then writes the tile's 128 rows of 128 bytes with 16-byte stores.
// ===========================================================================
__global__ void __launch_bounds__(256)
k_dequant_t(const uint8_t* __restrict__ packed, int N, int K, int dq,
            const float* __restrict__ absmax, const int8_t* __restrict__ qabsmax,
            const float* __restrict__ dq_scale, const float* __restrict__ dq_mean,
            __nv_bfloat16* __restrict__ Wt, CodeTables tb) {
  constexpr int kPitch = 36;                       // words per transposed row (32 + pad, 16-byte rows)
  __shared__ __align__(16) uint32_t tileT[128 * kPitch];
  __shared__ float s_q[16];
  if (threadIdx.x < 16) s_q[threadIdx.x] = tb.q[threadIdx.x];
  const int n0 = blockIdx.y * 64, k0 = blockIdx.x * 128;
  const int tid = threadIdx.x;
  const int pr = tid & 31, qk = tid >> 5;          // row pair, 16-column group
  // codes and scales of rows 2pr, 2pr + 1 (clamped: rows past N write zeros)
  uint2 cw[2];
  float a[2];
  const int k = k0 + 16 * qk;
  const bool kin = k < K;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int n = n0 + 2 * pr + h;
    const bool in = kin && n < N;
    const int64_t e = (int64_t)(in ? n : 0) * K + (in ? k : 0);
    cw[h] = in ? *reinterpret_cast<const uint2*>(packed + (e >> 1)) : make_uint2(0u, 0u);
    const int64_t blk = e >> 6;
    if (!in) a[h] = 0.0f;
    else if (dq) a[h] = __fadd_rn(__fmul_rn(dq_code_value((int)qabsmax[blk] + 128, dq), dq_scale[blk >> 8]), dq_mean[0]);
    else a[h] = absmax[blk];
  }
  __syncthreads();                                 // s_q
#pragma unroll
  for (int b = 0; b < 8; ++b) {                    // code byte b: columns 2b (high nibble), 2b + 1
    const uint32_t c0 = ((b < 4 ? cw[0].x : cw[0].y) >> (8 * (b & 3))) & 0xFFu;
    const uint32_t c1 = ((b < 4 ? cw[1].x : cw[1].y) >> (8 * (b & 3))) & 0xFFu;
    const uint32_t even = pack_bf16x2(__fmul_rn(s_q[c0 >> 4], a[0]), __fmul_rn(s_q[c1 >> 4], a[1]));
    const uint32_t odd = pack_bf16x2(__fmul_rn(s_q[c0 & 15], a[0]), __fmul_rn(s_q[c1 & 15], a[1]));
    tileT[(16 * qk + 2 * b) * kPitch + pr] = even;
    tileT[(16 * qk + 2 * b + 1) * kPitch + pr] = odd;
  }
  __syncthreads();
  const bool full_n = n0 + 64 <= N;
  for (int i = tid; i < 128 * 8; i += 256) {
    const int kr = i >> 3, ch = i & 7;             // transposed row, 16-byte chunk (8 columns n)
    const int kk = k0 + kr, nn = n0 + ch * 8;
    if (kk >= K) continue;
    const uint4 v = *reinterpret_cast<const uint4*>(&tileT[kr * kPitch + ch * 4]);
    if (full_n || nn + 8 <= N) {
      *reinterpret_cast<uint4*>(Wt + (int64_t)kk * N + nn) = v;
    } else if (nn < N) {                           // N % 8 == 0: never partial
      *reinterpret_cast<uint4*>(Wt + (int64_t)kk * N + nn) = v;
    }
  }
}

void launch_dequant_t(const nf4_weight* w, void* Wt, cudaStream_t st) {
  const dim3 grid((unsigned)((w->cols + 127) / 128), (unsigned)((w->rows + 63) / 64));
  k_dequant_t<<<grid, 256, 0, st>>>(w->packed, (int)w->rows, (int)w->cols, w->double_quant,
                                    w->absmax, w->qabsmax, w->dq_scale, w->dq_mean,
                                    (__nv_bfloat16*)Wt, host_tables(w->quant_type));
}

// At_pad[k, j] = A[j, k] for j < r, 0 for r <= j < RP.
__global__ void k_transpose_pad(const __nv_bfloat16* __restrict__ A, int r, int K, int RP,
                                __nv_bfloat16* __restrict__ At) {
  const int64_t total = (int64_t)K * RP;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t k = e / RP;
    const int j = (int)(e % RP);
    At[e] = j < r ? A[(int64_t)j * K + k] : __float2bfloat16_rn(0.0f);
  }
}

void launch_transpose_pad(const void* A, int r, int K, int RP, void* At, cudaStream_t st) {
  const int64_t total = (int64_t)K * RP;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, 148 * 8);
  k_transpose_pad<<<grid, 256, 0, st>>>((const __nv_bfloat16*)A, r, K, RP, (__nv_bfloat16*)At);
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
