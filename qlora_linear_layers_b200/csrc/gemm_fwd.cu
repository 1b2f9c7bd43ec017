// Fused NF4-dequantise-in-mainloop QLoRA forward GEMM on tcgen05 tensor cores.
//
//   Y = X deq(W)^T + s (X A^T) B^T
//
// Page "QLoRA Explained", section "Why the expansion cannot be skipped": the
// tensor core cannot decode a 4-bit row index, so for every matmul a kernel
// reads the codes, looks them up in the 16-entry table, multiplies by the
// block scale and hands bf16 values to the tensor core.  Page "LoRA vs
// QLoRA", section "How LoRA Works": the adapter adds (alpha/r) B A.
//
// Design (sm_100a):
//  * The product is computed transposed, Y^T[n, m] = sum_k W'[n, k] X[m, k],
//    so that the dequantised weights are the MMA's A operand.  tcgen05.mma can
//    read A from tensor memory: converter warps write the bf16 weights straight
//    into a TMEM ring with tcgen05.st (no shared-memory round trip); X tiles
//    arrive by TMA (128-byte swizzle) into a shared-memory ring.
//  * CTA tile: 128 weight rows (MMA M) x 256 tokens (MMA N); K step 64, which
//    is exactly one NF4 block per weight row, so a converter thread (one row)
//    needs one scale and one 16-entry bf16 table per K step.  The table is
//    built in registers as two byte planes and indexed with prmt.
//  * The adapter term is r/64 extra K steps of an SS MMA with
//    A = B_lora tile [128 x 64] and B = (s T) tile [256 x 64], accumulated
//    into the same TMEM accumulator.
//  * Persistent: one CTA per SM walks a static tile schedule.  Warp 0 issues
//    TMA, warp 1 issues MMA, warps 2-9 drain the accumulator (epilogue, two
//    warps per TMEM lane quadrant, 128 columns each), warps 10-13 convert NF4
//    to bf16.  The accumulator is released as soon as it is in registers, so
//    the next tile's MMAs overlap the stores.  Every wait is bounded.

#include <algorithm>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.h"

namespace qnf4 {

namespace fwd {

constexpr int BN = 128;          // weight rows per tile (MMA M)
constexpr int BM = 256;          // tokens per tile (MMA N)
constexpr int BK = 64;           // K per stage = one NF4 block
constexpr int STAGES = 4;
constexpr int MAX_NA = 2;        // adapter K steps (r <= 128)
constexpr int X_STAGE_BYTES = BM * BK * 2;      // 32 KB
constexpr int AUX_BYTES = BN * BK * 2;          // 16 KB
constexpr int ACC_COL = 0;                      // accumulator: columns [0, 256)
constexpr int A_COL = 256;                      // A ring: STAGES x 32 columns
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 448;   // 14 warps
constexpr int EPI_WARP0 = 2;       // warps 2-9: epilogue (2 per TMEM lane quadrant)
constexpr int CVT_WARP0 = 10;      // warps 10-13: converters (1 per quadrant)

struct Smem {
  uint8_t x[STAGES][X_STAGE_BYTES];
  uint8_t aux[MAX_NA][AUX_BYTES];
  uint64_t x_full[STAGES], x_empty[STAGES];
  uint64_t a_full[STAGES], a_empty[STAGES];
  uint64_t aux_full[MAX_NA], aux_empty[MAX_NA];
  uint64_t acc_full, acc_empty, done;
  uint32_t tmem_base;
  int abort;
  float inv127[256];
};

constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;

// 16-entry bf16 table for one block, held as byte planes: L[i] holds the low
// bytes of entries 4i..4i+3, H[i] the high bytes.
struct Lut { uint32_t L[4], H[4]; };

__device__ __forceinline__ Lut build_lut(float a, const float* q) {
  uint32_t P[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    P[i] = pack_bf16x2(__fmul_rn(q[2 * i], a), __fmul_rn(q[2 * i + 1], a));
  Lut l;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    l.L[i] = prmt(P[2 * i], P[2 * i + 1], 0x6420);
    l.H[i] = prmt(P[2 * i], P[2 * i + 1], 0x7531);
  }
  return l;
}

// Expand one 32-bit word of packed codes (8 weights, byte j = element 2j in
// the high nibble, 2j+1 in the low nibble) into 4 bf16x2 words ordered by K.
__device__ __forceinline__ void lookup8(uint32_t w, const Lut& l, uint32_t* out) {
  const uint32_t s7 = w & 0x77777777u;                       // entry index within a plane half
  const uint32_t t = ((w >> 1) & 0x44444444u) | 0x32103210u; // pick half 0-7 or 8-15 per byte
  {
    const uint32_t xl = prmt(l.L[0], l.L[1], s7), yl = prmt(l.L[2], l.L[3], s7);
    const uint32_t xh = prmt(l.H[0], l.H[1], s7), yh = prmt(l.H[2], l.H[3], s7);
    const uint32_t lo = prmt(xl, yl, t), hi = prmt(xh, yh, t);
    out[0] = prmt(lo, hi, 0x4051);
    out[1] = prmt(lo, hi, 0x6273);
  }
  {
    const uint32_t s7h = s7 >> 16, th = t >> 16;
    const uint32_t xl = prmt(l.L[0], l.L[1], s7h), yl = prmt(l.L[2], l.L[3], s7h);
    const uint32_t xh = prmt(l.H[0], l.H[1], s7h), yh = prmt(l.H[2], l.H[3], s7h);
    const uint32_t lo = prmt(xl, yl, th), hi = prmt(xh, yh, th);
    out[2] = prmt(lo, hi, 0x4051);
    out[3] = prmt(lo, hi, 0x6273);
  }
}

template <bool DQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_qlora_gemm_fwd(const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_t,
                 const __grid_constant__ CUtensorMap tm_b,
                 const FwdArgs p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_tiles_n = (p.N + BN - 1) / BN;
  const int n_tiles = n_tiles_n * ((p.M + BM - 1) / BM);
  const int nk = p.K / BK;
  const int na = p.na;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&S.x_full[i], 1);
      mbar_init(&S.x_empty[i], 1);
      mbar_init(&S.a_full[i], 128);
      mbar_init(&S.a_empty[i], 1);
    }
    for (int i = 0; i < MAX_NA; ++i) { mbar_init(&S.aux_full[i], 1); mbar_init(&S.aux_empty[i], 1); }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, 256);
    mbar_init(&S.done, 1);
    S.abort = 0;
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    S.inv127[i] = __fdiv_rn((float)(i - 127), 127.0f);
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_t);
    tma_prefetch_desc(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t xi = 0, lt = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++lt) {
        const int n0 = (tile % n_tiles_n) * BN;
        const int m0 = (tile / n_tiles_n) * BM;
        for (int ks = 0; ks < nk + na; ++ks, ++xi) {
          const int s = xi % STAGES;
          if (!mbar_wait(&S.x_empty[s], ((xi / STAGES) & 1) ^ 1, abort, p.status)) break;
          mbar_arrive_expect_tx(&S.x_full[s], X_STAGE_BYTES);
          if (ks < nk) {
            tma_load_2d(S.x[s], &tm_x, &S.x_full[s], ks * BK, m0);
          } else {
            const int j = ks - nk;
            tma_load_2d(S.x[s], &tm_t, &S.x_full[s], j * BK, m0);
            if (!mbar_wait(&S.aux_empty[j], (lt & 1) ^ 1, abort, p.status)) break;
            mbar_arrive_expect_tx(&S.aux_full[j], AUX_BYTES);
            tma_load_2d(S.aux[j], &tm_b, &S.aux_full[j], j * BK, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BN, BM);
      uint32_t xi = 0, ai = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
        ok = mbar_wait(&S.acc_empty, (lt & 1) ^ 1, abort, p.status);
        if (!ok) break;
        tc_fence_after();
        for (int ks = 0; ks < nk && ok; ++ks, ++xi, ++ai) {
          const int s = xi % STAGES, sa = ai % STAGES;
          ok = mbar_wait(&S.x_full[s], (xi / STAGES) & 1, abort, p.status) &&
               mbar_wait(&S.a_full[sa], (ai / STAGES) & 1, abort, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(S.x[s]));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ts(tmem + ACC_COL, tmem + A_COL + sa * 32 + kk * 8, bdesc + (uint64_t)(kk * 2),
                   idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&S.x_empty[s]);
          mma_commit(&S.a_empty[sa]);
        }
        for (int j = 0; j < na && ok; ++j, ++xi) {
          const int s = xi % STAGES;
          ok = mbar_wait(&S.x_full[s], (xi / STAGES) & 1, abort, p.status) &&
               mbar_wait(&S.aux_full[j], lt & 1, abort, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(S.aux[j]));
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(S.x[s]));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(tmem + ACC_COL, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc, 1u);
          mma_commit(&S.x_empty[s]);
          mma_commit(&S.aux_empty[j]);
        }
        if (ok) mma_commit(&S.acc_full);
      }
      // all MMAs issued by this thread are complete once `done` flips
      mma_commit(&S.done);
      mbar_wait(&S.done, 0, abort, p.status);
    }
  } else if (warp >= CVT_WARP0) {
    // ------------------------------------------------------------ NF4 -> bf16 converters
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t tmem_lane = (uint32_t)(quad * 32) << 16;
    const float mu = DQ ? __ldg(p.dq_mean) : 0.0f;
    const int64_t kb_per_row = p.K / 64;
    uint32_t ai = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int n = (tile % n_tiles_n) * BN + row_in_tile;
      const bool valid = n < p.N;
      const uint4* codes = reinterpret_cast<const uint4*>(p.packed + (int64_t)(valid ? n : 0) * (p.K / 2));
      const int64_t blk0 = (int64_t)(valid ? n : 0) * kb_per_row;
      // software pipeline: data for step ks+1 is loaded while step ks converts
      uint4 c0 = __ldcg(codes), c1 = __ldcg(codes + 1);
      float a_raw = 0.0f;
      int qa = 0;
      if (DQ) qa = __ldcg(p.qabsmax + blk0); else a_raw = __ldcg(p.absmax + blk0);
      float sg = DQ ? __ldg(p.dq_scale + (blk0 >> 8)) : 0.0f;
      for (int ks = 0; ks < nk; ++ks, ++ai) {
        uint4 n0v = c0, n1v = c1;
        int nqa = qa;
        float na_raw = a_raw, nsg = sg;
        if (ks + 1 < nk) {
          n0v = __ldcg(codes + 2 * (ks + 1));
          n1v = __ldcg(codes + 2 * (ks + 1) + 1);
          const int64_t b = blk0 + ks + 1;
          if (DQ) { nqa = __ldcg(p.qabsmax + b); nsg = __ldg(p.dq_scale + (b >> 8)); }
          else na_raw = __ldcg(p.absmax + b);
        }
        const float a = DQ ? __fadd_rn(__fmul_rn(S.inv127[qa + 127], sg), mu) : a_raw;
        uint32_t v[32];
        if (valid) {
          const Lut l = build_lut(a, p.q);
          const uint32_t wds[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) lookup8(wds[i], l, v + 4 * i);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        const int sa = ai % STAGES;
        if (!mbar_wait(&S.a_empty[sa], ((ai / STAGES) & 1) ^ 1, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem + tmem_lane + A_COL + sa * 32;
        __syncwarp();
        tmem_st16(taddr, v);
        tmem_st16(taddr + 16, v + 16);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&S.a_full[sa]);
        c0 = n0v; c1 = n1v; qa = nqa; a_raw = na_raw; sg = nsg;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9)
    constexpr int COLS = BM / 2;                 // accumulator columns per epilogue warp
    const int quad = warp & 3;
    const int col0 = ((warp - EPI_WARP0) >> 2) * COLS;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t tmem_lane = (uint32_t)(quad * 32) << 16;
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++lt) {
      const int n0 = (tile % n_tiles_n) * BN;
      const int m0 = (tile / n_tiles_n) * BM + col0;
      if (!mbar_wait(&S.acc_full, lt & 1, abort, p.status)) break;
      __syncwarp();
      tc_fence_after();
      uint32_t packed[COLS / 2];
#pragma unroll
      for (int c = 0; c < COLS; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + tmem_lane + ACC_COL + col0 + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          packed[c / 2 + j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
      }
      tc_fence_before();
      mbar_arrive(&S.acc_empty);
      // lane pairs (n, n+1) swap halves so each lane stores two adjacent
      // outputs of one token row: even lanes row m, odd lanes row m+1
      const bool odd = lane & 1;
      const int ncol = n0 + row_in_tile - (odd ? 1 : 0);
      const int mfirst = m0 + (odd ? 1 : 0);
      const int rows_left = (ncol < p.N) ? p.M - mfirst : 0;
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.Y + (int64_t)mfirst * p.N + ncol);
      const int step = p.N;                      // two bf16 rows = N words
#pragma unroll
      for (int c = 0; c < COLS; c += 2) {
        const uint32_t mine = packed[c / 2];
        const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
        const uint32_t out = odd ? prmt(other, mine, 0x7632) : prmt(mine, other, 0x5410);
        if (c < rows_left) *dst = out;
        dst += step;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fwd

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

bool make_tmap_2d_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_outer);

int launch_qlora_fwd_gemm(const FwdArgs& a, const void* X, const void* sT, const void* Bpad,
                          int RP, cudaStream_t s, int num_sms) {
  using namespace fwd;
  CUtensorMap tmx, tmt, tmb;
  if (!make_tmap_2d_bf16(&tmx, X, a.K, a.M, a.K, BK, BM)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&tmt, sT, RP, a.M, RP, BK, BM)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&tmb, Bpad, RP, a.N, RP, BK, BN)) return QLORA_ERR_CUDA;
  static bool attr_set[2] = {false, false};
  const int n_tiles = ((a.N + BN - 1) / BN) * ((a.M + BM - 1) / BM);
  const int grid = std::min(n_tiles, num_sms);
  if (a.double_quant) {
    if (!attr_set[1]) {
      cudaFuncSetAttribute(k_qlora_gemm_fwd<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
      attr_set[1] = true;
    }
    k_qlora_gemm_fwd<true><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(tmx, tmt, tmb, a);
  } else {
    if (!attr_set[0]) {
      cudaFuncSetAttribute(k_qlora_gemm_fwd<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
      attr_set[0] = true;
    }
    k_qlora_gemm_fwd<false><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(tmx, tmt, tmb, a);
  }
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qnf4
