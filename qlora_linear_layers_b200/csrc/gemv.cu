// Decode-sized QLoRA forward (M <= 16 tokens): HBM-bound NF4 GEMV on the
// warp-level tensor-core path.
//
// Page "QLoRA Explained", section "Why it is ever worth paying": a step reads
// every weight at least once, and when few tokens share that read the layer
// waits on memory -- NF4 reads a quarter of the bf16 bytes.  This kernel's job
// is to stream the packed codes at HBM rate.
//
// Design:
//  * Work units are (row group, stage): a row group is 64 NF4 rows (or 16
//    rows of the adapter factor A), a stage is 8 NF4 blocks (512 columns) of
//    it.  The unit list (adapter groups first) is cut into P = min(148, units)
//    equal, non-empty contiguous ranges, one per CTA (a partition fixed by the
//    shapes: results do not depend on the device).  A CTA's range covers
//    parts of one to three row groups; each part ("piece") leaves one fp32
//    partial per output, and the pieces of a row group belong to consecutive
//    CTAs.
//  * One producer warp streams the CTA's units through a ring of TMA stages
//    (five for one token tile, three for two), two or three copies per
//    stage: the codes as two 64-row x 128-byte boxes (128B-swizzled: wide
//    rows, conflict-free reads) or the 8 blocks of 16 rows of A as one 3-D
//    box, and the tokens' 8 blocks of X as one 3-D box (8 or 16 rows x 64
//    per block, 128B-swizzled).
//  * Sixteen consumer warps: warp (j, h) takes NF4 block j of the stage for
//    rows [32h, 32h+32) as two 16-row tiles of mma.m16n8k16 (tokens are the
//    8-column operand, one or two tiles).
//  * Inside each 64-wide NF4 block the contraction order is permuted the same
//    way for both operands, so that lane (g, c) takes code bytes [8c, 8c+8) of
//    the tile's rows 2g and 2g+1 (its MMA rows g and g+8: any row order works,
//    and this one keeps the code loads free of bank conflicts) and the
//    activations k in [16c, 16c+16) of its token; the
//    sum is unchanged.
//  * A code byte (two weights) becomes a bf16 pair through a 256-entry table
//    of the unscaled NF4 values, replicated per bank so the 32 lanes never
//    conflict (index: one shift and one mask-or).  The block scale multiplies
//    the block's fp32 partial product: Y = sum_b a^_b (sum_{k in b} q[c_k] x_k)
//    -- the real-valued layer with the table rounded to bf16 instead of the
//    scaled weights (both within the layer's tolerance of the exact
//    dequantised weights).  Each lane decodes the scale of one of its warp's
//    32 rows one unit ahead; the others take them by shuffle.
//  * At the end of a piece the eight warps' sums (different blocks) are added
//    in warp order through shared memory and written as the piece's partial.
//  * The epilogue kernel sums each output's pieces in order, reduces T,
//    adds s (T B^T) in fp32 and writes Y (and T when asked).

#include <algorithm>
#include <cstdint>
#include <cuda.h>
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

// Same with a zero accumulator input.
__device__ __forceinline__ void mma16816_z(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

constexpr int kBlk = 8;                          // NF4 blocks per stage
constexpr int kCW = 2 * kBlk;                    // consumer warps: (block, row half)
constexpr int kThreads = (kCW + 1) * 32;         // + the producer warp
constexpr int kRows = 64;                        // NF4 rows per row group
constexpr int kARows = 16;                       // adapter rows per row group
constexpr int kWBytes = 16384;                   // 64 rows x 256 B of codes, or 8 x 16 A rows x 128 B
// per stage: weights, then X of the stage's 8 blocks (8 * NT rows x 128 B each)
template <int NT> __host__ __device__ constexpr int stage_bytes() { return kWBytes + kBlk * 1024 * NT; }
// Shared-memory map (shared-window addresses): [start, 64 KB) the small state
// and, for one token tile, one ring stage; [64 KB, 128 KB) the pair table;
// [128 KB, ...) the other ring stages.  The table's fixed address lets one
// prmt build a lookup address (see the consumers).
constexpr uint32_t kTableAddr = 0x10000;
constexpr uint32_t kRingAddr = 0x20000;
template <int NT> __host__ __device__ constexpr int n_stages_low() { return NT == 1 ? 1 : 0; }
template <int NT> __host__ __device__ constexpr int n_stages_high() { return NT == 1 ? 4 : 3; }
template <int NT> __host__ __device__ constexpr int n_stages() { return n_stages_low<NT>() + n_stages_high<NT>(); }
constexpr int kMaxParts = 148;                   // ranges of the unit list (at most)

struct GemvArgs {
  const int8_t* qabsmax;
  const float* absmax;
  const float* dq_scale;
  const float* dq_mean;
  float* part;                // [pieces, M, N + r]
  int* status;
  int M, N, K, r;
  int nb;                     // NF4 blocks per row
  int spr;                    // stages per row group: ceil(nb / 8)
  int nat;                    // adapter row groups: ceil(r / 16)
  int nrg;                    // NF4 row groups: ceil(N / 64)
  int64_t U;                  // units: (nat + nrg) * spr
  int P;                      // ranges (CTAs): min(148, U)
  uint32_t smem_base;         // shared-window address of dynamic shared memory
  int dq_type;                // 1: int8 block-scale codes, 2: E4M3
  float q[16];
};

template <int NT>
struct GemvSmem {                                // at the start of dynamic shared memory
  float red[kBlk][kRows * 16];                   // per-block sums of a piece
  float inv127[256];
  uint64_t full[n_stages<NT>()], empty[n_stages<NT>()];
  int abort;
};
// byte offset (from the start of dynamic shared memory) of the low ring stage
template <int NT> __host__ __device__ constexpr uint32_t low_stage_off() {
  return (uint32_t)((sizeof(GemvSmem<NT>) + 1023) / 1024 * 1024);
}

// Range (CTA) that owns unit x when U units are cut into P <= U ranges
// start(j) = floor(j U / P); every range is non-empty.
__host__ __device__ __forceinline__ int64_t owner_cta(int64_t x, int64_t U, int P) {
  return ((x + 1) * P - 1) / U;
}

// Number of pieces (owning CTAs) of row group rgp.
__host__ __device__ __forceinline__ int n_pieces(int rgp, int spr, int64_t U, int P) {
  return (int)(owner_cta((int64_t)rgp * spr + spr - 1, U, P) - owner_cta((int64_t)rgp * spr, U, P) + 1);
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" :: "n"(kCW * 32) : "memory");
}

// Wait for a stage's copy after an abort, bounded, ignoring the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const int* st) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t limit = wait_limit_ns(st);
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit) break;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// 16 bf16 of row `row` of a 128-byte-swizzled 64-column bf16 tile: logical
// columns [16c, 16c+16) (16-byte chunks 2c and 2c+1, stored at chunk ^ (row & 7)).
__device__ __forceinline__ void lds_row16(const uint8_t* tile, int row, int c, uint32_t (&w)[8]) {
  const uint8_t* base = tile + row * 128;
  const uint4 lo = *reinterpret_cast<const uint4*>(base + (((2 * c) ^ (row & 7)) << 4));
  const uint4 hi = *reinterpret_cast<const uint4*>(base + (((2 * c + 1) ^ (row & 7)) << 4));
  w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
  w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
}

template <bool DQ, int NT>
__global__ void __launch_bounds__(kThreads, 1)
k_qlora_gemv(const __grid_constant__ CUtensorMap tm_codes,   // packed [N, K/2] u8, box 128 x 64, 128B swizzle
             const __grid_constant__ CUtensorMap tm_a,       // A as [K/64][r][64] bf16, box 64 x 16 x 8, 128B swizzle
             const __grid_constant__ CUtensorMap tm_x,       // X as [K/64][M][64] bf16, box 64 x 8*NT x 8, 128B swizzle
             const GemvArgs p) {
  extern __shared__ __align__(1024) uint8_t gsm_raw[];
  const uint32_t base = smem_u32(gsm_raw);
  if (base != p.smem_base) {                     // the map needs the base the host sized it for
    if (threadIdx.x == 0) set_status(p.status, QLORA_ERR_CUDA);
    return;
  }
  GemvSmem<NT>& S = *reinterpret_cast<GemvSmem<NT>*>(gsm_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kStages = n_stages<NT>();
  constexpr uint32_t kTx = stage_bytes<NT>();
  auto stage_ptr = [&](int s) -> uint8_t* {
    return s < n_stages_low<NT>() ? gsm_raw + low_stage_off<NT>() + s * stage_bytes<NT>()
                                  : gsm_raw + (kRingAddr - base) + (s - n_stages_low<NT>()) * stage_bytes<NT>();
  };

  // byte-pair -> bf16 pair table: entry e (a code byte) for lane l at shared
  // address kTableAddr + e * 256 + l * 4 (a copy per lane: no bank conflicts)
  {
    uint32_t* tbl = reinterpret_cast<uint32_t*>(gsm_raw + (kTableAddr - base));
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
      const int e = i >> 5, l = i & 31;
      tbl[e * 64 + l] = pack_bf16x2(p.q[e >> 4], p.q[e & 15]);   // element 2j (high nibble) low half
    }
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) S.inv127[i] = dq_code_value(i, p.dq_type);   // entry c + 128: any code byte
  if (threadIdx.x == 0) {
    S.abort = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.full[i], 1);
      mbar_init(&S.empty[i], kCW);
    }
    mbar_fence_init();
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_x);
  }
  __syncthreads();

  asm volatile("griddepcontrol.launch_dependents;");   // the epilogue may start its prologue
  volatile int* abort = &S.abort;
  const int64_t u0 = (int64_t)blockIdx.x * p.U / p.P;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * p.U / p.P;

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t k = 0;
      bool ok = true;
      int rgp = (int)(u0 / p.spr), st = (int)(u0 - (int64_t)rgp * p.spr);
      // test switch: CTA 0 leaves its first stage unfilled, so that its
      // consumers' bounded waits run out (QLORA_ERR_TIMEOUT)
      const bool withhold = blockIdx.x == 0 &&
                            reinterpret_cast<const volatile DevState*>(p.status)->withhold_first_fill != 0;
      int s = 0;
      uint32_t ph = 0;                           // phase of stage s's current use
      for (int64_t u = u0; u < u1; ++u, ++k, s = (s + 1 == kStages) ? 0 : s + 1, ph ^= (s == 0)) {
        if (!(ok = mbar_wait(&S.empty[s], ph ^ 1, abort, p.status))) break;
        const int b = st * kBlk;
        uint8_t* dst = stage_ptr(s);
        if (withhold && k == 0) {
          if (++st == p.spr) { st = 0; ++rgp; }
          continue;
        }
        mbar_arrive_expect_tx(&S.full[s], kTx);
        if (rgp < p.nat) {
          tma_load_3d(dst, &tm_a, &S.full[s], 0, rgp * kARows, b);
        } else {
          const int row0 = (rgp - p.nat) * kRows;
          tma_load_2d(dst, &tm_codes, &S.full[s], b * 32, row0);
          tma_load_2d(dst + 8192, &tm_codes, &S.full[s], b * 32 + 128, row0);
        }
        tma_load_3d(dst + kWBytes, &tm_x, &S.full[s], 0, 0, b);
        if (++st == p.spr) { st = 0; ++rgp; }
      }
      if (!ok) {
        // a wait gave up: let the copies in flight land before the CTA exits
        for (uint32_t i = (k > (uint32_t)kStages ? k - kStages : 0); i < k; ++i)
          drain_wait(&S.full[i % kStages], (i / kStages) & 1, p.status);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int w = warp;
  const int j = w & (kBlk - 1), h = w >> 3;      // block of the stage, row half
  const int g = lane >> 2, c = lane & 3;
  // prmt source of a lookup address: byte 0 = lane * 4, byte 2 = 1
  // (kTableAddr), bytes 1 and 3 zero; the code byte goes to byte 1
  const uint32_t tsrc = kTableAddr | ((uint32_t)lane * 4);
  const float mu = DQ ? __ldg(p.dq_mean) : 0.0f;
  const int NE = p.N + p.r;
  // MMA row i of a 16-row tile holds weight row 2i (i < 8) or 2(i - 8) + 1:
  // lane (g, c) reads rows 2g and 2g + 1, whose 128-byte swizzle patterns
  // (row & 7) put a half-warp's 16 eight-byte reads on all 32 banks.
  // codes: box (j >> 2), logical bytes [(j & 3) * 32 + 8c, +8) of a 128-byte row
  const int cj = (j & 3) * 2 + (c >> 1);
  const int code_off_g = (j >> 2) * 8192 + (32 * h + 2 * g) * 128 + ((cj ^ ((2 * g) & 7)) << 4) + 8 * (c & 1);
  const int code_off_h = (j >> 2) * 8192 + (32 * h + 2 * g + 1) * 128 + ((cj ^ ((2 * g + 1) & 7)) << 4) + 8 * (c & 1);
  const int xoff = kWBytes + j * 1024 * NT;      // X of block j: 8*NT rows x 128 B
  // the row whose scale this lane decodes: tile (c & 1), MMA row g + 8 (c >> 1)
  const int srow = 32 * h + 16 * (c & 1) + 2 * g + (c >> 1);

  float acc[2][NT][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][nt][i] = 0.f;

  // sum the eight blocks' values of the current piece (in block order) and
  // write its partial
  auto flush = [&](int rgp) {
    const bool ad = rgp < p.nat;
    float* red = S.red[j];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = 32 * h + 16 * t + 2 * g + ((i & 2) ? 1 : 0);
          const int tok = nt * 8 + 2 * c + (i & 1);
          if (!ad || (h == 0 && t == 0)) red[row * 16 + tok] = acc[t][nt][i];
          acc[t][nt][i] = 0.f;
        }
    consumer_sync();
    const int64_t first = owner_cta((int64_t)rgp * p.spr, p.U, p.P);
    const int64_t piece = blockIdx.x - first;
    const int nrows = ad ? kARows : kRows;
    const int col0 = ad ? p.N + rgp * kARows : (rgp - p.nat) * kRows;
    const int lim = ad ? NE : p.N;
    for (int o = w * 32 + lane; o < nrows * 16; o += kCW * 32) {
      const int row = o >> 4, tok = o & 15;
      float v = 0.f;
#pragma unroll
      for (int jj = 0; jj < kBlk; ++jj) v = __fadd_rn(v, S.red[jj][o]);
      if (tok < p.M && col0 + row < lim)
        p.part[((int64_t)piece * p.M + tok) * NE + col0 + row] = v;
    }
    consumer_sync();
  };

  int cur = -1;
  bool ok = true;
  int rgp = (int)(u0 / p.spr), st = (int)(u0 - (int64_t)rgp * p.spr);
  // scale inputs of units u, u+1, u+2 (loaded three units ahead of use: the
  // first touch of a row's codes comes from DRAM)
  constexpr int kAhead = 3;
  int sq[kAhead] = {0, 0, 0};
  float sf[kAhead] = {0.f, 0.f, 0.f};
  int prgp = rgp, pst = st;                       // next unit to prefetch
  // the prefetch cursor's block index (row srow of row group prgp, block pst*8+j)
  int64_t pbi = 0;
  auto set_pbi = [&]() {
    pbi = (int64_t)min((prgp - p.nat) * kRows + srow, p.N - 1) * p.nb + pst * kBlk + j;
  };
  set_pbi();
  auto load_next = [&](int& qs_, float& fs_) {
    if (prgp >= p.nat && pst * kBlk + j < p.nb) {
      if (DQ) {
        qs_ = __ldg(p.qabsmax + pbi);
        fs_ = __ldg(p.dq_scale + (pbi >> 8));
      } else {
        fs_ = __ldg(p.absmax + pbi);
      }
    }
    if (++pst == p.spr) { pst = 0; ++prgp; set_pbi(); }
    else pbi += kBlk;
  };
  const int L = (int)(u1 - u0);
#pragma unroll
  for (int d = 0; d < kAhead; ++d)
    if (d < L) load_next(sq[d], sf[d]);
  int s = 0;
  uint32_t ph = 0;                               // phase of stage s's current use
  for (int i = 0; i < L; ++i, s = (s + 1 == kStages) ? 0 : s + 1, ph ^= (s == 0)) {
    const int b = st * kBlk + j;
    int nrgp = rgp, nst = st + 1;                 // the next unit
    if (nst == p.spr) { nst = 0; ++nrgp; }
    if (rgp != cur) {
      if (cur >= 0) flush(cur);
      cur = rgp;
    }
    const int qs = sq[0];
    const float fs = sf[0];
#pragma unroll
    for (int d = 0; d + 1 < kAhead; ++d) { sq[d] = sq[d + 1]; sf[d] = sf[d + 1]; }
    if (i + kAhead < L) load_next(sq[kAhead - 1], sf[kAhead - 1]);
    if (!(ok = mbar_wait(&S.full[s], ph, abort, p.status))) break;
    const uint8_t* sb = stage_ptr(s);
    const bool nf4 = rgp >= p.nat;
    if (b < p.nb && (nf4 || h == 0)) {
      uint32_t xw[NT][8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (nt * 8 + g < p.M) {
          lds_row16(sb + xoff, nt * 8 + g, c, xw[nt]);
        } else {                                 // token rows past M are zero
#pragma unroll
          for (int i = 0; i < 8; ++i) xw[nt][i] = 0u;
        }
      }
      if (nf4) {
        // ---- 32 NF4 rows x one block
        uint2 wg[2], wh[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          wg[t] = *reinterpret_cast<const uint2*>(sb + code_off_g + t * 16 * 128);
          wh[t] = *reinterpret_cast<const uint2*>(sb + code_off_h + t * 16 * 128);
        }
        float cb[2][NT][4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // bytes 2kk and 2kk+1 of this lane's 8 bytes (physical pairs 8c+2kk, 8c+2kk+1)
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t vg = (kk < 2) ? wg[t].x : wg[t].y;
            const uint32_t vh = (kk < 2) ? wh[t].x : wh[t].y;
            // lookup address kTableAddr + byte * 256 + lane * 4: one prmt
            // (selector 0x76j4: tsrc byte 0, code byte j, tsrc bytes 2 and 3)
            const uint32_t s0 = (kk & 1) ? 0x7624u : 0x7604u;   // byte 2kk of the lane's 8
            const uint32_t s1 = (kk & 1) ? 0x7634u : 0x7614u;   // byte 2kk + 1
            const uint32_t a0 = lds_u32(prmt(vg, tsrc, s0));
            const uint32_t a2 = lds_u32(prmt(vg, tsrc, s1));
            const uint32_t a1 = lds_u32(prmt(vh, tsrc, s0));
            const uint32_t a3 = lds_u32(prmt(vh, tsrc, s1));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (kk == 0) mma16816_z(cb[t][nt], a0, a1, a2, a3, xw[nt][0], xw[nt][1]);
              else mma16816(cb[t][nt], a0, a1, a2, a3, xw[nt][2 * kk], xw[nt][2 * kk + 1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[s]);
        // a^ = RN32(RN32(RN32(c / 127) * s_g) + mean), or the fp32 absmax
        const float a_mine = DQ ? __fadd_rn(__fmul_rn(S.inv127[qs + 128], fs), mu) : fs;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float ag = __shfl_sync(0xffffffffu, a_mine, g * 4 + t);
          const float ah = __shfl_sync(0xffffffffu, a_mine, g * 4 + 2 + t);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[t][nt][0] = fmaf(ag, cb[t][nt][0], acc[t][nt][0]);
            acc[t][nt][1] = fmaf(ag, cb[t][nt][1], acc[t][nt][1]);
            acc[t][nt][2] = fmaf(ah, cb[t][nt][2], acc[t][nt][2]);
            acc[t][nt][3] = fmaf(ah, cb[t][nt][3], acc[t][nt][3]);
          }
        }
      } else {
        // ---- 16 bf16 rows of A x one block: T[m, j] = sum_k X[m, k] A[j, k]
        uint32_t gw4[8], hw4[8];
        lds_row16(sb + j * 2048, 2 * g, c, gw4);   // rows past r were zero-filled
        lds_row16(sb + j * 2048, 2 * g + 1, c, hw4);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[s]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma16816(acc[0][nt], gw4[2 * kk], hw4[2 * kk], gw4[2 * kk + 1], hw4[2 * kk + 1],
                     xw[nt][2 * kk], xw[nt][2 * kk + 1]);
      }
    } else {
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);
    }
    rgp = nrgp;
    st = nst;
  }
  if (ok && cur >= 0) flush(cur);
}

// Y[m, n] = RNbf16( sum_pieces part[.][m][n] + sum_j RNbf16(s T[m, j]) B[n, j] )
// with T[m, j] = sum_pieces part[.][m][N + j] (pieces summed in order; every
// CTA reduces T into shared memory, CTA 0 also writes T_save = RNbf16(T)).
// The adapter product runs on mma.m16n8k16: a warp owns 16 output features
// (rows of B) and both 8-token tiles.  Launched as a programmatic dependent of
// the GEMV: the B fragments load before the wait for the GEMV's partials, and
// the partial loads are all issued before the first use.
__global__ void __launch_bounds__(256)
k_gemv_epilogue(const float* __restrict__ part, int64_t U, int P, int spr, int nat, int M, int N, int r,
                float s, const __nv_bfloat16* __restrict__ B, __nv_bfloat16* __restrict__ Y,
                __nv_bfloat16* __restrict__ T_save) {
  __shared__ __align__(16) uint32_t sT[kDecodeMaxTokens][64 + 4];   // bf16 pairs of s*T (r <= 128)
  __shared__ int s_np[8];                        // pieces of the adapter row groups (r <= 128)
  const int NE = N + r;
  const int64_t plane = (int64_t)M * NE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = (blockIdx.x * 8 + warp) * 16;
  const bool active = n0 < N;
  const int ng = min(n0 + g, N - 1), nh = min(n0 + g + 8, N - 1);
  // B fragments (independent of the GEMV): rows ng, nh; columns j0 + 2c (+8)
  uint32_t bf[8][4];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j0 = 16 * q;
    bf[q][0] = bf[q][1] = bf[q][2] = bf[q][3] = 0u;
    if (active && j0 < r) {
      bf[q][0] = __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)ng * r + j0 + 2 * c));
      bf[q][1] = __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)nh * r + j0 + 2 * c));
      if (j0 + 8 < r) {
        bf[q][2] = __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)ng * r + j0 + 8 + 2 * c));
        bf[q][3] = __ldg(reinterpret_cast<const uint32_t*>(B + (int64_t)nh * r + j0 + 8 + 2 * c));
      }
    }
  }
  if (threadIdx.x < nat) s_np[threadIdx.x] = n_pieces(threadIdx.x, spr, U, P);
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the GEMV's partials are complete
  // this lane's outputs: tokens nt*8 + 2c (+1), features n0+g (+8)
  const int np = active ? n_pieces(nat + n0 / kRows, spr, U, P) : 0;   // 16 features share a row group
  float v[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = nt * 8 + 2 * c + (i & 1);
      const int n = n0 + g + ((i & 2) ? 8 : 0);
      const bool ok = tok < M && n < N;
      const float* src = part + (int64_t)(ok ? tok : 0) * NE + (ok ? n : 0);
      float a = 0.f;
      for (int k = 0; k < np; ++k) a = __fadd_rn(a, ok ? __ldcg(src + k * plane) : 0.f);
      v[nt][i] = a;
    }
  __syncthreads();                               // s_np visible
  for (int e = threadIdx.x; e < kDecodeMaxTokens * 64; e += blockDim.x) {
    const int m = e / 64, jp = e % 64;            // token, pair of adapter columns
    float t0 = 0.f, t1 = 0.f;
    if (m < M && 2 * jp < r) {
      const int npt = s_np[(2 * jp) / kARows];    // columns 2jp and 2jp+1 share a row group
      const float* src = part + (int64_t)m * NE + N + 2 * jp;
      for (int k = 0; k < npt; ++k) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(src + k * plane));
        t0 = __fadd_rn(t0, x.x);
        t1 = __fadd_rn(t1, x.y);
      }
      if (T_save && blockIdx.x == 0)
        *reinterpret_cast<uint32_t*>(T_save + (int64_t)m * r + 2 * jp) = pack_bf16x2(t0, t1);
    }
    sT[m][jp] = pack_bf16x2(__fmul_rn(s, t0), __fmul_rn(s, t1));
  }
  __syncthreads();
  if (!active) return;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (16 * q >= r) break;
    // A = B rows (row-major, j contiguous); B operand = s*T, column j, token
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const uint32_t b0 = sT[nt * 8 + g][8 * q + c];
      const uint32_t b1 = sT[nt * 8 + g][8 * q + 4 + c];
      mma16816(acc[nt], bf[q][0], bf[q][1], bf[q][2], bf[q][3], b0, b1);
    }
  }
  // fragment: acc[nt][0..1] = feature n0+g, tokens nt*8 + 2c, +1; [2..3] = feature n0+g+8
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = nt * 8 + 2 * c + (i & 1);
      const int n = n0 + g + ((i & 2) ? 8 : 0);
      if (tok < M && n < N) Y[(int64_t)tok * N + n] = __float2bfloat16_rn(v[nt][i] + acc[nt][i]);
    }
}

struct Plan {
  int nb, spr, nat, nrg;
  int64_t U;
  int P;
  int max_pieces;
};

Plan plan(int N, int K, int r) {
  Plan pl;
  pl.nb = K / 64;
  pl.spr = (pl.nb + kBlk - 1) / kBlk;
  pl.nat = (r + kARows - 1) / kARows;
  pl.nrg = (N + kRows - 1) / kRows;
  pl.U = (int64_t)(pl.nat + pl.nrg) * pl.spr;
  pl.P = (int)std::min<int64_t>(kMaxParts, pl.U);
  pl.max_pieces = 1;
  for (int rgp = 0; rgp < pl.nat + pl.nrg; ++rgp)
    pl.max_pieces = std::max(pl.max_pieces, n_pieces(rgp, pl.spr, pl.U, pl.P));
  return pl;
}

// Dynamic shared memory for the map above when it starts at shared address
// `base` (the block's reserved shared memory; the kernel has no static
// shared memory).
template <int NT>
constexpr int gemv_smem_bytes(uint32_t base) {
  return (int)(kRingAddr - base) + n_stages_high<NT>() * stage_bytes<NT>();
}
static_assert(low_stage_off<1>() + stage_bytes<1>() + 1024 <= kTableAddr, "low stage below the table");
static_assert(sizeof(GemvSmem<2>) + 1024 <= kTableAddr, "state below the table");
static_assert(gemv_smem_bytes<1>(0) <= 232448 && gemv_smem_bytes<2>(0) <= 232448, "shared memory per CTA");

template <bool DQ, int NT>
void launch_gemv_kernel(const CUtensorMap& tw, const CUtensorMap& ta, const CUtensorMap& tx,
                        const GemvArgs& a, cudaStream_t st) {
  const int smem = gemv_smem_bytes<NT>(a.smem_base);
  static std::atomic<unsigned long long> attr_devs{0};
  set_smem_attr_once(k_qlora_gemv<DQ, NT>, smem, attr_devs);
  k_qlora_gemv<DQ, NT><<<a.P, kThreads, smem, st>>>(tw, ta, tx, a);
}

}  // namespace

size_t gemv_workspace_bytes(int M, int N, int K, int r) {
  return (size_t)plan(N, K, r).max_pieces * M * (N + r) * 4;
}

int launch_qlora_gemv(const nf4_weight* w, const void* X, int M, const void* A, const void* B,
                      int r, float s, void* Y, void* T_save, float* part, const float* q,
                      int* status, cudaStream_t st, int num_sms) {
  (void)num_sms;   // the partition is fixed; extra SMs idle, fewer run it in waves
  GemvArgs a{};
  a.status = status;
  a.absmax = w->absmax; a.qabsmax = w->qabsmax;
  a.dq_type = w->double_quant;
  a.dq_scale = w->dq_scale; a.dq_mean = w->dq_mean;
  a.part = part;
  a.M = M; a.N = (int)w->rows; a.K = (int)w->cols; a.r = r;
  const Plan pl = plan(a.N, a.K, r);
  a.nb = pl.nb; a.spr = pl.spr; a.nat = pl.nat; a.nrg = pl.nrg; a.U = pl.U; a.P = pl.P;
  {
    // dynamic shared memory starts after the block's reserved shared memory
    int dev = 0, reserved = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
      cudaGetLastError();
      return -1;
    }
    a.smem_base = (uint32_t)reserved;
  }
  for (int i = 0; i < 16; ++i) a.q[i] = q[i];
  const int NT = M <= 8 ? 1 : 2;
  CUtensorMap tw, ta, tx;
  // A and X viewed as [K/64 blocks][rows][64]: one box brings a stage's 8 blocks
  const uint64_t ad[3] = {64, (uint64_t)r, (uint64_t)pl.nb}, xd[3] = {64, (uint64_t)M, (uint64_t)pl.nb};
  const uint64_t rs[2] = {(uint64_t)a.K * 2, 128};
  const uint32_t abox[3] = {64, kARows, kBlk}, xbox[3] = {64, (uint32_t)(8 * NT), kBlk};
  if (!make_tmap_2d_u8(&tw, w->packed, (uint64_t)a.K / 2, (uint64_t)a.N, (uint64_t)a.K / 2, 128, kRows, true) ||
      !make_tmap_3d(&ta, A, true, ad, rs, abox, true) ||
      !make_tmap_3d(&tx, X, true, xd, rs, xbox, true))
    return -1;
  if (w->double_quant) {
    if (NT == 1) launch_gemv_kernel<true, 1>(tw, ta, tx, a, st);
    else launch_gemv_kernel<true, 2>(tw, ta, tx, a, st);
  } else {
    if (NT == 1) launch_gemv_kernel<false, 1>(tw, ta, tx, a, st);
    else launch_gemv_kernel<false, 2>(tw, ta, tx, a, st);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::max(1, (a.N + 127) / 128), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, k_gemv_epilogue, (const float*)part, pl.U, pl.P, pl.spr, pl.nat, M, a.N, r, s,
                     (const __nv_bfloat16*)B, (__nv_bfloat16*)Y, (__nv_bfloat16*)T_save);
  return 2;
}

}  // namespace qnf4
