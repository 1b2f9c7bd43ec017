// Tensor-core GEMM engine of the QLoRA layer (tcgen05 / TMEM / TMA, sm_100a).
//
//   out[m, o] = sum_c tok[m, c] * Wt[o, c]  +  sum_j tokad[m, j] * Wad[o, j]
//
// computed transposed (out^T = Wt tok^T) so that the weight side is the MMA's
// A operand (128 rows per tile) and the token side its B operand (256 tokens
// per tile).  Two modes:
//
//  MODE_NF4 (forward, Y = X deq(W)^T + (s T) B^T).  Page "QLoRA Explained",
//    section "Why the expansion cannot be skipped": the tensor core cannot
//    decode a 4-bit row index, so a kernel reads the codes, looks them up in
//    the 16-entry table, multiplies by the block scale and hands bf16 to the
//    tensor core.  Here converter warps do that for one weight row per thread
//    and one NF4 block per K step (64 = the block size): a 16-entry bf16 table
//    per block is built in registers as two byte planes, codes are expanded
//    with prmt, and the bf16 row goes straight into a tensor-memory ring with
//    tcgen05.st -- tcgen05.mma reads A from TMEM, so the dequantised weights
//    never touch shared memory.
//
//  MODE_BF16 (backward dX = dY deq(W) + (s U) A).  Both operands arrive by
//    TMA; the weight side is deq(W)^T prepared by a dequantise-transpose pass.
//
// The adapter term (page "LoRA vs QLoRA", section "How LoRA Works": W' = W +
// (alpha/r) B A) is ceil(r/64) extra K steps of an SS MMA into the same TMEM
// accumulator, with the rank padded to 64 by zeros.
//
// Persistent: one CTA per SM walks a static tile schedule.  Warp 0 issues
// TMA, warp 1 issues MMA, warps 2-5 drain the accumulator (one per TMEM lane
// quadrant, in two halves of 128 columns; the accumulator is released once the
// second half sits in registers, so the next tile's MMAs overlap the stores),
// warps 6-13 convert NF4 (MODE_NF4): two warps per quadrant take alternate K
// steps, so one warp's TMEM-store wait and barrier hand-off overlap the other's
// table expansion.  Every wait is bounded (status QLORA_ERR_TIMEOUT).

#include <algorithm>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.h"
#include "nf4_lut.cuh"

namespace qnf4 {

namespace eng {

constexpr int BN = 128;          // weight-side rows per tile (MMA M)
constexpr int BM = 256;          // tokens per tile (MMA N)
constexpr int BK = 64;           // contraction per stage (= one NF4 block)
constexpr int X_BYTES = BM * BK * 2;            // 32 KB token tile
constexpr int W_BYTES = BN * BK * 2;            // 16 KB weight tile
constexpr int ACC_COL = 0;                      // accumulator: TMEM columns [0, 256)
constexpr int A_COL = 256;                      // NF4 A ring: stages x 32 columns
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 448;                // 14 warps
constexpr int CVT_WARP0 = 6;                    // warps 6-13: converters

// Pipeline depth.  MODE_NF4 keeps only token tiles in shared memory (the
// weight side lives in TMEM), so it affords 6 stages of 32 KB; MODE_BF16 holds
// a 16 KB weight tile beside each token tile and keeps 4.
template <int MODE> __host__ __device__ constexpr int stages() { return MODE == MODE_NF4 ? 6 : 4; }

template <int MODE>
struct Smem {
  static constexpr int NS = stages<MODE>();
  uint8_t x[NS][X_BYTES];
  uint8_t w[MODE == MODE_NF4 ? 1 : NS][MODE == MODE_NF4 ? 16 : W_BYTES];
  uint64_t x_full[NS], x_empty[NS];
  uint64_t a_full[NS], a_empty[NS];
  uint64_t acc_full, acc_empty, done;
  uint32_t tmem_base;
  int abort;
  float inv127[256];
};

template <int MODE>
constexpr size_t smem_bytes() { return sizeof(Smem<MODE>) + 1024; }

template <int MODE, bool DQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_qlora_gemm(const __grid_constant__ CUtensorMap tm_tok,     // [Mtok, Kc]  bf16
             const __grid_constant__ CUtensorMap tm_tokad,   // [Mtok, RP]  bf16
             const __grid_constant__ CUtensorMap tm_wad,     // [Nout, RP]  bf16
             const __grid_constant__ CUtensorMap tm_w,       // [Nout, Kc]  bf16 (MODE_BF16)
             const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<MODE>& S =
      *reinterpret_cast<Smem<MODE>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_tiles_n = (p.Nout + BN - 1) / BN;
  const int n_tiles = n_tiles_n * ((p.Mtok + BM - 1) / BM);
  const int nk = (p.Kc + BK - 1) / BK;
  const int na = p.na;

  constexpr int NS = stages<MODE>();
  const int nsteps = nk + na;                      // ring steps per tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&S.x_full[i], 1);
      mbar_init(&S.x_empty[i], 1);
      mbar_init(&S.a_full[i], 128);
      mbar_init(&S.a_empty[i], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, 128);
    mbar_init(&S.done, 1);
    S.abort = 0;
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    S.inv127[i] = dq_code_value(i, p.double_quant);     // entry c + 128: any code byte
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_tok);
    tma_prefetch_desc(&tm_tokad);
    if (MODE == MODE_BF16) {
      tma_prefetch_desc(&tm_wad);
      tma_prefetch_desc(&tm_w);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Step ks < nk: token tile of contraction block ks (and, MODE_BF16, the
    // weight tile); ks >= nk: adapter step j = ks - nk (s*T or s*U tile, and,
    // MODE_BF16, the adapter weight tile).
    if (lane == 0) {
      uint32_t xi = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int n0 = (tile % n_tiles_n) * BN;
        const int m0 = (tile / n_tiles_n) * BM;
        for (int ks = 0; ks < nsteps; ++ks, ++xi) {
          const int s = xi % NS;
          if (!(ok = mbar_wait(&S.x_empty[s], ((xi / NS) & 1) ^ 1, abort, p.status))) break;
          const bool ad = ks >= nk;
          const int kc = (ad ? ks - nk : ks) * BK;
          if (MODE == MODE_BF16) {
            mbar_arrive_expect_tx(&S.x_full[s], X_BYTES + W_BYTES);
            tma_load_2d(S.x[s], ad ? &tm_tokad : &tm_tok, &S.x_full[s], kc, m0);
            tma_load_2d(S.w[s], ad ? &tm_wad : &tm_w, &S.x_full[s], kc, n0);
          } else {
            mbar_arrive_expect_tx(&S.x_full[s], X_BYTES);
            tma_load_2d(S.x[s], ad ? &tm_tokad : &tm_tok, &S.x_full[s], kc, m0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BN, BM);
      uint32_t xi = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
        ok = mbar_wait(&S.acc_empty, (lt & 1) ^ 1, abort, p.status);
        if (!ok) break;
        tc_fence_after();
        for (int ks = 0; ks < nsteps && ok; ++ks, ++xi) {
          const int s = xi % NS;
          const uint32_t par = (xi / NS) & 1;
          ok = mbar_wait(&S.x_full[s], par, abort, p.status);
          if (ok && MODE == MODE_NF4) ok = mbar_wait(&S.a_full[s], par, abort, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(S.x[s]));
          if (MODE == MODE_NF4) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_ts(tmem + ACC_COL, tmem + A_COL + s * 32 + kk * 8, bdesc + (uint64_t)(kk * 2),
                     idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&S.x_empty[s]);
            mma_commit(&S.a_empty[s]);
          } else {
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(S.w[s]));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_ss(tmem + ACC_COL, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc,
                     (ks > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&S.x_empty[s]);
          }
        }
        if (ok) mma_commit(&S.acc_full);
      }
      // all MMAs issued by this thread are complete once `done` flips
      mma_commit(&S.done);
      mbar_wait(&S.done, 0, abort, p.status);
    }
  } else if (warp >= CVT_WARP0) {
    // ------------------------------------------------------------ A-operand producers (TMEM)
    // MODE_NF4 only.  Step ks < nk: NF4 -> bf16 for block ks of the thread's
    // weight row; step ks >= nk: copy 64 bf16 of the row's adapter factor
    // B[n, j*64 .. j*64+63] (zero-padded to RP columns).
    if (MODE == MODE_NF4) {
      const int quad = warp & 3;
      const uint32_t par = (uint32_t)((warp - CVT_WARP0) >> 2);   // steps of this parity
      const int row_in_tile = quad * 32 + lane;
      const uint32_t tmem_lane = (uint32_t)(quad * 32) << 16;
      const float mu = DQ ? __ldg(p.dq_mean) : 0.0f;
      const int64_t kb_per_row = p.Kc / 64;
      // ring step ai is step (ai % nsteps) of this CTA's tile (ai / nsteps)
      struct Src { uint4 c[8]; float a_raw, sg; int qa; bool valid, ad; };
      auto fetch = [&](uint32_t ai, Src& d) -> bool {
        const uint32_t lt = ai / (uint32_t)nsteps;
        const int ks = (int)(ai - lt * (uint32_t)nsteps);
        const int tile = blockIdx.x + (int)lt * gridDim.x;
        if (tile >= n_tiles) return false;
        const int n = (tile % n_tiles_n) * BN + row_in_tile;
        d.valid = n < p.Nout;
        d.ad = ks >= nk;
        const int64_t nn = d.valid ? n : 0;
        if (d.ad) {
          const uint4* src = reinterpret_cast<const uint4*>(p.wad + nn * p.RP + (ks - nk) * BK);
#pragma unroll
          for (int i = 0; i < 8; ++i) d.c[i] = __ldcg(src + i);
        } else {
          const uint4* codes = reinterpret_cast<const uint4*>(p.packed + nn * (p.Kc / 2)) + 2 * ks;
          d.c[0] = __ldcg(codes);
          d.c[1] = __ldcg(codes + 1);
          const int64_t b = nn * kb_per_row + ks;
          if (DQ) { d.qa = __ldcg(p.qabsmax + b); d.sg = __ldg(p.dq_scale + (b >> 8)); d.a_raw = 0.f; }
          else { d.a_raw = __ldcg(p.absmax + b); d.qa = 0; d.sg = 0.f; }
        }
        return true;
      };
      Src cur, nxt;
      uint32_t ai = par;
      bool have = fetch(ai, cur);
      while (have) {
        const bool more = fetch(ai + 2, nxt);     // prefetch this warp's next step
        uint32_t v[32];
        if (!cur.valid) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        } else if (cur.ad) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[4 * i] = cur.c[i].x; v[4 * i + 1] = cur.c[i].y;
            v[4 * i + 2] = cur.c[i].z; v[4 * i + 3] = cur.c[i].w;
          }
        } else {
          // a^ = RN32(RN32(RN32(c / 127) * s_g) + mean), or the fp32 absmax
          const float a = DQ ? __fadd_rn(__fmul_rn(S.inv127[cur.qa + 128], cur.sg), mu) : cur.a_raw;
          const Lut l = build_lut(a, p.q);
          const uint32_t wds[8] = {cur.c[0].x, cur.c[0].y, cur.c[0].z, cur.c[0].w,
                                   cur.c[1].x, cur.c[1].y, cur.c[1].z, cur.c[1].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) lookup8(wds[i], l, v + 4 * i);
        }
        const int sa = ai % NS;
        if (!mbar_wait(&S.a_empty[sa], ((ai / NS) & 1) ^ 1, abort, p.status)) break;
        __syncwarp();
        tc_fence_after();
        const uint32_t taddr = tmem + tmem_lane + A_COL + sa * 32;
        tmem_st16(taddr, v);
        tmem_st16(taddr + 16, v + 16);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&S.a_full[sa]);
        cur = nxt;
        have = more;
        ai += 2;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    constexpr int HALF = BM / 2;                 // columns drained per round
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t tmem_lane = (uint32_t)(quad * 32) << 16;
    const bool odd = lane & 1;
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++lt) {
      const int n0 = (tile % n_tiles_n) * BN;
      const int mt = (tile / n_tiles_n) * BM;
      if (!mbar_wait(&S.acc_full, lt & 1, abort, p.status)) break;
      __syncwarp();
      tc_fence_after();
      // lane pairs (o, o+1) swap halves so each lane stores two adjacent
      // outputs of one token row: even lanes row m, odd lanes row m+1
      const int ocol = n0 + row_in_tile - (odd ? 1 : 0);
      const int step = p.Nout;                   // two bf16 rows = Nout words
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t packed[HALF / 2];
#pragma unroll
        for (int c = 0; c < HALF; c += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + tmem_lane + ACC_COL + h * HALF + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            packed[c / 2 + j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
        }
        if (h == 1) {
          tc_fence_before();
          mbar_arrive(&S.acc_empty);
        }
        const int mfirst = mt + h * HALF + (odd ? 1 : 0);
        const int rows_left = (ocol < p.Nout) ? p.Mtok - mfirst : 0;
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (int64_t)mfirst * p.Nout + ocol);
#pragma unroll
        for (int c = 0; c < HALF; c += 2) {
          const uint32_t mine = packed[c / 2];
          const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
          const uint32_t out = odd ? prmt(other, mine, 0x7632) : prmt(mine, other, 0x5410);
          if (c < rows_left) *dst = out;
          dst += step;
        }
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

template <int MODE, bool DQ>
static void launch_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                       const CUtensorMap& d, const GemmArgs& p, int grid, cudaStream_t s) {
  static std::atomic<unsigned long long> attr_devs{0};
  set_smem_attr_once(k_qlora_gemm<MODE, DQ>, (int)smem_bytes<MODE>(), attr_devs);
  k_qlora_gemm<MODE, DQ><<<grid, NUM_THREADS, smem_bytes<MODE>(), s>>>(a, b, c, d, p);
}

}  // namespace eng

int launch_qlora_gemm(int mode, const GemmArgs& a, const void* tok, const void* tokad,
                      const void* wad, const void* w, int RP, cudaStream_t s, int num_sms) {
  using namespace eng;
  CUtensorMap t_tok, t_tokad, t_wad, t_w;
  if (!make_tmap_2d_bf16(&t_tok, tok, a.Kc, a.Mtok, a.Kc, BK, BM)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&t_tokad, tokad, RP, a.Mtok, RP, BK, BM)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&t_wad, wad, RP, a.Nout, RP, BK, BN)) return QLORA_ERR_CUDA;
  if (mode == MODE_BF16) {
    if (!make_tmap_2d_bf16(&t_w, w, a.Kc, a.Nout, a.Kc, BK, BN)) return QLORA_ERR_CUDA;
  } else {
    t_w = t_wad;                                  // unused
  }
  const int n_tiles = ((a.Nout + BN - 1) / BN) * ((a.Mtok + BM - 1) / BM);
  const int grid = std::min(n_tiles, num_sms);
  if (mode == MODE_BF16)
    launch_one<MODE_BF16, false>(t_tok, t_tokad, t_wad, t_w, a, grid, s);
  else if (a.double_quant)
    launch_one<MODE_NF4, true>(t_tok, t_tokad, t_wad, t_w, a, grid, s);
  else
    launch_one<MODE_NF4, false>(t_tok, t_tokad, t_wad, t_w, a, grid, s);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qnf4
