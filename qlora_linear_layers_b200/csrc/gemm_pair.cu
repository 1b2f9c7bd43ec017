// Backward dX GEMM on paired SMs (tcgen05 cta_group::2):
//
//   dX = dY deq(W) + (s U) A     (weights supplied as deq(W)^T, bf16)
//
// Page "QLoRA Explained", config walk-through: the input gradient flows
// through the frozen 4-bit base (dequantised, never updated) and the adapter.
// Two SMs of a cluster share each 256 x BM output tile:
//  * MMA M = 256 (CTA r owns weight rows 128r..128r+127 of the tile), MMA N =
//    BM (CTA r loads tokens BM/2 r..BM/2 r + BM/2 - 1).  Each SM streams half
//    the token tile per K step, halving the shared-memory port traffic (TMA
//    writes + MMA reads of the token operand).
//  * Both operands arrive by TMA (each CTA its 128 weight rows and its BM/2
//    tokens), 6 stages of 16 + 16 KB; the adapter term runs as RP/64 extra K
//    steps over [s U | A^T].
//  * The even CTA's elected thread issues tcgen05.mma.cta_group::2 with both
//    operands in shared memory and commits with an arrival multicast to both
//    CTAs' "empty" and "full" barriers.  Both CTAs' TMA loads (no multicast:
//    each CTA loads its own half) complete on the even CTA's "full" barrier;
//    the odd CTA's epilogue warps arrive on the even CTA's barriers through
//    mapa.
// Every wait is bounded (status QLORA_ERR_TIMEOUT); both CTAs meet at a
// cluster barrier before the paired TMEM is released.

#include <algorithm>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.h"

namespace qnf4 {

namespace pair {

constexpr int BN = 128;          // weight rows per CTA (MMA M = 256 per pair)
constexpr int BK = 64;           // contraction per stage
constexpr int NS = 6;            // pipeline stages
// BM (template argument, a multiple of 32 up to 256): tokens per pair tile =
// MMA N; each CTA loads BM / 2 tokens, BM * 64 bytes per stage.
constexpr int ACC_COL = 0;                       // accumulator: TMEM columns [0, 256)
constexpr int TMEM_COLS = 256;
constexpr int NUM_THREADS = 192;                 // warp 0 TMA, 1 MMA, 2-5 epilogue
constexpr uint16_t kBoth = 0x3;                  // cluster CTA mask of the pair

constexpr int W_BYTES = BN * BK * 2;             // 16 KB weight tile per CTA and stage

template <int BM>
struct Smem {
  uint8_t x[NS][BM * BK];
  uint8_t w[NS][W_BYTES];
  uint64_t x_full[NS], x_empty[NS];
  uint64_t acc_full, acc_empty, done;
  uint32_t tmem_base;
  int abort;
};

template <int BM>
constexpr size_t smem_bytes() { return sizeof(Smem<BM>) + 1024; }

template <int BM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_qlora_gemm_pair(const __grid_constant__ CUtensorMap tm_tok,     // [Mtok, Kc]  bf16
                  const __grid_constant__ CUtensorMap tm_tokad,   // [Mtok, RP]  bf16
                  const __grid_constant__ CUtensorMap tm_w,       // [Nout, Kc]  bf16
                  const __grid_constant__ CUtensorMap tm_wad,     // [Nout, RP]  bf16
                  const GemmArgs p) {
  static_assert(BM % 32 == 0 && BM >= 32 && BM <= 256, "token tile");
  constexpr int BMH = BM / 2;                      // tokens loaded by each CTA
  constexpr int X_BYTES = BMH * BK * 2;
  extern __shared__ uint8_t smem_raw[];
  Smem<BM>& S =
      *reinterpret_cast<Smem<BM>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();        // 0: issues the MMAs
  const bool leader = rank == 0;

  const int n_pairs_n = (p.Nout + 2 * BN - 1) / (2 * BN);
  const int n_tiles = n_pairs_n * ((p.Mtok + BM - 1) / BM);
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const int nk = (p.Kc + BK - 1) / BK;
  const int nsteps = nk + p.na;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&S.x_full[i], 1);                  // leader's expect_tx; tx from both CTAs
      mbar_init(&S.x_empty[i], 1);                 // multicast commit
    }
    mbar_init(&S.acc_full, 1);                     // multicast commit
    mbar_init(&S.acc_empty, 8);                    // 4 epilogue warps per CTA
    mbar_init(&S.done, 1);
    S.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_tok);
    tma_prefetch_desc(&tm_tokad);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_wad);
  }
  tc_fence_before();
  cluster_sync();                                  // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t xi = 0;
      bool ok = true;
      for (int tile = cluster; tile < n_tiles && ok; tile += n_clusters) {
        const int m0 = (tile / n_pairs_n) * BM + (int)rank * BMH;
        const int n0 = (tile % n_pairs_n) * (2 * BN) + (int)rank * BN;
        for (int ks = 0; ks < nsteps; ++ks, ++xi) {
          const int s = xi % NS;
          if (!(ok = mbar_wait_cluster(&S.x_empty[s], ((xi / NS) & 1) ^ 1, abort, p.status))) break;
          if (leader) mbar_arrive_expect_tx(&S.x_full[s], 2 * (X_BYTES + W_BYTES));
          const bool ad = ks >= nk;
          const int kc = (ad ? ks - nk : ks) * BK;
          const uint32_t full0 = mapa_shared(smem_u32(&S.x_full[s]), 0);
          tma_load_2d_pair(S.x[s], ad ? &tm_tokad : &tm_tok, full0, kc, m0);
          tma_load_2d_pair(S.w[s], ad ? &tm_wad : &tm_w, full0, kc, n0);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_bf16_f32(2 * BN, BM);
      uint32_t xi = 0, lt = 0;
      bool ok = true;
      for (int tile = cluster; tile < n_tiles && ok; tile += n_clusters, ++lt) {
        ok = mbar_wait_cluster(&S.acc_empty, (lt & 1) ^ 1, abort, p.status);
        if (!ok) break;
        tc_fence_after();
        for (int ks = 0; ks < nsteps && ok; ++ks, ++xi) {
          const int s = xi % NS;
          const uint32_t par = (xi / NS) & 1;
          ok = mbar_wait_cluster(&S.x_full[s], par, abort, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(S.x[s]));
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(S.w[s]));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss_pair(tmem + ACC_COL, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2),
                        idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit_pair_mc(&S.x_empty[s], kBoth);
        }
        if (ok) mma_commit_pair_mc(&S.acc_full, kBoth);
      }
      // all MMAs issued by this thread are complete once `done` flips
      mma_commit_pair_mc(&S.done, 0x1);
      mbar_wait(&S.done, 0, abort, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5, both CTAs)
    constexpr int HALF = BM / 2;                 // columns drained per round
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t tmem_lane = (uint32_t)(quad * 32) << 16;
    const bool odd = lane & 1;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(&S.acc_empty), 0);
    uint32_t lt = 0;
    for (int tile = cluster; tile < n_tiles; tile += n_clusters, ++lt) {
      const int n0 = (tile % n_pairs_n) * (2 * BN) + (int)rank * BN;
      const int mt = (tile / n_pairs_n) * BM;
      if (!mbar_wait_cluster(&S.acc_full, lt & 1, abort, p.status)) break;
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
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty0);
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
  cluster_sync();                                  // both CTAs done with the paired TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

template <int BM>
static cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2,
                               const CUtensorMap& a3, const GemmArgs& a, int clusters, cudaStream_t s) {
  static std::atomic<unsigned long long> attr_devs{0};
  set_smem_attr_once(k_qlora_gemm_pair<BM>, (int)smem_bytes<BM>(), attr_devs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<BM>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_qlora_gemm_pair<BM>, a0, a1, a2, a3, a);
}

}  // namespace pair

// Token-tile width of the paired GEMM for an [Mtok x Nout] output on
// `clusters_max` SM pairs.  A pair tile costs (fixed + width) per K step --
// the fixed part, the weight-tile TMA, is about 480 width units as timed on
// B200 -- and a launch lasts as many rounds as the busiest pair runs tiles.
// The narrower width pays only where it removes a round.
static int pair_token_tile(int64_t Mtok, int64_t Nout, int clusters_max) {
  static const int kWidths[] = {256, 224};
  const int64_t fixed = 480;
  const int64_t n_pairs_n = (Nout + 255) / 256;
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int bm : kWidths) {
    const int64_t tiles = n_pairs_n * ((Mtok + bm - 1) / bm);
    const int64_t clusters = std::max<int64_t>(1, std::min<int64_t>(tiles, clusters_max));
    const int64_t rounds = (tiles + clusters - 1) / clusters;
    const int64_t cost = rounds * (bm + fixed);
    if (cost < best_cost) { best_cost = cost; best = bm; }
  }
  return best;
}

// Paired-SM dX GEMM: w [Nout, Kc] and wad [Nout, RP] bf16 by TMA.  Returns
// QLORA_OK or QLORA_ERR_CUDA.
int launch_qlora_gemm_pair(const GemmArgs& a, const void* tok, const void* tokad, const void* wad,
                           const void* w, int RP, cudaStream_t s, int num_sms) {
  using namespace pair;
  const int bm = pair_token_tile(a.Mtok, a.Nout, num_sms / 2);
  CUtensorMap t_tok, t_tokad, t_w, t_wad;
  if (!make_tmap_2d_bf16(&t_tok, tok, a.Kc, a.Mtok, a.Kc, BK, bm / 2)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&t_tokad, tokad, RP, a.Mtok, RP, BK, bm / 2)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&t_w, w, a.Kc, a.Nout, a.Kc, BK, BN)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&t_wad, wad, RP, a.Nout, RP, BK, BN)) return QLORA_ERR_CUDA;
  const int n_tiles = ((a.Nout + 2 * BN - 1) / (2 * BN)) * ((a.Mtok + bm - 1) / bm);
  const int clusters = std::max(1, std::min(n_tiles, num_sms / 2));
  cudaError_t e;
  if (bm == 224) e = launch_pair<224>(t_tok, t_tokad, t_w, t_wad, a, clusters, s);
  else e = launch_pair<256>(t_tok, t_tokad, t_w, t_wad, a, clusters, s);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qnf4
