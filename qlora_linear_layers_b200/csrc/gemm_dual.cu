// Fused NF4-dequant forward GEMM on paired SMs, two token tiles per weight
// tile (tcgen05 cta_group::2, both operands in shared memory).
//
//   Y = X deq(W)^T + (s T) B^T       (computed as Y^T = deq(W) X^T)
//
// Page "QLoRA Explained", section "Why the expansion cannot be skipped": the
// tensor core cannot decode a 4-bit row index, so the kernel reads the codes,
// looks them up in the 16-entry table, multiplies by the block scale and
// hands bf16 to the tensor core.  The expansion is the cost this kernel is
// built around: converter warps expand a 256-row x 64-column weight stage
// once (each CTA of the pair its own 128 rows, into its own shared memory, in
// the 128-byte-swizzled K-major layout a TMA load would write) and the MMA
// issuer runs that stage against TWO token tiles of up to 256 tokens each,
// into two TMEM accumulators (columns [0, BM) and [256, 256 + BM)).  Per
// FLOP, half the conversion work of a one-accumulator tile.
//
//  * Warp 0 (both CTAs): TMA of the tokens, each CTA its BM/2 tokens of each
//    token tile per stage; completion counted on the even CTA's barrier.
//  * Warp 1 (even CTA): tcgen05.mma.cta_group::2, 2 x 4 per stage, commit
//    with a multicast arrival to both CTAs' stage barriers.
//  * Warps 2-5 (both CTAs): drain both accumulators (TMEM -> registers ->
//    bf16 -> global), releasing them once the last columns are in registers.
//  * Warps 6-13 (both CTAs): converters, one weight row per thread, two warps
//    per 32 rows taking alternate stages; each builds its block's 16-entry
//    bf16 table in registers (RNbf16(RN32(q[i] * a^)), the exact values of
//    nf4_dequantize), expands 8 codes per 21 integer ops and stores the row's
//    eight 16-byte chunks at their swizzled positions; a proxy fence makes the
//    stores visible to the tensor core before the stage is signalled.
//  * The adapter term s T B^T runs as ceil(r/64) extra stages: the converters
//    copy rows of B (zero-padded to 64 columns), the tokens are s T.
// Every wait is bounded (status QLORA_ERR_TIMEOUT); both CTAs meet at a
// cluster barrier before the paired TMEM is released.

#include <algorithm>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.h"
#include "nf4_lut.cuh"

namespace qnf4 {

namespace dual {

constexpr int BN = 128;                    // weight rows per CTA (MMA M = 256 per pair)
constexpr int BK = 64;                     // contraction per stage (= one NF4 block)
constexpr int NS = 4;                      // pipeline stages
constexpr int XH_MAX = 128 * 128;          // one token tile's half per stage: <= 128 rows x 128 B
constexpr int A_BYTES = BN * 128;          // converted weights per stage: 128 rows x 128 B
constexpr int ACC1_COL = 256;              // second accumulator: TMEM columns [256, 256 + BM)
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 448;           // 14 warps
constexpr int CVT_WARP0 = 6;
constexpr uint16_t kBoth = 0x3;

struct Smem {
  uint8_t x[NS][2][XH_MAX];                // tokens of token tiles 0 and 1
  uint8_t a[NS][A_BYTES];                  // converted weight rows
  uint64_t x_full[NS], x_empty[NS];
  uint64_t a_full[NS], a_empty[NS];
  uint64_t acc_full, acc_empty, done;
  uint32_t tmem_base;
  int abort;
  float inv127[256];
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }

// L2 policy for the weight codes: keep them (a launch re-reads each code once
// per round of token tiles, while the token stream passes through L2).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ldg_hint(const uint4* ptr, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(ptr), "l"(pol));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor core's operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <bool DQ>
__global__ void __launch_bounds__(NUM_THREADS, 1)
k_qlora_gemm_dual(const __grid_constant__ CUtensorMap tm_tok,     // [Mtok, Kc] bf16, box 64 x BM/2
                  const __grid_constant__ CUtensorMap tm_tokad,   // [Mtok, RP] bf16, box 64 x BM/2
                  const GemmArgs p, const int BM) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();        // 0: issues the MMAs
  const bool leader = rank == 0;
  const int BMH = BM >> 1;                         // tokens of a token tile loaded by each CTA
  const uint32_t xh_bytes = (uint32_t)BMH * 128u;

  const int n_pairs_n = (p.Nout + 2 * BN - 1) / (2 * BN);
  const int n_tiles = n_pairs_n * ((p.Mtok + 2 * BM - 1) / (2 * BM));
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const int nk = (p.Kc + BK - 1) / BK;
  const int nsteps = nk + p.na;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&S.x_full[i], 1);                  // leader's expect_tx; tx from both CTAs
      mbar_init(&S.x_empty[i], 1);                 // multicast commit
      mbar_init(&S.a_full[i], 8);                  // 4 converter warps per CTA
      mbar_init(&S.a_empty[i], 1);                 // multicast commit
    }
    mbar_init(&S.acc_full, 1);                     // multicast commit
    mbar_init(&S.acc_empty, 8);                    // 4 epilogue warps per CTA
    mbar_init(&S.done, 1);
    S.abort = 0;
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    S.inv127[i] = dq_code_value(i, p.double_quant);     // entry c + 128: any code byte
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_tok);
    tma_prefetch_desc(&tm_tokad);
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
        const int m0 = (tile / n_pairs_n) * (2 * BM) + (int)rank * BMH;
        for (int ks = 0; ks < nsteps; ++ks, ++xi) {
          const int s = xi % NS;
          if (!(ok = mbar_wait_cluster(&S.x_empty[s], ((xi / NS) & 1) ^ 1, abort, p.status))) break;
          if (leader) mbar_arrive_expect_tx(&S.x_full[s], 4u * xh_bytes);
          const bool ad = ks >= nk;
          const int kc = (ad ? ks - nk : ks) * BK;
          const uint32_t full0 = mapa_shared(smem_u32(&S.x_full[s]), 0);
          const CUtensorMap* tm = ad ? &tm_tokad : &tm_tok;
          tma_load_2d_pair(S.x[s][0], tm, full0, kc, m0);
          tma_load_2d_pair(S.x[s][1], tm, full0, kc, m0 + BM);
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
          if (ok) ok = mbar_wait_cluster(&S.a_full[s], par, abort, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(S.a[s]));
          const uint64_t b0 = sw128_kmajor_desc(smem_u32(S.x[s][0]));
          const uint64_t b1 = sw128_kmajor_desc(smem_u32(S.x[s][1]));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            mma_ss_pair(tmem, adesc + (uint64_t)(kk * 2), b0 + (uint64_t)(kk * 2), idesc, acc);
            mma_ss_pair(tmem + ACC1_COL, adesc + (uint64_t)(kk * 2), b1 + (uint64_t)(kk * 2), idesc, acc);
          }
          mma_commit_pair_mc(&S.x_empty[s], kBoth);
          mma_commit_pair_mc(&S.a_empty[s], kBoth);
        }
        if (ok) mma_commit_pair_mc(&S.acc_full, kBoth);
      }
      // all MMAs issued by this thread are complete once `done` flips
      mma_commit_pair_mc(&S.done, 0x1);
      mbar_wait(&S.done, 0, abort, p.status);
    }
  } else if (warp >= CVT_WARP0) {
    // ------------------------------------------------------------ converters (shared memory)
    // Step ks < nk: NF4 -> bf16 for block ks of the thread's weight row; step
    // ks >= nk: 64 bf16 of the row's adapter factor B (zero-padded to RP).
    const int quad = warp & 3;
    const uint32_t par = (uint32_t)((warp - CVT_WARP0) >> 2);   // stages of this parity
    const int row = quad * 32 + lane;                           // row within the CTA's 128
    const float mu = DQ ? __ldg(p.dq_mean) : 0.0f;
    const int64_t kb_per_row = p.Kc / 64;
    const uint64_t pol = policy_evict_last();
    // What a converter needs of one stage, fetched two of its stages ahead:
    // the row's 32 code bytes and scale inputs (an adapter stage's 128 bytes
    // of B are read when it is converted: one stage in nk + RP/64).
    struct Src { uint4 c0, c1; float sg; int qa; int n; bool valid, ad; int ks; };
    auto fetch = [&](uint32_t ai, Src& d) -> bool {
      const uint32_t lt = ai / (uint32_t)nsteps;
      const int ks = (int)(ai - lt * (uint32_t)nsteps);
      const int tile = cluster + (int)lt * n_clusters;
      if (tile >= n_tiles) return false;
      const int n = (tile % n_pairs_n) * (2 * BN) + (int)rank * BN + row;
      d.valid = n < p.Nout;
      d.ad = ks >= nk;
      d.ks = ks;
      d.n = d.valid ? n : 0;
      if (!d.ad) {
        const uint4* codes = reinterpret_cast<const uint4*>(p.packed + (int64_t)d.n * (p.Kc / 2)) + 2 * ks;
        d.c0 = ldg_hint(codes, pol);
        d.c1 = ldg_hint(codes + 1, pol);
        const int64_t b = (int64_t)d.n * kb_per_row + ks;
        if (DQ) { d.qa = __ldcg(p.qabsmax + b); d.sg = __ldg(p.dq_scale + (b >> 8)); }
        else { d.sg = __ldcg(p.absmax + b); d.qa = 0; }
      }
      return true;
    };
    const uint32_t arow = smem_u32(&S.a[0][0]) + (uint32_t)row * 128u;
    const uint32_t swz = (uint32_t)(row & 7);
    Src s0, s1, s2;
    uint32_t ai = par;
    bool have0 = fetch(ai, s0);
    bool have1 = have0 && fetch(ai + 2, s1);
    while (have0) {
      const bool have2 = have1 && fetch(ai + 4, s2);   // this warp's stage after next
      uint32_t v[32];
      if (!s0.valid) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      } else if (s0.ad) {
        const uint4* src = reinterpret_cast<const uint4*>(p.wad + (int64_t)s0.n * p.RP + (s0.ks - nk) * BK);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 c = __ldcg(src + i);
          v[4 * i] = c.x; v[4 * i + 1] = c.y; v[4 * i + 2] = c.z; v[4 * i + 3] = c.w;
        }
      } else {
        // a^ = RN32(RN32(RN32(c / 127) * s_g) + mean), or the fp32 absmax
        const float a = DQ ? __fadd_rn(__fmul_rn(S.inv127[s0.qa + 128], s0.sg), mu) : s0.sg;
        const Lut l = build_lut(a, p.q);
        const uint32_t wds[8] = {s0.c0.x, s0.c0.y, s0.c0.z, s0.c0.w, s0.c1.x, s0.c1.y, s0.c1.z, s0.c1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) lookup8(wds[i], l, v + 4 * i);
      }
      const int sa = ai % NS;
      if (!mbar_wait_cluster(&S.a_empty[sa], ((ai / NS) & 1) ^ 1, abort, p.status)) break;
      // 16-byte chunk j (K elements 8j..8j+7) of the row at chunk position j ^ (row & 7)
      const uint32_t dst = arow + (uint32_t)sa * (uint32_t)A_BYTES;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        sts128(dst + ((((uint32_t)j) ^ swz) << 4), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&S.a_full[sa]), 0));
      s0 = s1;
      s1 = s2;
      have0 = have1;
      have1 = have2;
      ai += 2;
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5, both CTAs)
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t tmem_lane = (uint32_t)(quad * 32) << 16;
    const bool odd = lane & 1;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(&S.acc_empty), 0);
    uint32_t lt = 0;
    for (int tile = cluster; tile < n_tiles; tile += n_clusters, ++lt) {
      const int n0 = (tile % n_pairs_n) * (2 * BN) + (int)rank * BN;
      const int m0 = (tile / n_pairs_n) * (2 * BM);
      if (!mbar_wait_cluster(&S.acc_full, lt & 1, abort, p.status)) break;
      __syncwarp();
      tc_fence_after();
      // lane pairs (o, o+1) swap halves so each lane stores two adjacent
      // outputs of one token row: even lanes token m, odd lanes token m+1
      const int ocol = n0 + row_in_tile - (odd ? 1 : 0);
      // 32 columns per TMEM round trip (BM is a multiple of 16: a last
      // half-round of 16)
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
#pragma unroll 1
        for (int c0 = 0; c0 < BM; c0 += 32) {
          const bool two = c0 + 16 < BM;
          uint32_t v[32];
          tmem_ld16(tmem + tmem_lane + (uint32_t)(t * ACC1_COL + c0), v);
          if (two) tmem_ld16(tmem + tmem_lane + (uint32_t)(t * ACC1_COL + c0 + 16), v + 16);
          tmem_wait_ld();
          if (t == 1 && c0 + 32 >= BM) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          const int mfirst = m0 + t * BM + c0 + (odd ? 1 : 0);
          const int rows_left = (ocol < p.Nout) ? min(p.Mtok - mfirst, (two ? 32 : 16) - (odd ? 1 : 0)) : 0;
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (int64_t)mfirst * p.Nout + ocol);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const uint32_t mine = pk[c / 2];
            const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
            const uint32_t o = odd ? prmt(other, mine, 0x7632) : prmt(mine, other, 0x5410);
            if (c < rows_left) *dst = o;
            dst += p.Nout;                         // two bf16 rows = Nout words
          }
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

}  // namespace dual

// Token-tile width BM (per accumulator; two token tiles per weight tile) for
// an [Mtok x Nout] output on `clusters_max` SM pairs.  A pair tile costs
// about (fixed + 2 BM) per stage -- the fixed part is the converters' work
// and the pipeline hand-offs, measured in units of MMA token columns -- and a
// launch lasts as many rounds as the busiest pair runs tiles.
int dual_token_tile(int64_t Mtok, int64_t Nout, int clusters_max) {
  const int64_t fixed = 96;
  const int64_t n_pairs_n = (Nout + 255) / 256;
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int bm = 256; bm >= 64; bm -= 16) {
    const int64_t tiles = n_pairs_n * ((Mtok + 2 * bm - 1) / (2 * bm));
    const int64_t clusters = std::max<int64_t>(1, std::min<int64_t>(tiles, clusters_max));
    const int64_t rounds = (tiles + clusters - 1) / clusters;
    const int64_t cost = rounds * (2 * bm + fixed);
    if (cost < best_cost) { best_cost = cost; best = bm; }
  }
  return best;
}

// Forward NF4 GEMM with two token tiles per weight tile.  Returns QLORA_OK
// or QLORA_ERR_CUDA.
int launch_qlora_gemm_dual(const GemmArgs& a, const void* tok, const void* tokad, int RP,
                           cudaStream_t s, int num_sms) {
  using namespace dual;
  const int bm = dual_token_tile(a.Mtok, a.Nout, num_sms / 2);
  CUtensorMap t_tok, t_tokad;
  if (!make_tmap_2d_bf16(&t_tok, tok, a.Kc, a.Mtok, a.Kc, BK, bm / 2)) return QLORA_ERR_CUDA;
  if (!make_tmap_2d_bf16(&t_tokad, tokad, RP, a.Mtok, RP, BK, bm / 2)) return QLORA_ERR_CUDA;
  const int n_tiles = ((a.Nout + 2 * BN - 1) / (2 * BN)) * ((a.Mtok + 2 * bm - 1) / (2 * bm));
  const int clusters = std::max(1, std::min(n_tiles, num_sms / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (a.double_quant) {
    static std::atomic<unsigned long long> attr_devs{0};
    set_smem_attr_once(k_qlora_gemm_dual<true>, (int)smem_bytes(), attr_devs);
    e = cudaLaunchKernelEx(&cfg, k_qlora_gemm_dual<true>, t_tok, t_tokad, a, bm);
  } else {
    static std::atomic<unsigned long long> attr_devs{0};
    set_smem_attr_once(k_qlora_gemm_dual<false>, (int)smem_bytes(), attr_devs);
    e = cudaLaunchKernelEx(&cfg, k_qlora_gemm_dual<false>, t_tok, t_tokad, a, bm);
  }
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qnf4
