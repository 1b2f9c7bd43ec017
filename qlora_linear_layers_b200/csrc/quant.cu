// 4-bit blockwise quantise, double quantise and dequantise kernels
// (HBM-bound).
//
// Page "QLoRA Explained": section "The table, and the number that stretches
// it" (scale = block absmax, divide, round to the closest row, read back as
// row x scale), "Why the groups are small" (blocks of 64), "Shrink the scale
// factors too" (8-bit scales in groups of 256, one 32-bit constant each).

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace qnf4 {

// ===========================================================================
// Quantise: a 64-weight block belongs to two threads (bf16 input: 32
// weights, four 16-byte loads and a 16-byte code store each) or four (fp32
// input: 16 weights, an 8-byte store); the block max takes one or two
// shuffles, and a warp's blocks are contiguous.  A persistent grid (three
// CTAs per SM) walks the blocks; each thread loads its next block's words
// before it computes the current block's codes.  absmax is an integer max over |w| bit
// patterns (exact; NaN/Inf show up as >= 0x7f800000).
//
// Code of x = RN32(w / a):  x' = RN32(w * rcp(a)) with the hardware reciprocal
// (at most 1 ulp off) is within 3.5 ulp of x.  A 64-entry bucket table over
// [-1, 1] (width 1/16, index = round(16 x + 16), one 8-byte shared load from
// a copy per lane, so the 32 lanes never meet on a bank) holds the single
// threshold T that can fall in the bucket and the codes on either side of
// it.  When x' is more than 8 ulp from T, x and x' are on the same side of
// every threshold and the code follows from x' >= T; a block with any x'
// within 8 ulp of its T -- or whose absmax is 0 or below 2^-125 -- is redone
// with the IEEE division (rare; out of line).  Thresholds sit >= 1e-4 from
// bucket edges (checked on the host), so x' may pick the neighbouring bucket
// near an edge without effect.
//
// With a histogram pointer the kernel also adds every block absmax into the
// exponent histogram of the double quantisation (below): the significand of
// each absmax, summed per fp32 exponent over the warp (match + reduce), then
// into shared memory and, once per CTA, into the global 256-bin histogram.
// ===========================================================================

struct Bucket { float thr; uint32_t codes; };    // codes: lo (code = rank), or lo | hi << 8

__device__ __forceinline__ float rcp_approx(float a) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}

// Shared-memory address of x's bucket entry in this lane's copy of the table
// (bucket b, lane l at byte (b * 32 + l) * 8 from the table): 16 x + 16 + 2^23
// rounds to 2^23 + round(16 x + 16), whose bit pattern is 0x4B000000 + b; the
// shift by 8 drops the exponent bits and leaves b * 256.
__device__ __forceinline__ uint32_t bucket_addr(float x, uint32_t lane_base) {
  return (__float_as_uint(fmaf(x, 16.0f, 8388624.0f)) << 8) + lane_base;
}

__device__ __forceinline__ Bucket lds_bucket(uint32_t addr) {
  Bucket b;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(b.thr), "=r"(b.codes) : "r"(addr));
  return b;
}

template <bool MONO>
__device__ __forceinline__ uint32_t code_of(float x, uint32_t lane_base, uint32_t& nearm) {
  const Bucket b = lds_bucket(bucket_addr(x, lane_base));
  // same sign near T, so the bit patterns differ by the ulp distance
  nearm = __viaddmin_u32((uint32_t)(__float_as_int(x) - __float_as_int(b.thr)), 8u, nearm);
  const bool up = x >= b.thr;
  if (MONO) return b.codes + (up ? 1u : 0u);
  return up ? (b.codes >> 8) : (b.codes & 0xFFu);
}

// Threads that share one 64-weight block, and CTAs per SM: every thread
// holds 64 bytes of input (four 16-byte loads), so a bf16 block is split
// between two threads and an fp32 block between four; three CTAs per SM.
// Smaller parts give an SM more warps over the same bytes in flight.
template <typename T> struct QuantShape;
template <> struct QuantShape<__nv_bfloat16> { static constexpr int kTPB = 2, kCTAs = 3; };
template <> struct QuantShape<float> { static constexpr int kTPB = 4, kCTAs = 3; };

// Store N code words (N = 2, 4 or 8) at a 4N-byte aligned address.
template <int N>
__device__ __forceinline__ void store_code_words(uint8_t* dst, const uint32_t (&out)[N]) {
  if constexpr (N == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(out[0], out[1]);
  } else {
#pragma unroll
    for (int q = 0; q < N / 4; ++q)
      reinterpret_cast<uint4*>(dst)[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
  }
}

// Weight i of a thread's part of a block as an fp32 bit pattern, from the
// part's words, and the part's max |w| bit pattern.
template <typename T> struct PartWords;
template <> struct PartWords<__nv_bfloat16> {
  static constexpr int kWords = 32 / QuantShape<__nv_bfloat16>::kTPB;   // bf16 pairs, element 2j in the low half
  __device__ __forceinline__ static uint32_t elem(const uint32_t (&w)[kWords], int i) {
    return (i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16);
  }
  __device__ __forceinline__ static uint32_t absmax_bits(const uint32_t (&w)[kWords]) {
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < kWords; ++j) m[j & 3] = __vmaxu2(m[j & 3], w[j] & 0x7FFF7FFFu);
    const uint32_t mm = __vmaxu2(__vmaxu2(m[0], m[1]), __vmaxu2(m[2], m[3]));
    return max(mm << 16, mm & 0xFFFF0000u);
  }
};
template <> struct PartWords<float> {
  static constexpr int kWords = 64 / QuantShape<float>::kTPB;
  __device__ __forceinline__ static uint32_t elem(const uint32_t (&w)[kWords], int i) { return w[i]; }
  __device__ __forceinline__ static uint32_t absmax_bits(const uint32_t (&w)[kWords]) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < kWords; ++j) m = max(m, w[j] & 0x7FFFFFFFu);
    return m;
  }
};

// Exact codes of part `part` of block `blk` (weights [part * kW, +kW); x =
// RN32(w / a), or 0 for a zero block), written straight to `packed`: the rare
// path, kept out of line so the hot loop keeps its registers.
template <typename T, bool MONO>
__device__ __noinline__ void exact_part_codes(const void* W, int64_t blk, int part, float a,
                                              bool zero_block, uint32_t lane_base, uint8_t* packed) {
  constexpr int kW = 64 / QuantShape<T>::kTPB;
  uint32_t out[kW / 8];
#pragma unroll
  for (int k = 0; k < kW / 8; ++k) out[k] = 0u;
  uint32_t unused = 0;
  for (int i = 0; i < kW; ++i) {
    const int64_t idx = blk * 64 + part * kW + i;
    float w;
    if (sizeof(T) == 2) w = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[idx]);
    else w = reinterpret_cast<const float*>(W)[idx];
    const float x = zero_block ? 0.0f : __fdiv_rn(w, a);
    const uint32_t code = code_of<MONO>(x, lane_base, unused);
    const int sh = 8 * ((i >> 1) & 3) + ((i & 1) ? 0 : 4);
#pragma unroll
    for (int k = 0; k < kW / 8; ++k)
      if (k == (i >> 3)) out[k] |= code << sh;
  }
  store_code_words(packed + blk * 32 + part * (kW / 2), out);
}

template <typename T, bool MONO, bool HIST>
__global__ void __launch_bounds__(256, QuantShape<T>::kCTAs)
k_quantize(const void* __restrict__ W, int64_t nblk, uint8_t* __restrict__ packed,
           float* __restrict__ absmax, unsigned long long* __restrict__ hist, CodeTables tb,
           int* status) {
  constexpr int kTPB = QuantShape<T>::kTPB;
  constexpr int kWords = PartWords<T>::kWords;   // 32-bit words of a thread's part
  constexpr int kOut = 8 / kTPB;                 // code words of a part
  __shared__ __align__(8) Bucket s_bk[64 * 32];  // bucket b, lane l at b * 32 + l
  __shared__ unsigned long long s_hist[HIST ? 256 : 1];
  for (int i = threadIdx.x; i < 64 * 32; i += blockDim.x) {
    s_bk[i].thr = tb.bucket_thr[i >> 5];
    s_bk[i].codes = MONO ? tb.bucket_lo[i >> 5]
                         : (uint32_t)tb.bucket_lo[i >> 5] | ((uint32_t)tb.bucket_hi[i >> 5] << 8);
  }
  if (HIST)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_hist[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int pb = lane / kTPB, part = lane % kTPB;   // block of the warp's 32 / kTPB, part of it
  const uint32_t lane_base = smem_u32(s_bk) + (uint32_t)lane * 8u;
  bool bad = false;
  // warp-uniform loop (the histogram's match/reduce need whole warps); the
  // next block's words are loaded before this block's codes are computed
  const int64_t first = ((int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) / kTPB;
  const int64_t gstride = (int64_t)gridDim.x * blockDim.x / kTPB;
  uint32_t wn[kWords];
  auto load_words = [&](int64_t base_) {
    const int64_t b = base_ + pb;
    const bool v_ = b < nblk;
    const uint4* src = reinterpret_cast<const uint4*>(W) + (int64_t)(kWords * kTPB / 4) * (v_ ? b : 0) +
                       (kWords / 4) * part;
#pragma unroll
    for (int k = 0; k < kWords / 4; ++k) {
      const uint4 v = v_ ? __ldcs(src + k) : make_uint4(0u, 0u, 0u, 0u);
      wn[4 * k] = v.x; wn[4 * k + 1] = v.y; wn[4 * k + 2] = v.z; wn[4 * k + 3] = v.w;
    }
  };
  if (first < nblk) load_words(first);
  for (int64_t base = first; base < nblk; base += gstride) {
    const int64_t blk = base + pb;
    const bool valid = blk < nblk;
    uint32_t w[kWords];
#pragma unroll
    for (int k = 0; k < kWords; ++k) w[k] = wn[k];
    if (base + gstride < nblk) load_words(base + gstride);
    uint32_t m = PartWords<T>::absmax_bits(w);
#pragma unroll
    for (int o = 1; o < kTPB; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (m >= 0x7F800000u) { bad = true; m = 0; }
    const float a = __uint_as_float(m);
    if (valid) {
      const bool exact_block = m < 0x01000000u;   // a == 0 or a < 2^-125
      const float inv = exact_block ? 0.0f : rcp_approx(a);
      uint32_t out[kOut];
      uint32_t nearm = 0xFFFFFFFFu;               // min over the part of (ulp distance to T) + 8
#pragma unroll
      for (int k = 0; k < kOut; ++k) {
        uint32_t o = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = 8 * k + e;
          const float x = __fmul_rn(__uint_as_float(PartWords<T>::elem(w, i)), inv);
          // element 2j -> high nibble of byte j (fields disjoint: add = or)
          o += code_of<MONO>(x, lane_base, nearm) << (8 * (e >> 1) + ((e & 1) ? 0 : 4));
        }
        out[k] = o;
      }
      if (exact_block || nearm <= 16u) {
        exact_part_codes<T, MONO>(W, blk, part, a, m == 0, lane_base, packed);
      } else {
        store_code_words(packed + blk * 32 + part * (kOut * 4), out);
      }
      if (part == 0) absmax[blk] = a;
    }
    if (HIST) {
      const bool add = valid && m != 0u && part == 0;
      const uint32_t e = add ? (m >> 23) : 0xFFFFFFFFu;
      const uint32_t mant = add ? ((m & 0x7FFFFFu) | (e ? 0x800000u : 0u)) : 0u;
      const uint32_t grp = __match_any_sync(0xffffffffu, e);
      const uint32_t sum = __reduce_add_sync(grp, mant);       // < 32 * 2^24
      if (add && lane == __ffs(grp) - 1) atomicAdd(&s_hist[e], (unsigned long long)sum);
    }
  }
  if (HIST) {
    __syncthreads();
    for (int i = threadIdx.x; i < 255; i += blockDim.x)
      if (s_hist[i]) atomicAdd(&hist[i], s_hist[i]);
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
}

template <typename T, bool MONO>
static void launch_quantize_t(const void* W, int64_t nblk, uint8_t* packed, float* absmax,
                              unsigned long long* hist, const CodeTables& tb, int* status,
                              cudaStream_t s) {
  constexpr int kThreads = 256;
  constexpr int kTPB = QuantShape<T>::kTPB;
  // persistent grid: kCTAs per SM; other CTAs' loads cover each block's compute
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((nblk * kTPB + kThreads - 1) / kThreads,
                                                                 (int64_t)sms * QuantShape<T>::kCTAs));
  if (hist)
    k_quantize<T, MONO, true><<<blocks, kThreads, 0, s>>>(W, nblk, packed, absmax, hist, tb, status);
  else
    k_quantize<T, MONO, false><<<blocks, kThreads, 0, s>>>(W, nblk, packed, absmax, nullptr, tb, status);
}

int launch_quantize(const void* W, int dtype, int64_t n, int quant_type, uint8_t* packed,
                    float* absmax, unsigned long long* hist, int* status, cudaStream_t s,
                    int num_sms) {
  (void)num_sms;
  const CodeTables& tb = host_tables(quant_type);
  int launched = 1;
  if (hist) {
    cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned long long), s);
    ++launched;
  }
  const int64_t nblk = n / 64;
  if (dtype == QLORA_BF16) {
    if (tb.monotone) launch_quantize_t<__nv_bfloat16, true>(W, nblk, packed, absmax, hist, tb, status, s);
    else launch_quantize_t<__nv_bfloat16, false>(W, nblk, packed, absmax, hist, tb, status, s);
  } else {
    if (tb.monotone) launch_quantize_t<float, true>(W, nblk, packed, absmax, hist, tb, status, s);
    else launch_quantize_t<float, false>(W, nblk, packed, absmax, hist, tb, status, s);
  }
  return launched;
}

// ===========================================================================
// Double quantisation in two passes.
//   1. The exact per-tensor sum of absmax as a histogram: the 24-bit
//      significand of every absmax added (integer adds: exact and
//      order-independent) into the bin of its fp32 exponent field.  The
//      quantise kernel builds it on the fly; k_dq_hist builds it from an
//      absmax array.  Histograms of disjoint parts of a tensor add up to the
//      tensor's histogram (the multi-GPU sharding sums them).
//   2. k_dq_finalize: every CTA turns the complete histogram into the
//      correctly rounded fp64 sum and mean = RN32(RN64(sum) / n) -- the same
//      bits everywhere -- while its warps load their groups; then one warp
//      per group of 256: d = RN32(a - mean), s = max|d|,
//      c = rint(RN32(RN32(d / s) * 127)).
// ===========================================================================

// Exact integer S = sum_e hist[e] * 2^(max(e,1)-1) in units of 2^-149 (a float
// with exponent field e and significand m is m * 2^(max(e,1) - 150)), rounded
// to the nearest double (ties to even); returns RN32(RN64(S * 2^-149) / n).
// Called by one full warp: lane w < 12 sums the bins whose shift falls in
// 32-bit word w as a 128-bit integer (at most 32 terms below 2^95), then lane
// 0 carries the words into a 384-bit integer and rounds it.  Every lane
// returns the result.
__device__ float exact_mean_warp(const unsigned long long* hist, int64_t n) {
  constexpr int L = 12;                  // 384-bit integer, little-endian 32-bit words
  const int lane = threadIdx.x & 31;
  unsigned __int128 part = 0;
  if (lane < L) {
    // bins with shift sh = max(e,1) - 1 in [32 lane, 32 lane + 31]
    const int e_lo = lane == 0 ? 0 : 32 * lane + 1;
    const int e_hi = min(32 * lane + 32, 254);
    for (int e = e_lo; e <= e_hi; ++e) {
      const unsigned long long v = hist[e];
      const int sh = (e > 0 ? e : 1) - 1;
      part += (unsigned __int128)v << (sh & 31);
    }
  }
  uint32_t acc[L];
  unsigned __int128 carry = 0;
#pragma unroll
  for (int w = 0; w < L; ++w) {
    unsigned __int128 pw = 0;
    const uint64_t lo = __shfl_sync(0xffffffffu, (uint64_t)part, w);
    const uint64_t hi = __shfl_sync(0xffffffffu, (uint64_t)(part >> 64), w);
    pw = ((unsigned __int128)hi << 64) | lo;
    const unsigned __int128 t = pw + carry;
    acc[w] = (uint32_t)t;
    carry = t >> 32;
  }
  // word i of S, branch-free (i may be out of range: 0)
  auto word = [&](int i) -> uint32_t {
    uint32_t r = 0;
#pragma unroll
    for (int w = 0; w < L; ++w) r = (i == w) ? acc[w] : r;
    return r;
  };
  int tw = -1;
#pragma unroll
  for (int w = 0; w < L; ++w) tw = acc[w] ? w : tw;
  double S = 0.0;
  if (tw >= 0) {
    const int top = 32 * tw + 31 - __clz(word(tw));
    // 64 bits of S starting at bit position lo (lo >= 0)
    auto bits64 = [&](int lo) -> unsigned long long {
      const int w = lo >> 5, b = lo & 31;
      const unsigned long long w0 = word(w), w1 = word(w + 1), w2 = word(w + 2);
      const unsigned long long low = w0 | (w1 << 32);
      return b ? ((low >> b) | (w2 << (64 - b))) : low;
    };
    if (top <= 52) {
      S = ldexp((double)bits64(0), -149);             // exact
    } else {
      const int sh = top - 52;                         // the 53-bit significand is bits [sh, top]
      unsigned long long mant = bits64(sh) & ((1ull << 53) - 1);
      const uint32_t round_bit = (uint32_t)(bits64(sh - 1) & 1ull);
      // sticky: any set bit below sh - 1
      const int below = sh - 1;
      bool sticky = false;
#pragma unroll
      for (int w = 0; w < L; ++w) {
        const uint32_t m = (32 * w + 32 <= below) ? 0xFFFFFFFFu
                         : (32 * w < below) ? ((1u << (below - 32 * w)) - 1u) : 0u;
        sticky |= (acc[w] & m) != 0;
      }
      if (round_bit && (sticky || (mant & 1ull))) ++mant;
      int expo = sh;
      if (mant == (1ull << 53)) { mant >>= 1; ++expo; }
      S = ldexp((double)mant, expo - 149);
    }
  }
  return __double2float_rn(__ddiv_rn(S, (double)n));
}

// Pass 1 on an absmax array (standalone double quantisation).  Every lane of
// a warp runs the same number of iterations (match/reduce need the full
// warp); a thread's kU loads are all issued before the first is used.
__global__ void __launch_bounds__(512)
k_dq_hist(const float* __restrict__ absmax, int64_t n, unsigned long long* __restrict__ hist,
          int* status) {
  __shared__ unsigned long long sh[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sh[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  bool bad = false;
  constexpr int kU = 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t first = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  for (int64_t base0 = first; base0 < n; base0 += kU * stride) {
    uint32_t u[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int64_t i = base0 + k * stride + lane;
      u[k] = i < n ? __float_as_uint(__ldcs(absmax + i)) : 0xFFFFFFFFu;   // sentinel: no element
    }
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      if (base0 + k * stride >= n) break;        // warp-uniform
      uint32_t e = 0xFFFFFFFFu, mant = 0;
      if (u[k] != 0xFFFFFFFFu) {
        if (u[k] >= 0x7F800000u) {     // negative (sign set, nonzero) or NaN/Inf
          if (u[k] != 0x80000000u) bad = true;
        } else {
          e = u[k] >> 23;
          mant = (u[k] & 0x7FFFFFu) | (e ? 0x800000u : 0u);
        }
      }
      const uint32_t grp = __match_any_sync(0xffffffffu, e);
      const uint32_t sum = __reduce_add_sync(grp, mant);     // < 32 * 2^24
      const int leader = __ffs(grp) - 1;
      if (lane == leader && e != 0xFFFFFFFFu && sum)
        atomicAdd(&sh[e], (unsigned long long)sum);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 255; i += blockDim.x)
    if (sh[i]) atomicAdd(&hist[i], sh[i]);
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
}

// Pass 2: the mean over n_total absmax values (this array's n and any other
// shards' absmax whose histograms were added in), then the int8 codes and
// fp32 scales of this array's groups.
template <int DQT>
__global__ void __launch_bounds__(512)
k_dq_finalize(const float* __restrict__ absmax, int64_t n, const unsigned long long* __restrict__ hist,
              int64_t n_total, int8_t* __restrict__ qabsmax, float* __restrict__ dq_scale,
              float* __restrict__ mean) {
  __shared__ unsigned long long sh[256];
  __shared__ float s_mu;
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sh[i] = i < 255 ? __ldcg(&hist[i]) : 0ull;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ngroups = (n + 255) / 256;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  float av[8];
  auto load = [&](int64_t gg) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t i = gg * 256 + j * 32 + lane;
      av[j] = i < n ? __ldcg(absmax + i) : 0.0f;
    }
  };
  if (g < ngroups) load(g);                      // in flight while the mean is formed
  __syncthreads();
  if (warp == 0) {
    const float mu = exact_mean_warp(sh, n_total);
    if (lane == 0) {
      s_mu = mu;
      if (blockIdx.x == 0) mean[0] = mu;
    }
  }
  __syncthreads();
  const float mu = s_mu;
  for (bool first = true; g < ngroups; g += nw, first = false) {
    if (!first) load(g);
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t i = g * 256 + j * 32 + lane;
      d[j] = (i < n) ? __fsub_rn(av[j], mu) : 0.0f;
      m = fmaxf(m, fabsf(d[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t i = g * 256 + j * 32 + lane;
      if (i < n) {
        int c = 0;
        if (m != 0.0f) {
          if (DQT == 2) {
            // E4M3 code of 256 * RN32(d / s_g) (exact scaling), nearest, ties to even
            c = (int)(int8_t)__nv_cvt_float_to_fp8(__fmul_rn(__fdiv_rn(d[j], m), 256.0f), __NV_SATFINITE, __NV_E4M3);
          } else {
            c = __float2int_rn(__fmul_rn(__fdiv_rn(d[j], m), 127.0f));
            c = min(max(c, -127), 127);
          }
        }
        qabsmax[i] = (int8_t)c;
      }
    }
    if (lane == 0) dq_scale[g] = m;
  }
}

// Returns the number of kernels launched.
int launch_double_quantize_from_hist(const float* absmax, int64_t n, const unsigned long long* hist,
                                     int64_t n_total, int8_t* qabsmax, float* dq_scale, float* dq_mean,
                                     cudaStream_t s, int num_sms, int dq_type) {
  const int64_t ngroups = (n + 255) / 256;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((ngroups + 15) / 16, (int64_t)num_sms * 2));
  if (dq_type == 2)
    k_dq_finalize<2><<<blocks, 512, 0, s>>>(absmax, n, hist, n_total, qabsmax, dq_scale, dq_mean);
  else
    k_dq_finalize<1><<<blocks, 512, 0, s>>>(absmax, n, hist, n_total, qabsmax, dq_scale, dq_mean);
  return 1;
}

int launch_double_quantize(const float* absmax, int64_t n, int8_t* qabsmax, float* dq_scale,
                           float* dq_mean, unsigned long long* hist, int* status, cudaStream_t s,
                           int num_sms) {
  cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned long long), s);
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n + 8191) / 8192, (int64_t)num_sms));
  k_dq_hist<<<blocks, 512, 0, s>>>(absmax, n, hist, status);
  return 2 + launch_double_quantize_from_hist(absmax, n, hist, n, qabsmax, dq_scale, dq_mean, s, num_sms, 1);
}

// ===========================================================================
// Dequantise: a thread expands 8 weights per chunk (a 4-byte code load, a
// 16-byte bf16 store; contiguous per warp) and keeps four chunks in flight;
// 8 lanes share a block's scale.  w' = RNbf16(RN32(q[code] * a^)), a^
// recovered from the double-quantised constants as
// RN32(RN32(RN32(c / 127) * s_g) + mean).
// ===========================================================================

template <bool DQ>
__global__ void __launch_bounds__(256)
k_dequantize(const uint32_t* __restrict__ packed, int64_t nchunks,
             const float* __restrict__ absmax, const int8_t* __restrict__ qabsmax,
             const float* __restrict__ dq_scale, const float* __restrict__ dq_mean,
             uint4* __restrict__ out, CodeTables tb, int dq_type) {
  constexpr int kU = 4;
  __shared__ float s_q[16];
  __shared__ float s_inv127[256];
  if (threadIdx.x < 16) s_q[threadIdx.x] = tb.q[threadIdx.x];
  s_inv127[threadIdx.x] = dq_code_value((int)threadIdx.x, dq_type);   // entry c + 128: any code byte
  __syncthreads();
  const float mu = DQ ? dq_mean[0] : 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c0 < nchunks; c0 += kU * stride) {
    uint32_t wd[kU];
    float a[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t c = c0 + u * stride;
      const int64_t blk = (c < nchunks ? c : 0) >> 3;
      wd[u] = c < nchunks ? __ldcs(packed + c) : 0u;
      if (DQ) a[u] = __fadd_rn(__fmul_rn(s_inv127[qabsmax[blk] + 128], __ldg(dq_scale + (blk >> 8))), mu);
      else a[u] = __ldg(absmax + blk);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t c = c0 + u * stride;
      if (c >= nchunks) break;
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {            // byte j -> elements 2j (high nibble), 2j+1 (low)
        const uint32_t byte = (wd[u] >> (8 * j)) & 0xFFu;
        o[j] = pack_bf16x2(__fmul_rn(s_q[byte >> 4], a[u]), __fmul_rn(s_q[byte & 15], a[u]));
      }
      __stcs(out + c, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

void launch_dequantize(const nf4_weight* w, void* out, cudaStream_t s, int num_sms) {
  const int64_t n = w->rows * w->cols;
  const int64_t nchunks = n / 8;
  int blocks = (int)std::min<int64_t>((nchunks + 1023) / 1024, (int64_t)num_sms * 8);
  blocks = std::max(blocks, 1);
  const CodeTables& tb = host_tables(w->quant_type);
  if (w->double_quant)
    k_dequantize<true><<<blocks, 256, 0, s>>>((const uint32_t*)w->packed, nchunks, nullptr, w->qabsmax,
                                              w->dq_scale, w->dq_mean, (uint4*)out, tb, w->double_quant);
  else
    k_dequantize<false><<<blocks, 256, 0, s>>>((const uint32_t*)w->packed, nchunks, w->absmax, nullptr,
                                               nullptr, nullptr, (uint4*)out, tb, 0);
}

}  // namespace qnf4
