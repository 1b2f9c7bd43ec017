// NF4 quantise, double quantise and dequantise kernels (HBM-bound).
//
// Page "QLoRA Explained": section "The table, and the number that stretches
// it" (scale = block absmax, divide, round to the closest row, read back as
// row x scale), "Why the groups are small" (blocks of 64), "Shrink the scale
// factors too" (8-bit scales in groups of 256, one 32-bit constant each).

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace qnf4 {

// ===========================================================================
// Quantise: one thread owns one 64-weight block (eight 16-byte bf16 loads or
// sixteen fp32 ones, a 32-byte code store and its absmax), so the block max,
// the reciprocal and the stores cost one thread's work per 64 weights.
// absmax is an integer max over |w| bit patterns (exact; NaN/Inf show up as
// >= 0x7f800000).
//
// Code of x = RN32(w / a):  x' = RN32(w * rcp(a)) with the hardware reciprocal
// (at most 1 ulp off) is within 3.5 ulp of x.  A 64-entry bucket table over
// [-1, 1] (width 1/16, index = round(16 x + 16), one 8-byte shared load from
// a copy per lane, so the 32 lanes never meet on a bank) holds the single
// threshold T that can fall in the bucket and the number of thresholds below
// it.  When x' is more than 8 ulp from T, x and x'
// are on the same side of every threshold and the code is base + (x' >= T);
// a block with any x' within 8 ulp of its T -- or whose absmax is 0 or below
// 2^-125 -- is redone with the IEEE division (rare; out of line).  Thresholds
// sit >= 1e-4 from bucket edges (checked on the host), so x' may pick the
// neighbouring bucket near an edge without effect.
// ===========================================================================

struct Bucket { float thr; uint32_t base; };

__device__ __forceinline__ uint32_t bucket_index(float x) {
  // round(16 x + 16) lands in the low mantissa bits of 16 x + 16 + 2^23
  return __float_as_uint(fmaf(x, 16.0f, 8388624.0f)) & 63u;
}

__device__ __forceinline__ float rcp_approx(float a) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}

// Weight i (0..63) of a block as an fp32 bit pattern, from the block's words.
template <typename T> struct BlockWords;
template <> struct BlockWords<__nv_bfloat16> {
  static constexpr int kWords = 32;               // bf16 pairs, element 2j in the low half
  __device__ __forceinline__ static uint32_t elem(const uint32_t (&w)[kWords], int i) {
    return (i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16);
  }
  __device__ __forceinline__ static uint32_t absmax_bits(const uint32_t (&w)[kWords]) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < kWords; ++j) m = __vmaxu2(m, w[j] & 0x7FFF7FFFu);
    return max(m << 16, m & 0xFFFF0000u);
  }
};
template <> struct BlockWords<float> {
  static constexpr int kWords = 64;
  __device__ __forceinline__ static uint32_t elem(const uint32_t (&w)[kWords], int i) { return w[i]; }
  __device__ __forceinline__ static uint32_t absmax_bits(const uint32_t (&w)[kWords]) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < kWords; ++j) m = max(m, w[j] & 0x7FFFFFFFu);
    return m;
  }
};

// Exact codes of block `blk` (x = RN32(w / a), or 0 for a zero block),
// written straight to `packed`: the rare path, kept out of line so the hot
// loop keeps its registers.
template <typename T>
__device__ __noinline__ void exact_block_codes(const void* W, int64_t blk, float a, bool zero_block,
                                               const Bucket* bks, uint8_t* packed) {
  uint32_t out[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) out[k] = 0u;
  for (int i = 0; i < 64; ++i) {
    float w;
    if (sizeof(T) == 2) w = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[blk * 64 + i]);
    else w = reinterpret_cast<const float*>(W)[blk * 64 + i];
    const float x = zero_block ? 0.0f : __fdiv_rn(w, a);
    const Bucket bk = bks[bucket_index(x) * 32];
    const uint32_t code = bk.base + (x >= bk.thr ? 1u : 0u);
    const int sh = 8 * ((i >> 1) & 3) + ((i & 1) ? 0 : 4);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k == (i >> 3)) out[k] |= code << sh;
  }
  uint4* dst = reinterpret_cast<uint4*>(packed) + 2 * blk;
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
}

template <typename T>
__global__ void __launch_bounds__(256)
k_nf4_quantize(const void* __restrict__ W, int64_t nblk, uint8_t* __restrict__ packed,
               float* __restrict__ absmax, Nf4Tables tb, int* status) {
  __shared__ Bucket s_bk[64 * 32];               // bucket b, lane l at b * 32 + l
  for (int i = threadIdx.x; i < 64 * 32; i += blockDim.x) {
    s_bk[i].thr = tb.bucket_thr[i >> 5];
    s_bk[i].base = tb.bucket_base[i >> 5];
  }
  __syncthreads();
  const Bucket* bk_lane = s_bk + (threadIdx.x & 31);
  constexpr int kWords = BlockWords<T>::kWords;
  bool bad = false;
  for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblk;
       blk += (int64_t)gridDim.x * blockDim.x) {
    uint32_t w[kWords];
    const uint4* src = reinterpret_cast<const uint4*>(W) + (int64_t)(kWords / 4) * blk;
#pragma unroll
    for (int k = 0; k < kWords / 4; ++k) {
      const uint4 v = __ldg(src + k);
      w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
    }
    uint32_t m = BlockWords<T>::absmax_bits(w);
    if (m >= 0x7F800000u) { bad = true; m = 0; }
    const float a = __uint_as_float(m);
    const bool exact_block = m < 0x01000000u;     // a == 0 or a < 2^-125
    const float inv = exact_block ? 0.0f : rcp_approx(a);
    uint32_t out[8];
    uint32_t nearm = 0xFFFFFFFFu;                 // min over the block of (ulp distance to T) + 8
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t o = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = 8 * k + e;
        const float x = __fmul_rn(__uint_as_float(BlockWords<T>::elem(w, i)), inv);
        const Bucket bk = bk_lane[bucket_index(x) * 32];
        // same sign near T, so the bit patterns differ by the ulp distance
        nearm = min(nearm, (uint32_t)(__float_as_int(x) - __float_as_int(bk.thr) + 8));
        const uint32_t code = bk.base + (x >= bk.thr ? 1u : 0u);
        // element 2j -> high nibble of byte j (fields disjoint: add = or)
        o += code << (8 * (e >> 1) + ((e & 1) ? 0 : 4));
      }
      out[k] = o;
    }
    if (exact_block || nearm <= 16u) {
      exact_block_codes<T>(W, blk, a, m == 0, s_bk, packed);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(packed) + 2 * blk;
      dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
      dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
    absmax[blk] = a;
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
}

void launch_quantize(const void* W, int dtype, int64_t n, uint8_t* packed, float* absmax,
                     int* status, cudaStream_t s, int num_sms) {
  const int64_t nblk = n / 64;
  const int threads = 256;
  // one block per thread: other CTAs' loads cover each block's compute
  int blocks = (int)std::min<int64_t>((nblk + threads - 1) / threads, (int64_t)1 << 30);
  blocks = std::max(blocks, 1);
  const Nf4Tables& tb = host_tables();
  if (dtype == QLORA_BF16)
    k_nf4_quantize<__nv_bfloat16><<<blocks, threads, 0, s>>>(W, nblk, packed, absmax, tb, status);
  else
    k_nf4_quantize<float><<<blocks, threads, 0, s>>>(W, nblk, packed, absmax, tb, status);
}

// ===========================================================================
// Double quantisation, one cooperative kernel:
//   1. exact per-tensor sum of absmax: histogram of 24-bit significands per
//      fp32 exponent (integer adds: exact and order-independent), per block
//      in shared memory, then added into a global histogram;
//   2. one grid barrier (counted in bin 255, which no finite value uses);
//      every block turns the complete histogram into the correctly rounded
//      fp64 sum and mean = RN32(RN64(sum) / n) -- the same bits everywhere;
//   3. one warp per group of 256: d = RN32(a - mean), s = max|d|,
//      c = rint(RN32(RN32(d / s) * 127)) (the group re-read from L2).
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

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(512)
k_double_quant(const float* __restrict__ absmax, int64_t n, unsigned long long* __restrict__ hist,
               int8_t* __restrict__ qabsmax, float* __restrict__ dq_scale, float* __restrict__ mean,
               int* status) {
  __shared__ unsigned long long sh[256];
  __shared__ float s_mu;
  __shared__ int s_ok;
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sh[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  bool bad = false;
  // ---- 1. histogram; every lane of a warp runs the same number of
  // iterations (match/reduce below need the full warp).  A thread's kU loads
  // are all issued before the first is used.
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
  // ---- 2. grid barrier (all blocks are co-resident: cooperative launch),
  // bounded; then the exact mean from the complete histogram
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(&hist[255], 1ull);
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u64(&hist[255]) < (unsigned long long)gridDim.x) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        ok = 0;
        set_status(status, QLORA_ERR_TIMEOUT);
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return;
  for (int i = threadIdx.x; i < 255; i += blockDim.x) sh[i] = __ldcg(&hist[i]);
  __syncthreads();
  if (threadIdx.x < 32) {
    const float mu = exact_mean_warp(sh, n);
    if (threadIdx.x == 0) {
      s_mu = mu;
      if (blockIdx.x == 0) mean[0] = mu;
    }
  }
  __syncthreads();
  // ---- 3. one warp per group of 256
  const float mu = s_mu;
  const int64_t ngroups = (n + 255) / 256;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t g = warp; g < ngroups; g += nwarps) {
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t i = g * 256 + j * 32 + lane;
      d[j] = (i < n) ? __fsub_rn(__ldcg(absmax + i), mu) : 0.0f;
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
          c = __float2int_rn(__fmul_rn(__fdiv_rn(d[j], m), 127.0f));
          c = min(max(c, -127), 127);
        }
        qabsmax[i] = (int8_t)c;
      }
    }
    if (lane == 0) dq_scale[g] = m;
  }
}

// Returns the number of kernels launched (1), or -1 if the cooperative launch
// was refused.
int launch_double_quantize(const float* absmax, int64_t n, int8_t* qabsmax, float* dq_scale,
                           float* dq_mean, unsigned long long* hist, int* status,
                           cudaStream_t s, int num_sms) {
  cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned long long), s);
  // one wide block per SM (fewer blocks meet on the few busy histogram bins)
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n + 8191) / 8192, (int64_t)num_sms));
  void* args[] = {(void*)&absmax, (void*)&n, (void*)&hist, (void*)&qabsmax, (void*)&dq_scale,
                  (void*)&dq_mean, (void*)&status};
  return cudaLaunchCooperativeKernel((const void*)k_double_quant, dim3(blocks), dim3(512), args, 0, s) ==
                 cudaSuccess ? 1 : -1;
}

// ===========================================================================
// Dequantise: one thread owns 8 weights (a 4-byte code load, a 16-byte bf16
// store; contiguous per warp), 8 lanes share a block's scale.
// w' = RNbf16(RN32(q[code] * a^)), a^ recovered from the double-quantised
// constants as RN32(RN32(RN32(c / 127) * s_g) + mean).
// ===========================================================================

template <bool DQ>
__global__ void __launch_bounds__(256)
k_nf4_dequantize(const uint8_t* __restrict__ packed, int64_t nchunks,
                 const float* __restrict__ absmax, const int8_t* __restrict__ qabsmax,
                 const float* __restrict__ dq_scale, const float* __restrict__ dq_mean,
                 uint4* __restrict__ out, Nf4Tables tb) {
  __shared__ float s_q[16];
  __shared__ float s_inv127[256];
  if (threadIdx.x < 16) s_q[threadIdx.x] = tb.q[threadIdx.x];
  s_inv127[threadIdx.x] = __fdiv_rn((float)((int)threadIdx.x - 128), 127.0f);   // entry c + 128: any int8 c
  __syncthreads();
  const float mu = DQ ? dq_mean[0] : 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < nchunks;
       chunk += stride) {
    const int64_t blk = chunk >> 3;
    float a;
    if (DQ) a = __fadd_rn(__fmul_rn(s_inv127[qabsmax[blk] + 128], __ldg(dq_scale + (blk >> 8))), mu);
    else a = __ldg(absmax + blk);
    const uint32_t wd = __ldcs(reinterpret_cast<const uint32_t*>(packed) + chunk);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {            // byte j -> elements 2j (high nibble), 2j+1 (low)
      const uint32_t byte = (wd >> (8 * j)) & 0xFFu;
      o[j] = pack_bf16x2(__fmul_rn(s_q[byte >> 4], a), __fmul_rn(s_q[byte & 15], a));
    }
    __stcs(out + chunk, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

void launch_dequantize(const nf4_weight* w, void* out, cudaStream_t s, int num_sms) {
  const int64_t n = w->rows * w->cols;
  const int64_t nchunks = n / 8;
  int blocks = (int)std::min<int64_t>((nchunks + 255) / 256, (int64_t)num_sms * 8);
  blocks = std::max(blocks, 1);
  const Nf4Tables& tb = host_tables();
  if (w->double_quant)
    k_nf4_dequantize<true><<<blocks, 256, 0, s>>>(w->packed, nchunks, nullptr, w->qabsmax,
                                                  w->dq_scale, w->dq_mean, (uint4*)out, tb);
  else
    k_nf4_dequantize<false><<<blocks, 256, 0, s>>>(w->packed, nchunks, w->absmax, nullptr,
                                                   nullptr, nullptr, (uint4*)out, tb);
}

}  // namespace qnf4
