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
// Quantise: one thread owns 8 consecutive weights (one 16-byte bf16 load, a
// 4-byte code store), 8 adjacent lanes own one 64-weight block, so every warp
// access is contiguous.  absmax is an integer max over |w| bit patterns
// (exact; NaN/Inf show up as >= 0x7f800000), joined by 3 shuffles.
//
// Code of x = RN32(w / a):  x' = RN32(w * RN32(1/a)) is within 2.5 ulp of x.
// A 64-entry bucket table over [-1, 1] (width 1/16, index = round(16 x + 16),
// read with one 8-byte shared load) holds the single threshold T that can
// fall in the bucket and the number of thresholds below it.  When x' is more
// than 8 ulp from T, x and x' are on the same side of every threshold and the
// code is base + (x' >= T); otherwise -- and for blocks whose absmax is 0 or
// below 2^-125 -- x is computed exactly with the IEEE division (a rarely
// taken branch, kept out of the unrolled loop).  Thresholds sit >= 1e-4 from bucket edges (checked on the
// host), so x' may pick the neighbouring bucket near an edge without effect.
// ===========================================================================

// Loaders return the 8 weights as fp32 bit patterns and the max of their
// magnitudes' bit patterns (bf16: a 16-bit SIMD max over packed pairs).
template <typename T> struct Loader8;
template <> struct Loader8<__nv_bfloat16> {
  __device__ __forceinline__ static uint32_t load(const void* base, int64_t chunk, uint32_t (&u)[8]) {
    const uint4 q = __ldcs(reinterpret_cast<const uint4*>(base) + chunk);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t mp = __vmaxu2(__vmaxu2(w[0] & 0x7FFF7FFFu, w[1] & 0x7FFF7FFFu),
                           __vmaxu2(w[2] & 0x7FFF7FFFu, w[3] & 0x7FFF7FFFu));
#pragma unroll
    for (int j = 0; j < 4; ++j) { u[2 * j] = w[j] << 16; u[2 * j + 1] = w[j] & 0xFFFF0000u; }
    return max(mp << 16, mp & 0xFFFF0000u);
  }
};
template <> struct Loader8<float> {
  __device__ __forceinline__ static uint32_t load(const void* base, int64_t chunk, uint32_t (&u)[8]) {
    const uint4* p = reinterpret_cast<const uint4*>(base) + 2 * chunk;
    const uint4 a = __ldcs(p), b = __ldcs(p + 1);
    u[0] = a.x; u[1] = a.y; u[2] = a.z; u[3] = a.w; u[4] = b.x; u[5] = b.y; u[6] = b.z; u[7] = b.w;
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = max(m, u[i] & 0x7FFFFFFFu);
    return m;
  }
};

struct Bucket { float thr; uint32_t base; };

__device__ __forceinline__ uint32_t bucket_index(float x) {
  // round(16 x + 16) lands in the low mantissa bits of 16 x + 16 + 2^23
  return __float_as_uint(fmaf(x, 16.0f, 8388624.0f)) & 63u;
}

// Exact codes x = RN32(w / a) for the elements of `chunk` flagged in `mask`
// (rare: a fast quotient within 8 ulp of a threshold, or a zero / tiny absmax
// block).  The flagged weights are re-read (cached) rather than passed in, so
// the hot loop keeps its values in registers.
template <typename T>
__device__ __noinline__ uint32_t exact_codes(const void* W, int64_t chunk, float a, bool zero_block,
                                             uint32_t mask, uint32_t out, const Bucket* bks) {
  for (int i = 0; i < 8; ++i) {
    if (!((mask >> i) & 1u)) continue;
    float w;
    if (sizeof(T) == 2) w = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[chunk * 8 + i]);
    else w = reinterpret_cast<const float*>(W)[chunk * 8 + i];
    const float x = zero_block ? 0.0f : __fdiv_rn(w, a);
    const Bucket bk = bks[bucket_index(x)];
    const uint32_t code = bk.base + (x >= bk.thr ? 1u : 0u);
    const int sh = 8 * (i >> 1) + ((i & 1) ? 0 : 4);
    out = (out & ~(0xFu << sh)) | (code << sh);
  }
  return out;
}

template <typename T>
__global__ void __launch_bounds__(256)
k_nf4_quantize(const void* __restrict__ W, int64_t nchunks, uint8_t* __restrict__ packed,
               float* __restrict__ absmax, Nf4Tables tb, int* status) {
  __shared__ Bucket s_bk[64];
  if (threadIdx.x < 64) {
    const int b = threadIdx.x;
    s_bk[b].thr = tb.bucket_thr[b];
    s_bk[b].base = tb.bucket_base[b];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  bool bad = false;
  // Two chunks per iteration (both loads in flight before either is used);
  // every lane of a warp runs the same number of iterations (shuffles below).
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < nchunks;
       base += 2 * stride) {
    uint32_t u[2][8], mloc[2] = {0u, 0u};
    int64_t chunk[2];
    bool active[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      chunk[h] = base + h * stride + lane;
      active[h] = chunk[h] < nchunks;             // whole 8-lane groups (nchunks % 8 == 0)
      if (active[h]) mloc[h] = Loader8<T>::load(W, chunk[h], u[h]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t m = mloc[h];
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
      if (!active[h]) continue;
      if (m >= 0x7F800000u) { bad = true; m = 0; }
      const float a = __uint_as_float(m);
      const bool exact_block = m < 0x01000000u;   // a == 0 or a < 2^-125
      const float inv = exact_block ? 0.0f : __frcp_rn(a);
      uint32_t out = 0;
      bool anynear = exact_block;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = __fmul_rn(__uint_as_float(u[h][i]), inv);
        const Bucket bk = s_bk[bucket_index(x)];
        // within 8 ulp of the threshold (same sign there, so the bit patterns
        // differ by the ulp distance): decide exactly below
        anynear |= (uint32_t)(__float_as_int(x) - __float_as_int(bk.thr) + 8) <= 16u;
        const uint32_t code = bk.base + (x >= bk.thr ? 1u : 0u);
        // element 2j -> high nibble of byte j; byte j at bits 8j (fields disjoint: add = or)
        out += code << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
      }
      if (anynear) out = exact_codes<T>(W, chunk[h], a, m == 0, 0xFFu, out, s_bk);
      reinterpret_cast<uint32_t*>(packed)[chunk[h]] = out;
      if ((lane & 7) == 0) absmax[chunk[h] >> 3] = a;
    }
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
}

void launch_quantize(const void* W, int dtype, int64_t n, uint8_t* packed, float* absmax,
                     int* status, cudaStream_t s, int num_sms) {
  const int64_t nchunks = n / 8;
  const int threads = 256;
  int blocks = (int)std::min<int64_t>((nchunks + threads - 1) / threads, (int64_t)num_sms * 8);
  blocks = std::max(blocks, 1);
  const Nf4Tables& tb = host_tables();
  if (dtype == QLORA_BF16)
    k_nf4_quantize<__nv_bfloat16><<<blocks, threads, 0, s>>>(W, nchunks, packed, absmax, tb, status);
  else
    k_nf4_quantize<float><<<blocks, threads, 0, s>>>(W, nchunks, packed, absmax, tb, status);
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
  s_inv127[threadIdx.x] = __fdiv_rn((float)((int)threadIdx.x - 127), 127.0f);
  __syncthreads();
  const float mu = DQ ? dq_mean[0] : 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < nchunks;
       chunk += stride) {
    const int64_t blk = chunk >> 3;
    float a;
    if (DQ) a = __fadd_rn(__fmul_rn(s_inv127[qabsmax[blk] + 127], __ldg(dq_scale + (blk >> 8))), mu);
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
