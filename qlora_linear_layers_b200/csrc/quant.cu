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
// Quantise: one thread owns 32 consecutive weights, an adjacent lane pair owns
// one 64-weight block.  absmax is an integer max over |w| bit patterns (exact,
// and any NaN/Inf shows up as >= 0x7f800000); one shuffle joins the pair.
// ===========================================================================

template <typename T> struct Loader;

template <> struct Loader<__nv_bfloat16> {
  // 32 bf16 = 4 x 16 bytes; returns the fp32 bit patterns.
  __device__ __forceinline__ static void load(const void* base, int64_t chunk, uint32_t (&u)[32]) {
    const uint4* p = reinterpret_cast<const uint4*>(base) + chunk * 4;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 q = __ldcs(p + v);
      uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        u[8 * v + 2 * j] = w[j] << 16;
        u[8 * v + 2 * j + 1] = w[j] & 0xFFFF0000u;
      }
    }
  }
};

template <> struct Loader<float> {
  __device__ __forceinline__ static void load(const void* base, int64_t chunk, uint32_t (&u)[32]) {
    const uint4* p = reinterpret_cast<const uint4*>(base) + chunk * 8;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint4 q = __ldcs(p + v);
      u[4 * v] = q.x; u[4 * v + 1] = q.y; u[4 * v + 2] = q.z; u[4 * v + 3] = q.w;
    }
  }
};

template <typename T>
__global__ void __launch_bounds__(256)
k_nf4_quantize(const void* __restrict__ W, int64_t nchunks, uint8_t* __restrict__ packed,
               float* __restrict__ absmax, Nf4Tables tb, int* status) {
  __shared__ uint32_t s_base[32];
  __shared__ float s_thr[32];
  if (threadIdx.x < 32) {
    s_base[threadIdx.x] = tb.bucket_base[threadIdx.x];
    s_thr[threadIdx.x] = tb.bucket_thr[threadIdx.x];
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  bool bad = false;

  for (int64_t base = warp * 32; base < nchunks; base += nwarps * 32) {
    const int64_t chunk = base + lane;
    const bool active = chunk < nchunks;      // uniform over each lane pair (nchunks even)
    uint32_t u[32];
    uint32_t m = 0;
    if (active) {
      Loader<T>::load(W, chunk, u);
#pragma unroll
      for (int i = 0; i < 32; ++i) m = max(m, u[i] & 0x7FFFFFFFu);
    }
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    if (!active) continue;
    if (m >= 0x7F800000u) { bad = true; m = 0; }
    const float a = __uint_as_float(m);

    uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      // x = RN32(w / a); an all-zero block has x = 0 everywhere.
      const float w = __uint_as_float(u[i]);
      const float x = (m == 0) ? 0.0f : __fdiv_rn(w, a);
      int b = __float2int_rz(__fmul_rn(__fadd_rn(x, 1.0f), 16.0f));
      b = min(max(b, 0), 31);
      const uint32_t code = s_base[b] + (x >= s_thr[b] ? 1u : 0u);
      // byte j of the 16-byte output holds elements 2j (high) and 2j+1 (low);
      // little-endian: byte j sits at bits 8*(j%4) of word j/4.
      const int byte = i >> 1;
      const int shift = 8 * (byte & 3) + ((i & 1) ? 0 : 4);
      out[byte >> 2] |= code << shift;
    }
    reinterpret_cast<uint4*>(packed)[chunk] = make_uint4(out[0], out[1], out[2], out[3]);
    if ((lane & 1) == 0) absmax[chunk >> 1] = a;
  }
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
}

void launch_quantize(const void* W, int dtype, int64_t n, uint8_t* packed, float* absmax,
                     int* status, cudaStream_t s, int num_sms) {
  const int64_t nchunks = n / 32;
  const int threads = 256;
  int64_t want = (nchunks + threads - 1) / threads;
  int blocks = (int)std::min<int64_t>(want, (int64_t)num_sms * 8);
  blocks = std::max(blocks, 1);
  const Nf4Tables& tb = host_tables();
  if (dtype == QLORA_BF16)
    k_nf4_quantize<__nv_bfloat16><<<blocks, threads, 0, s>>>(W, nchunks, packed, absmax, tb, status);
  else
    k_nf4_quantize<float><<<blocks, threads, 0, s>>>(W, nchunks, packed, absmax, tb, status);
}

// ===========================================================================
// Double quantisation
//   1. exact per-tensor sum of absmax: histogram of 24-bit significands per
//      fp32 exponent (integer adds: exact and order-independent);
//   2. one thread turns the histogram into the correctly rounded fp64 sum and
//      mean = RN32(RN64(sum) / n);
//   3. one warp per group of 256: d = RN32(a - mean), s = max|d|,
//      c = rint(RN32(RN32(d / s) * 127)).
// ===========================================================================

__global__ void __launch_bounds__(256)
k_absmax_hist(const float* __restrict__ absmax, int64_t n, unsigned long long* __restrict__ hist,
              int* status) {
  __shared__ unsigned long long sh[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sh[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  bool bad = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // every lane of a warp runs the same number of iterations (match/reduce
  // below need the full warp)
  const int64_t first = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  for (int64_t base = first; base < n; base += stride) {
    const int64_t i = base + lane;
    uint32_t e = 0xFFFFFFFFu, mant = 0;
    if (i < n) {
      const uint32_t u = __float_as_uint(absmax[i]);
      if (u >= 0x7F800000u) {          // negative (sign set, nonzero) or NaN/Inf
        if (u != 0x80000000u) bad = true;
      } else {
        e = u >> 23;
        mant = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
      }
    }
    const uint32_t grp = __match_any_sync(0xffffffffu, e);
    const uint32_t sum = __reduce_add_sync(grp, mant);       // < 32 * 2^24
    const int leader = __ffs(grp) - 1;
    if (lane == leader && e != 0xFFFFFFFFu && sum)
      atomicAdd(&sh[e], (unsigned long long)sum);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    if (sh[i]) atomicAdd(&hist[i], sh[i]);
  if (bad) set_status(status, QLORA_ERR_NONFINITE);
}

// One thread: exact integer S = sum_e hist[e] * 2^(max(e,1)-1) in units of
// 2^-149 (the value of a float with exponent field e and significand m is
// m * 2^(max(e,1) - 150)); round S to the nearest double (ties to even), then
// mean = RN32(RN64(S * 2^-149) / n).
__global__ void k_mean_finalize(const unsigned long long* __restrict__ hist, int64_t n,
                                float* __restrict__ mean) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  constexpr int L = 12;                  // 384-bit accumulator
  uint32_t acc[L];
  for (int i = 0; i < L; ++i) acc[i] = 0;
  for (int e = 0; e < 255; ++e) {
    unsigned long long v = hist[e];
    if (!v) continue;
    const int sh = (e > 0 ? e : 1) - 1;  // 0..253
    const int w = sh >> 5, b = sh & 31;
    // v << b is a 96-bit number (v < 2^64, b < 32): low 64 bits and the
    // bits shifted out of them
    const unsigned long long lo64 = v << b;
    const unsigned long long hi = b ? (v >> (64 - b)) : 0ull;
    uint64_t carry = 0;
    const uint32_t parts[3] = {(uint32_t)lo64, (uint32_t)(lo64 >> 32), (uint32_t)hi};
    for (int k = 0; k < L - w; ++k) {
      uint64_t t = (uint64_t)acc[w + k] + (k < 3 ? parts[k] : 0u) + carry;
      acc[w + k] = (uint32_t)t;
      carry = t >> 32;
      if (k >= 2 && carry == 0) break;
    }
  }
  int top = -1;
  for (int i = L - 1; i >= 0 && top < 0; --i)
    if (acc[i]) top = 32 * i + 31 - __clz(acc[i]);
  double S;
  if (top < 0) {
    S = 0.0;
  } else if (top <= 52) {
    unsigned long long x = ((unsigned long long)acc[1] << 32) | acc[0];
    S = ldexp((double)x, -149);                        // exact
  } else {
    auto bit = [&](int pos) -> uint32_t { return (acc[pos >> 5] >> (pos & 31)) & 1u; };
    unsigned long long mant = 0;
    for (int pos = top; pos > top - 53; --pos) mant = (mant << 1) | bit(pos);
    const int rpos = top - 53;
    const uint32_t round_bit = bit(rpos);
    uint32_t sticky = 0;
    for (int pos = rpos - 1; pos >= 0 && !sticky; --pos) sticky |= bit(pos);
    if (round_bit && (sticky || (mant & 1ull))) ++mant;
    int expo = top - 52;
    if (mant == (1ull << 53)) { mant >>= 1; ++expo; }
    S = ldexp((double)mant, expo - 149);
  }
  mean[0] = __double2float_rn(__ddiv_rn(S, (double)n));
}

__global__ void __launch_bounds__(256)
k_dq_blockwise(const float* __restrict__ absmax, int64_t n, const float* __restrict__ mean,
               int8_t* __restrict__ qabsmax, float* __restrict__ dq_scale) {
  const int lane = threadIdx.x & 31;
  const int64_t ngroups = (n + 255) / 256;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float mu = mean[0];
  for (int64_t g = warp; g < ngroups; g += nwarps) {
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t i = g * 256 + j * 32 + lane;
      d[j] = (i < n) ? __fsub_rn(absmax[i], mu) : 0.0f;
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

void launch_double_quantize(const float* absmax, int64_t n, int8_t* qabsmax, float* dq_scale,
                            float* dq_mean, unsigned long long* hist, int* status,
                            cudaStream_t s, int num_sms) {
  cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned long long), s);
  int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 4);
  k_absmax_hist<<<std::max(blocks, 1), 256, 0, s>>>(absmax, n, hist, status);
  k_mean_finalize<<<1, 32, 0, s>>>(hist, n, dq_mean);
  const int64_t ngroups = (n + 255) / 256;
  blocks = (int)std::min<int64_t>((ngroups + 7) / 8, (int64_t)num_sms * 8);
  k_dq_blockwise<<<std::max(blocks, 1), 256, 0, s>>>(absmax, n, dq_mean, qabsmax, dq_scale);
}

// ===========================================================================
// Dequantise: one thread owns 32 weights (16 packed bytes -> 64 output bytes).
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
  if (threadIdx.x < 16) s_q[threadIdx.x] = tb.q[threadIdx.x];
  __syncthreads();
  const float mu = DQ ? dq_mean[0] : 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < nchunks;
       chunk += stride) {
    const int64_t blk = chunk >> 1;
    float a;
    if (DQ) {
      const float c = (float)qabsmax[blk];
      a = __fadd_rn(__fmul_rn(__fdiv_rn(c, 127.0f), dq_scale[blk >> 8]), mu);
    } else {
      a = absmax[blk];
    }
    const uint4 pk = __ldcs(reinterpret_cast<const uint4*>(packed) + chunk);
    const uint32_t wds[4] = {pk.x, pk.y, pk.z, pk.w};
    uint32_t o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {            // byte j -> elements 2j (hi), 2j+1 (lo)
      const uint32_t byte = (wds[j >> 2] >> (8 * (j & 3))) & 0xFFu;
      const float v0 = __fmul_rn(s_q[byte >> 4], a);
      const float v1 = __fmul_rn(s_q[byte & 15], a);
      o[j] = pack_bf16x2(v0, v1);
    }
    uint4* dst = out + chunk * 4;
#pragma unroll
    for (int v = 0; v < 4; ++v)
      __stcs(dst + v, make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]));
  }
}

void launch_dequantize(const nf4_weight* w, void* out, cudaStream_t s, int num_sms) {
  const int64_t n = w->rows * w->cols;
  const int64_t nchunks = n / 32;
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
