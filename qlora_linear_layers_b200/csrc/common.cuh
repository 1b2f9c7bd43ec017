// Shared device-side helpers for the sm_100a kernels of libqlora_nf4.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/qlora_nf4.h"

namespace qnf4 {

// ---------------------------------------------------------------------------
// Per-device state block (defined in capi.cu): the sticky status word first,
// then the wait limit every bounded wait uses and one test switch.  Every
// kernel receives the address of the status word (the block's start); the
// first error is kept (atomicCAS from 0); qlora_check_status() reads and
// clears it.
// ---------------------------------------------------------------------------
struct DevState {
  int status;
  int withhold_first_fill;       // test switch: the decode kernel's CTA 0 skips its first stage fill
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void set_status(int* st, int code) {
  atomicCAS(st, 0, code);
}

__device__ __forceinline__ uint64_t wait_limit_ns(const int* st) {
  return *reinterpret_cast<const volatile unsigned long long*>(&reinterpret_cast<const DevState*>(st)->wait_limit_ns);
}

int* device_status_ptr();   // host: address of the status word on the current device

// Raise a kernel's dynamic shared-memory limit once per device: the attribute
// belongs to each device's context, so a process driving several GPUs sets it
// on each.  `done` is the call site's bitmask of devices already set (devices
// 64 and up are set on every call).
template <typename K>
inline void set_smem_attr_once(K kernel, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_relaxed) & bit)) return;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (bit) done.fetch_or(bit, std::memory_order_relaxed);
}

// Host-side launch accounting (capi.cu): count_launches(n) after every
// successful group of n kernel launches.
void count_launches(int n);

// A 4-bit data type's tables, computed on the host and passed to kernels by
// value (they live in the kernel-parameter constant bank).
struct CodeTables {
  float q[16];            // value of each code
  float t[15];            // thresholds between consecutive distinct values, ascending
  int nt;                 // number of thresholds: 15 (NF4), 14 (FP4)
  uint8_t rank_code[16];  // code of the k-th smallest distinct value
  int monotone;           // 1 when code == rank (NF4)
  // Buckets of width 1/16 around the points -1 + b/16: bucket b covers
  // [-1 + (b - 0.5)/16, -1 + (b + 0.5)/16), b = 0..32 (index round(16 x + 16)
  // for x in [-1, 1]); entries 33..63 are unused padding.  At most one
  // threshold falls in a bucket; code(x) = x >= bucket_thr[b] ? bucket_hi[b]
  // : bucket_lo[b] (thr = 2 where no threshold falls).
  float bucket_thr[64];
  uint8_t bucket_lo[64];
  uint8_t bucket_hi[64];
};

// Computed once on the host (table.cu); quant_type is QLORA_QUANT_NF4 or
// QLORA_QUANT_FP4 (anything else: NF4).
const CodeTables& host_tables(int quant_type = QLORA_QUANT_NF4);

// Every pipeline wait gives up after the device state's wait limit (1 s by
// default: far above any legitimate wait, the longest stage hand-off is
// microseconds; qlora_set_wait_limit changes it).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Value of an 8-bit block-scale code, as the entry idx = c + 128 of a 256-entry
// table (c the stored byte read as int8):
//   dq_type 1 (int8):  RN32(c / 127)
//   dq_type 2 (E4M3 byte b = idx ^ 0x80):  e4m3(b) / 256 (exact)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float dq_code_value(int idx, int dq_type) {
  if (dq_type == 2) {
    const uint32_t b = (uint32_t)idx ^ 0x80u;
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    // subnormal m * 2^-9; normal (1 + m/8) * 2^(e - 7): exponent field e + 120
    float v = e == 0 ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    if (e == 15u && m == 7u) v = __int_as_float(0x7fc00000);     // the NaN code (never written)
    v = v * 0x1p-8f;
    return (b & 0x80u) ? -v : v;
  }
  return __fdiv_rn((float)(idx - 128), 127.0f);
}

// ---------------------------------------------------------------------------
// LoRA dropout mask: Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel
// Random Numbers: As Easy as 1, 2, 3", SC 2011) with key (seed, 0) and
// counter (e / 8, 0, 0, 0) for element e = m * K + k of the adapter input;
// element e uses word (e % 8) / 2 of the block, bits 40..63 (e even) or
// 16..39 (e odd), as a 24-bit uniform, kept when >= thr.
// ---------------------------------------------------------------------------
struct Dropout {
  uint64_t seed;
  uint32_t thr;      // floor(p * 2^24 + 1/2); 0 keeps everything
  float scale;       // RN32(1 / RN32(1 - p))
  int on;
};

__device__ __forceinline__ void philox4x64_10(uint64_t& c0, uint64_t& c1, uint64_t& c2, uint64_t& c3,
                                              uint64_t k0, uint64_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B97F4A7C15ull;
      k1 += 0xBB67AE8584CAA73Bull;
    }
    const uint64_t hi0 = __umul64hi(0xD2E7470EE14C6C93ull, c0), lo0 = 0xD2E7470EE14C6C93ull * c0;
    const uint64_t hi1 = __umul64hi(0xCA5A826395121157ull, c2), lo1 = 0xCA5A826395121157ull * c2;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
}

// Keep bits of elements 8 blk .. 8 blk + 7 (bit i: element 8 blk + i).
__device__ __forceinline__ uint32_t dropout_keep8(uint64_t blk, uint64_t seed, uint32_t thr) {
  uint64_t w0 = blk, w1 = 0, w2 = 0, w3 = 0;
  philox4x64_10(w0, w1, w2, w3, seed, 0);
  const uint64_t w[4] = {w0, w1, w2, w3};
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t u = (uint32_t)(w[i >> 1] >> ((i & 1) ? 16 : 40)) & 0xFFFFFFu;
    bits |= (u >= thr ? 1u : 0u) << i;
  }
  return bits;
}

// ---------------------------------------------------------------------------
// Small bit helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// RNbf16 of two fp32 values packed as (lo, hi) halves of a 32-bit word.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Dropout on 8 consecutive bf16 (element i in half i % 2 of word i / 2):
// kept -> RNbf16(RN32(x * scale)), dropped -> 0.
__device__ __forceinline__ uint4 dropout8(uint4 v, uint32_t bits, float scale) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t pk = pack_bf16x2(__fmul_rn(bf16_lo(w[j]), scale), __fmul_rn(bf16_hi(w[j]), scale));
    const uint32_t keep = ((bits >> (2 * j)) & 1u ? 0x0000FFFFu : 0u) | ((bits >> (2 * j + 1)) & 1u ? 0xFFFF0000u : 0u);
    w[j] = pk & keep;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// The first 1024-byte-aligned address at or after a dynamic shared array,
// reached by offsetting the array itself so the compiler keeps shared-space
// (32-bit) addressing for everything derived from it.
template <typename T>
__device__ __forceinline__ T* smem_align1024(uint8_t* raw) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(raw));
  return reinterpret_cast<T*>(raw + ((1024u - (a & 1023u)) & 1023u));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and records QLORA_ERR_TIMEOUT) if the phase
// does not complete within the wait limit.  `abort` is a CTA-shared flag: once
// any waiter gives up, the others stop waiting too.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort, int* st) {
  // The clock and the limit (a global load) are read only once the wait has
  // lasted 256 tries: a wait that ends soon costs no memory round trip.
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > wait_limit_ns(st)) break;
    }
  }
  *abort = 1;
  set_status(st, QLORA_ERR_TIMEOUT);
  return false;
}

// ---------------------------------------------------------------------------
// TMA (tiled, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :: "r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (Blackwell tensor cores, tensor memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T   (kind::f16, one CTA)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T   (kind::f16, one CTA)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive (once) on an mbarrier when all prior tcgen05 ops of this thread finish.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Warp-wide: thread t writes 16 consecutive 32-bit columns of TMEM lane
// (lane base of taddr) + t.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
         "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]),
         "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Warp-wide: thread t reads 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters and the paired-SM (cta_group::2) forms
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
  return d;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by a shared::cluster address (possibly in the
// peer CTA), with the instruction's default semantics.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" :: "r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait on a barrier that the peer CTA also signals.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, int* st) {
  uint64_t t0 = 0;                               // read late, as in mbar_wait
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > wait_limit_ns(st)) break;
    }
  }
  *abort = 1;
  set_status(st, QLORA_ERR_TIMEOUT);
  return false;
}

// Tiled TMA load into this CTA's shared memory whose completion is counted
// on an mbarrier of either CTA of the pair (shared::cluster address).  No
// multicast: each CTA loads its own half.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, uint32_t mbar_cluster,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(smem_dst)), "l"(tmap), "r"(mbar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
               :: "r"(taddr), "r"(ncols) : "memory");
}

// Paired-SM MMA, issued by the even CTA: D (128 rows in each CTA's TMEM) (+)=
// A (each CTA's 128 rows, from its TMEM) * B^T (each CTA's half of the N
// columns, from its shared memory at the same offset).
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Paired-SM MMA with both operands in shared memory (A split by rows, B by
// columns across the pair, same offsets in both CTAs).
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive once on the mbarrier at this offset in every CTA of `cta_mask` when
// all prior tcgen05 ops of this thread are complete.
__device__ __forceinline__ void mma_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      :: "r"(smem_u32(bar)), "h"(cta_mask) : "memory");
}

// Shared-memory matrix descriptor for a K-major, 128-byte-swizzled bf16 tile
// whose rows are 128 bytes (64 elements) and whose 8-row groups are 1024 bytes
// apart (the layout a TMA load with SWIZZLE_128B writes).  Base must be
// 1024-byte aligned; advancing K by 16 elements adds 32 bytes to the start.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);        // start address
  d |= (uint64_t)1u << 16;                            // leading byte offset (unused, 16 B)
  d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset: 8-row group
  d |= (uint64_t)1u << 46;                            // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                            // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                       // D format fp32
       | (1u << 7)                       // A format bf16
       | (1u << 10)                      // B format bf16
       | ((uint32_t)(N >> 3) << 17)      // N / 8
       | ((uint32_t)(M >> 4) << 24);     // M / 16
}

}  // namespace qnf4
