// Arguments and launchers of the tensor-core kernels of the QLoRA layer.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/qlora_nf4.h"

namespace qnf4 {

constexpr int MODE_NF4 = 0;    // weight side dequantised from NF4 into TMEM
constexpr int MODE_BF16 = 1;   // weight side is a bf16 matrix loaded by TMA

// out[Mtok, Nout] = tok[Mtok, Kc] Wt[Nout, Kc]^T + tokad[Mtok, RP] Wad[Nout, RP]^T
struct GemmArgs {
  // MODE_NF4 weight (Wt = deq(W), W is [Nout, Kc])
  const uint8_t* packed;      // [Nout, Kc/2]
  const float* absmax;        // [Nout*Kc/64]     (double_quant == 0)
  const int8_t* qabsmax;      // [Nout*Kc/64]     (double_quant == 1)
  const float* dq_scale;      // [ceil(Nout*Kc/64/256)]
  const float* dq_mean;       // [1]
  const __nv_bfloat16* wad;   // [Nout, RP] adapter weight factor (MODE_NF4 reads it directly)
  int RP;                     // adapter width padded to a multiple of 64
  __nv_bfloat16* out;         // [Mtok, Nout]
  int Mtok, Nout, Kc;
  int na;                     // adapter K steps = RP / 64
  int double_quant;
  int* status;
  float q[16];                // NF4 table
};

// Backward dX GEMM on SM pairs (cluster of 2, tcgen05 cta_group::2): 256 x BM
// output tiles; tok: [Mtok, Kc]; tokad: [Mtok, RP]; weights w [Nout, Kc] and
// wad [Nout, RP] bf16.
int launch_qlora_gemm_pair(const GemmArgs& a, const void* tok, const void* tokad, const void* wad,
                           const void* w, int RP, cudaStream_t s, int num_sms);

// Forward NF4 GEMM on SM pairs with two token tiles per weight tile (the
// weights of a stage are dequantised once into shared memory and feed two
// 256-row x BM MMAs).  tok: [Mtok, Kc]; tokad: [Mtok, RP]; weights from `a`.
int launch_qlora_gemm_dual(const GemmArgs& a, const void* tok, const void* tokad, int RP,
                           cudaStream_t s, int num_sms);

// tok: [Mtok, Kc]; tokad: [Mtok, RP]; wad: [Nout, RP]; w: [Nout, Kc] (MODE_BF16 only).
int launch_qlora_gemm(int mode, const GemmArgs& a, const void* tok, const void* tokad,
                      const void* wad, const void* w, int RP, cudaStream_t s, int num_sms);

// Decode-sized forward (M <= 16): Y = X deq(W)^T + s (X A^T) B^T, T_save =
// RNbf16(X A^T) when not null.  `part` holds gemv_workspace_bytes(M, N, K, r)
// bytes.  Returns the number of kernels launched, or -1 when the tensor map
// of the codes cannot be built.  Waits that give up set QLORA_ERR_TIMEOUT in
// `status`.
constexpr int kDecodeMaxTokens = 16;
int launch_qlora_gemv(const nf4_weight* w, const void* X, int M, const void* A, const void* B,
                      int r, float s, void* Y, void* T_save, float* part, const float* q,
                      int* status, cudaStream_t st, int num_sms);
size_t gemv_workspace_bytes(int M, int N, int K, int r);

// 2-D bf16 tensor map, 128-byte swizzle, box [box_outer rows x box_inner cols].
bool make_tmap_2d_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_outer);
// Same for a uint8 matrix: inner extent and row stride in bytes; 128-byte
// swizzle (box_inner <= 128) or none.
bool make_tmap_2d_u8(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);
// 3-D tiled map (uint8 or bf16): extents (innermost first), strides of
// dimensions 1 and 2 in bytes (multiples of 16), box extents.
bool make_tmap_3d(CUtensorMap* tm, const void* base, bool bf16, const uint64_t dims[3],
                  const uint64_t strides_bytes[2], const uint32_t box[3], bool swizzle128);

// T = X A^T on tensor cores (mma.sync), written as
//   sT_pad[M, RP] = RNbf16(s * T)  (zero for columns >= r; may be null)
//   T_save[M, r]  = RNbf16(T)      (if not null)
// `part` holds skinny_workspace_bytes(M, K, RP) bytes of fp32 partial sums.
// Returns the number of kernels launched.
struct Dropout;
// With `drop` (LoRA dropout on X, may be null), T = X' A^T with X' the
// dropped-out input.
int launch_lora_down(const void* X, const void* A, int M, int K, int r, int RP, float s,
                     void* sT_pad, void* T_save, float* part, cudaStream_t st,
                     const Dropout* drop = nullptr);
size_t skinny_workspace_bytes(int M, int L, int RP);

// U = dY B:  sU_pad[M, RP] = RNbf16(s * U), zero beyond r.
int launch_lora_u(const void* dY, const void* B, int M, int N, int r, int RP, float s,
                  void* sU_pad, float* part, cudaStream_t st);

// C[Rdim, Cdim] = RNbf16(s * P^T Q) over M token rows, split over the tokens
// into fixed chunks summed in order; `part` holds atb_workspace_floats floats.
// With `dropq`, Q (the adapter input X) is dropped out on load.
void launch_atb(const void* P, int ldp, int Rdim, const void* Q, int ldq, int Cdim, int M, float s,
                void* out, float* part, int num_sms, cudaStream_t st, const Dropout* dropq = nullptr);

// Y[M, K] (bf16, in place) += D * c * (Bm[M, :r] A[r, K]) with D the dropout
// keep mask of Y's elements (drop.on == 0: no mask, c = 1): the adapter term
// of dX under LoRA dropout.
void launch_rank_add(const void* Bm, int ldb, const void* A, int r, int M, int K, void* Y,
                     const Dropout& drop, cudaStream_t st);
size_t atb_workspace_floats(int Rdim, int Cdim, int M);

// Wt[K, N] = deq(W)^T (bf16, the values of nf4_dequantize).
void launch_dequant_t(const nf4_weight* w, void* Wt, cudaStream_t st);

// At[K, RP] = A[r, K]^T zero-padded to RP columns.
void launch_transpose_pad(const void* A, int r, int K, int RP, void* At, cudaStream_t st);

// Bpad[N, RP] = B[N, r] zero-padded to RP columns.
void launch_pad_cols(const void* B, int rows, int r, int RP, void* Bpad, cudaStream_t st);

}  // namespace qnf4
