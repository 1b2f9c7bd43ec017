// Arguments and launchers of the tensor-core kernels of the QLoRA layer.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace qnf4 {

// Fused NF4 forward GEMM: Y[M, N] = X deq(W)^T + (s T) B^T.
struct FwdArgs {
  const uint8_t* packed;      // [N, K/2]
  const float* absmax;        // [N*K/64]       (double_quant == 0)
  const int8_t* qabsmax;      // [N*K/64]       (double_quant == 1)
  const float* dq_scale;      // [ceil(N*K/64/256)]
  const float* dq_mean;       // [1]
  __nv_bfloat16* Y;           // [M, N]
  int M, N, K;
  int na;                     // adapter K steps = ceil(r / 64)
  int double_quant;
  int* status;
  float q[16];                // NF4 table
};

int launch_qlora_fwd_gemm(const FwdArgs& a, const void* X, const void* sT, const void* Bpad,
                          int RP, cudaStream_t s, int num_sms);

// 2-D bf16 tensor map, 128-byte swizzle, box [box_outer rows x box_inner cols].
bool make_tmap_2d_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_outer);

// T = X A^T on tensor cores (mma.sync), written as
//   sT_pad[M, RP] = RNbf16(s * T)  (zero for columns >= r)
//   T_save[M, r]  = RNbf16(T)      (if not null)
void launch_lora_down(const void* X, const void* A, int M, int K, int r, int RP, float s,
                      void* sT_pad, void* T_save, cudaStream_t st);

// Bpad[N, RP] = B[N, r] zero-padded to RP columns.
void launch_pad_cols(const void* B, int rows, int r, int RP, void* Bpad, cudaStream_t st);

}  // namespace qnf4
