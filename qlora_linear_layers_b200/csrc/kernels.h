// Launchers shared between the C-ABI layer (capi.cu) and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qlora_nf4.h"

namespace qnf4 {

void launch_quantize(const void* W, int dtype, int64_t n, uint8_t* packed, float* absmax,
                     int* status, cudaStream_t s, int num_sms);

// One cooperative kernel; returns the kernels launched (1), -1 if refused.
int launch_double_quantize(const float* absmax, int64_t n, int8_t* qabsmax, float* dq_scale,
                            float* dq_mean, unsigned long long* hist, int* status,
                            cudaStream_t s, int num_sms);

void launch_dequantize(const nf4_weight* w, void* out, cudaStream_t s, int num_sms);

// All argument checks of qlora_linear_fwd except the workspace (capi.cu).
int validate_fwd_args(const nf4_weight* w, const void* X, int64_t M, const void* A, const void* B,
                      int r, float alpha, const void* Y, const void* T_save);

}  // namespace qnf4
