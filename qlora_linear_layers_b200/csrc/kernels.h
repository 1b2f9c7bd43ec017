// Launchers shared between the C-ABI layer (capi.cu) and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qlora_nf4.h"

namespace qnf4 {

// Returns the number of launches (the histogram zeroing counts as one).
// `hist` (256 u64, or null): zeroed, then filled with the exponent
// histogram of the block absmax values.
int launch_quantize(const void* W, int dtype, int64_t n, int quant_type, uint8_t* packed,
                    float* absmax, unsigned long long* hist, int* status, cudaStream_t s,
                    int num_sms);

// Double quantisation of an absmax array (histogram + finalise); returns the
// number of launches.
int launch_double_quantize(const float* absmax, int64_t n, int8_t* qabsmax, float* dq_scale,
                           float* dq_mean, unsigned long long* hist, int* status, cudaStream_t s,
                           int num_sms);

// Finalise from a complete histogram over n_total absmax values; returns the
// number of launches.
int launch_double_quantize_from_hist(const float* absmax, int64_t n, const unsigned long long* hist,
                                     int64_t n_total, int8_t* qabsmax, float* dq_scale, float* dq_mean,
                                     cudaStream_t s, int num_sms, int dq_type);

void launch_dequantize(const nf4_weight* w, void* out, cudaStream_t s, int num_sms);

// W_merged = RNbf16(deq(W) + s B A), [rows, cols] bf16 (merge.cu).
void launch_merge(const nf4_weight* w, const void* A, const void* B, int r, float s, void* out,
                  cudaStream_t st);

// All argument checks of qlora_linear_fwd except the workspace (capi.cu).
int validate_fwd_args(const nf4_weight* w, const void* X, int64_t M, const void* A, const void* B,
                      int r, float alpha, const void* Y, const void* T_save);

}  // namespace qnf4
