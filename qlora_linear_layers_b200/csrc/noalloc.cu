// qlora_linear_fwd_noalloc: the QLoRA forward for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace: a plugin loaded into a host
// program that owns every device allocation and hands out only the tensors of
// the call, code running while a stream is being captured into a CUDA graph
// (where cudaMalloc is not allowed), or a real-time loop that forbids any
// allocation after start-up.  This entry point needs no workspace argument:
// its scratch is a fixed array compiled into the library, which every GPU that
// loads the library keeps for the life of the process.
//
// The scratch holds the forward's intermediate s*T tile (and the zero-padded
// B when r < 64); every byte of it that a call reads is written earlier in
// the same call, so nothing needs clearing between calls.

#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/qlora_nf4.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = (size_t)QLORA_FWD_NOALLOC_SCRATCH_BYTES;

// One copy per device, 256-byte aligned (the forward needs 16-byte alignment).
static __device__ __align__(256) uint8_t g_fwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_fwd_scratch on the current device (set up once per
// device; the host-side symbol itself is not a device address).
int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fwd_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return QLORA_OK;
}

}  // namespace

extern "C" int qlora_linear_fwd_noalloc(const nf4_weight* w, const void* X, int64_t M,
                                        const void* A, const void* B, int r, float alpha,
                                        void* Y, void* T_save, qlora_stream_t stream) {
  // the same argument checks, in the same order, as qlora_linear_fwd; only
  // then the size of the fixed scratch
  int st = qnf4::validate_fwd_args(w, X, M, A, B, r, alpha, Y, T_save);
  if (st) return st;
  const size_t need = qlora_workspace_bytes(QLORA_OP_FWD, M, w->rows, w->cols, r);
  if (need > kScratchBytes) return QLORA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st) return st;
  return qlora_linear_fwd(w, X, M, A, B, r, alpha, Y, T_save, scratch, kScratchBytes, stream);
}
