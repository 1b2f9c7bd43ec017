// C ABI of libqlora_nf4.so: argument validation, workspace sizing, dispatch
// to the sm_100a kernels, and the sticky device status word.

#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <mutex>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "gemm.h"

namespace qnf4 {

// One state block per device (each device context has its own copy): the
// status word, the test switch and the wait limit.
static __device__ DevState g_state = {0, 0, kWaitLimitNs};

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int major = 0, minor = 0;
  int* status = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

// Returns QLORA_OK and fills `info` for the current device, or an error if
// there is no usable sm_100 device.
int current_device(DeviceInfo** info) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) { cudaGetLastError(); return QLORA_ERR_CUDA; }
    d.sms = p.multiProcessorCount;
    d.major = p.major;
    d.minor = p.minor;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_state) != cudaSuccess) { cudaGetLastError(); return QLORA_ERR_CUDA; }
    d.status = &static_cast<DevState*>(ptr)->status;
    d.ready = true;
  }
  if (d.major != 10) return QLORA_ERR_UNSUPPORTED;   // sm_100 family only
  *info = &d;
  return QLORA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool valid_rank(int r) { return r == 8 || r == 16 || r == 32 || r == 64 || r == 128; }

int padded_rank(int r) { return r <= 64 ? 64 : 128; }

// Forward workspace: sT_pad [M, RP] bf16, Bpad [N, RP] bf16 when r < RP,
// then the fp32 partial sums of T = X A^T.
struct FwdWs {
  size_t sT, Bpad, part, gemv, total;
};
FwdWs fwd_ws(int64_t M, int64_t N, int64_t K, int r, bool gemm_path = false) {
  FwdWs w{};
  const int RP = padded_rank(r);
  size_t off = 0;
  if (M <= kDecodeMaxTokens && !gemm_path) {   // decode path: only the GEMV's partial sums
    w.gemv = 0;
    w.total = align256(gemv_workspace_bytes((int)M, (int)N, (int)K, r));
    return w;
  }
  w.sT = off;   off += align256((size_t)M * RP * 2);
  w.Bpad = off; off += (r < RP ? align256((size_t)N * RP * 2) : 0);
  w.part = off; off += align256(skinny_workspace_bytes((int)M, (int)K, RP));
  w.total = off;
  return w;
}

// Backward workspace, in order: T [M, r] (recomputed when not passed),
// sU [M, RP], Wt = deq(W)^T [K, N], At = A^T [K, RP] (all bf16), then the
// fp32 split-M partial sums of dA and dB.
struct BwdWs {
  size_t T, sU, Wt, At, pA, pB, pT, pU, total;
};
BwdWs bwd_ws(int64_t M, int64_t N, int64_t K, int r) {
  BwdWs w{};
  const int RP = padded_rank(r);
  size_t off = 0;
  w.T = off;  off += align256((size_t)M * r * 2);
  w.sU = off; off += align256((size_t)M * RP * 2);
  w.Wt = off; off += align256((size_t)K * N * 2);
  w.At = off; off += align256((size_t)K * RP * 2);
  w.pA = off; off += align256(atb_workspace_floats(r, (int)K, (int)M) * 4);
  w.pB = off; off += align256(atb_workspace_floats((int)N, r, (int)M) * 4);
  w.pT = off; off += align256(skinny_workspace_bytes((int)M, (int)K, RP));
  w.pU = off; off += align256(skinny_workspace_bytes((int)M, (int)N, RP));
  w.total = off;
  return w;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int check_weight(const nf4_weight* w) {
  if (!w || !w->packed) return QLORA_ERR_INVALID_ARG;
  if (w->blocksize != 64) return QLORA_ERR_UNSUPPORTED;
  if (w->quant_type != QLORA_QUANT_NF4 && w->quant_type != QLORA_QUANT_FP4) return QLORA_ERR_INVALID_ARG;
  if (w->rows < 1 || w->cols < 64 || w->cols % 64) return QLORA_ERR_SHAPE;
  if (!aligned16(w->packed)) return QLORA_ERR_ALIGN;
  if (w->double_quant < 0 || w->double_quant > 2) return QLORA_ERR_INVALID_ARG;
  if (w->double_quant) {
    if (w->dq_blocksize != 256) return QLORA_ERR_UNSUPPORTED;
    if (!w->qabsmax || !w->dq_scale || !w->dq_mean) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(w->qabsmax) || !aligned16(w->dq_scale) || !aligned16(w->dq_mean))
      return QLORA_ERR_ALIGN;
  } else {
    if (!w->absmax) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(w->absmax)) return QLORA_ERR_ALIGN;
  }
  return QLORA_OK;
}

}  // namespace

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static std::mutex g_ev_mu;
static cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;

// Take (and clear) a pending event registration.
static void take_gemm_events(cudaEvent_t* a, cudaEvent_t* b) {
  std::lock_guard<std::mutex> lk(g_ev_mu);
  *a = g_ev_start; *b = g_ev_stop;
  g_ev_start = g_ev_stop = nullptr;
}

// Every check of qlora_linear_fwd's arguments except the workspace, in the
// order that entry point applies them.
int validate_fwd_args(const nf4_weight* w, const void* X, int64_t M, const void* A, const void* B,
                      int r, float alpha, const void* Y, const void* T_save) {
  int st = check_weight(w);
  if (st) return st;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if (!valid_rank(r) || !(alpha == alpha) || alpha > 3.0e38f || alpha < -3.0e38f) return QLORA_ERR_INVALID_ARG;
  const int64_t N = w->rows, K = w->cols;
  if (M < 1 || N % 8 || M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) ||
      (T_save && !aligned16(T_save)))
    return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

int* device_status_ptr() {
  DeviceInfo* d = nullptr;
  return current_device(&d) == QLORA_OK ? d->status : nullptr;
}

}  // namespace qnf4

using namespace qnf4;

extern "C" {

int qlora_abi_version(void) { return 200; }

uint64_t qlora_kernel_launches(void) { return g_launches.load(); }

int qlora_profile_gemm_events(void* start, void* stop) {
  if ((start == nullptr) != (stop == nullptr)) return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_ev_mu);
  g_ev_start = static_cast<cudaEvent_t>(start);
  g_ev_stop = static_cast<cudaEvent_t>(stop);
  return QLORA_OK;
}

const char* qlora_status_string(int s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_SHAPE: return "shape violates a constraint";
    case QLORA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QLORA_ERR_NONFINITE: return "non-finite value met on the device";
    case QLORA_ERR_TIMEOUT: return "a bounded device wait gave up";
    case QLORA_ERR_CUDA: return "CUDA call failed";
    case QLORA_ERR_UNSUPPORTED: return "unsupported device or mode";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int nf4_code_table(float* table16) {
  if (!table16) return QLORA_ERR_INVALID_ARG;
  std::memcpy(table16, host_tables().q, 16 * sizeof(float));
  return QLORA_OK;
}

int nf4_code_thresholds(float* thresholds15) {
  if (!thresholds15) return QLORA_ERR_INVALID_ARG;
  std::memcpy(thresholds15, host_tables().t, 15 * sizeof(float));
  return QLORA_OK;
}

int qlora_code_table(int quant_type, float* table16) {
  if (!table16 || (quant_type != QLORA_QUANT_NF4 && quant_type != QLORA_QUANT_FP4))
    return QLORA_ERR_INVALID_ARG;
  std::memcpy(table16, host_tables(quant_type).q, 16 * sizeof(float));
  return QLORA_OK;
}

int qlora_code_thresholds(int quant_type, float* thresholds15, int* count) {
  if (!thresholds15 || !count || (quant_type != QLORA_QUANT_NF4 && quant_type != QLORA_QUANT_FP4))
    return QLORA_ERR_INVALID_ARG;
  const CodeTables& tb = host_tables(quant_type);
  std::memcpy(thresholds15, tb.t, (size_t)tb.nt * sizeof(float));
  *count = tb.nt;
  return QLORA_OK;
}

// Host restatement of the device's exact mean: S = sum_e hist[e] *
// 2^(max(e,1)-1) in units of 2^-149 as a 384-bit integer, rounded to the
// nearest double (ties to even), divided by n in double, rounded to float.
int qlora_dq_mean_from_hist(const int64_t* hist, int64_t n_total, float* mean) {
  if (!hist || !mean || n_total < 1) return QLORA_ERR_INVALID_ARG;
  constexpr int L = 13;                                   // 416 bits, little-endian words
  uint32_t acc[L] = {};
  for (int e = 0; e < 255; ++e) {
    if (hist[e] < 0) return QLORA_ERR_INVALID_ARG;
    if (hist[e] == 0) continue;
    const int sh = (e > 0 ? e : 1) - 1;
    const int w0 = sh >> 5, b = sh & 31;
    // hist[e] << b spans at most three words
    const unsigned __int128 v = (unsigned __int128)(uint64_t)hist[e] << b;
    uint64_t carry = 0;
    for (int k = 0; k < L - w0; ++k) {
      const uint64_t add = k < 4 ? (uint64_t)(uint32_t)(v >> (32 * k)) : 0;
      const uint64_t t = (uint64_t)acc[w0 + k] + add + carry;
      acc[w0 + k] = (uint32_t)t;
      carry = t >> 32;
      if (k >= 3 && carry == 0) break;
    }
  }
  int top = -1;
  for (int w = L - 1; w >= 0 && top < 0; --w)
    if (acc[w]) top = 32 * w + 31 - __builtin_clz(acc[w]);
  auto bit = [&](int i) -> uint64_t { return (i >= 0 && i < 32 * L) ? (acc[i >> 5] >> (i & 31)) & 1u : 0u; };
  double S = 0.0;
  if (top >= 0) {
    const int lo = top > 52 ? top - 52 : 0;               // the 53-bit significand is bits [lo, top]
    uint64_t mant = 0;
    for (int i = top; i >= lo; --i) mant = (mant << 1) | bit(i);
    if (lo > 0) {
      const uint64_t rbit = bit(lo - 1);
      bool sticky = false;
      for (int i = 0; i < lo - 1 && !sticky; ++i) sticky = bit(i) != 0;
      if (rbit && (sticky || (mant & 1))) ++mant;
    }
    S = std::ldexp((double)mant, lo - 149);               // exact: mant <= 2^53
  }
  *mean = (float)(S / (double)n_total);
  return QLORA_OK;
}

size_t qlora_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r) {
  (void)K;
  switch (op) {
    case QLORA_OP_DOUBLE_QUANT: return QLORA_DQ_HIST_BYTES;
    case QLORA_OP_FWD:
      if (M < 1 || N < 1 || !valid_rank(r)) return 0;
      if (K < 1) return 0;
      return fwd_ws(M, N, K, r).total;
    case QLORA_OP_BWD:
    case QLORA_OP_BWD_DROPOUT:
      if (M < 1 || N < 1 || K < 1 || !valid_rank(r)) return 0;
      return bwd_ws(M, N, K, r).total;
    case QLORA_OP_FWD_DROPOUT:
      if (M < 1 || N < 1 || K < 1 || !valid_rank(r)) return 0;
      return fwd_ws(M, N, K, r, true).total;
    default: return 0;
  }
}

int qlora_quantize_4bit(const void* W, int dtype, int64_t rows, int64_t cols, int blocksize,
                        int quant_type, uint8_t* packed, float* absmax, int64_t* dq_hist,
                        qlora_stream_t stream) {
  if (!W || !packed || !absmax) return QLORA_ERR_INVALID_ARG;
  if (dtype != QLORA_F32 && dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (quant_type != QLORA_QUANT_NF4 && quant_type != QLORA_QUANT_FP4) return QLORA_ERR_INVALID_ARG;
  if (blocksize != 64) return QLORA_ERR_UNSUPPORTED;
  if (rows < 1 || cols < 64 || cols % 64 || rows > ((int64_t)1 << 40) / cols) return QLORA_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(absmax) || (dq_hist && !aligned16(dq_hist)))
    return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  int st = current_device(&d);
  if (st) return st;
  const int n = launch_quantize(W, dtype, rows * cols, quant_type, packed, absmax,
                                reinterpret_cast<unsigned long long*>(dq_hist), d->status,
                                (cudaStream_t)stream, d->sms);
  st = launch_status();
  if (!st) count_launches(n);
  return st;
}

int nf4_quantize(const void* W, int dtype, int64_t rows, int64_t cols, int blocksize,
                 uint8_t* packed, float* absmax, qlora_stream_t stream) {
  return qlora_quantize_4bit(W, dtype, rows, cols, blocksize, QLORA_QUANT_NF4, packed, absmax,
                             nullptr, stream);
}

int nf4_double_quantize(const float* absmax, int64_t n_absmax, int dq_blocksize, int8_t* qabsmax,
                        float* dq_scale, float* dq_mean, void* ws, size_t ws_bytes,
                        qlora_stream_t stream) {
  if (!absmax || !qabsmax || !dq_scale || !dq_mean) return QLORA_ERR_INVALID_ARG;
  if (dq_blocksize != 256) return QLORA_ERR_UNSUPPORTED;
  if (n_absmax < 1) return QLORA_ERR_SHAPE;
  if (!ws || ws_bytes < qlora_workspace_bytes(QLORA_OP_DOUBLE_QUANT, 0, n_absmax, 0, 0))
    return QLORA_ERR_WORKSPACE;
  if (!aligned16(absmax) || !aligned16(qabsmax) || !aligned16(dq_scale) || !aligned16(dq_mean) ||
      !aligned16(ws))
    return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  int st = current_device(&d);
  if (st) return st;
  const int n = launch_double_quantize(absmax, n_absmax, qabsmax, dq_scale, dq_mean,
                                       static_cast<unsigned long long*>(ws), d->status,
                                       (cudaStream_t)stream, d->sms);
  st = launch_status();
  if (!st) count_launches(n);
  return st;
}

int nf4_double_quantize_hist(const float* absmax, int64_t n_absmax, const int64_t* dq_hist,
                             int64_t n_total, int dq_blocksize, int8_t* qabsmax, float* dq_scale,
                             float* dq_mean, qlora_stream_t stream) {
  return qlora_double_quantize_hist(absmax, n_absmax, dq_hist, n_total, dq_blocksize, QLORA_DQ_INT8,
                                    qabsmax, dq_scale, dq_mean, stream);
}

int qlora_double_quantize_hist(const float* absmax, int64_t n_absmax, const int64_t* dq_hist,
                               int64_t n_total, int dq_blocksize, int dq_type, int8_t* qabsmax,
                               float* dq_scale, float* dq_mean, qlora_stream_t stream) {
  if (!absmax || !dq_hist || !qabsmax || !dq_scale || !dq_mean) return QLORA_ERR_INVALID_ARG;
  if (dq_type != QLORA_DQ_INT8 && dq_type != QLORA_DQ_FP8) return QLORA_ERR_INVALID_ARG;
  if (dq_blocksize != 256) return QLORA_ERR_UNSUPPORTED;
  if (n_absmax < 1 || n_total < n_absmax || n_total > ((int64_t)1 << 39)) return QLORA_ERR_SHAPE;
  if (!aligned16(absmax) || !aligned16(dq_hist) || !aligned16(qabsmax) || !aligned16(dq_scale) ||
      !aligned16(dq_mean))
    return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  int st = current_device(&d);
  if (st) return st;
  const int n = launch_double_quantize_from_hist(absmax, n_absmax,
                                                 reinterpret_cast<const unsigned long long*>(dq_hist),
                                                 n_total, qabsmax, dq_scale, dq_mean,
                                                 (cudaStream_t)stream, d->sms, dq_type);
  st = launch_status();
  if (!st) count_launches(n);
  return st;
}

int nf4_dequantize(const nf4_weight* w, void* W_out, qlora_stream_t stream) {
  int st = check_weight(w);
  if (st) return st;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st) return st;
  launch_dequantize(w, W_out, (cudaStream_t)stream, d->sms);
  st = launch_status();
  if (!st) count_launches(1);
  return st;
}

int qlora_merge(const nf4_weight* w, const void* A, const void* B, int r, float alpha, void* W_out,
                qlora_stream_t stream) {
  int st = check_weight(w);
  if (st) return st;
  if (!A || !B || !W_out) return QLORA_ERR_INVALID_ARG;
  if (!valid_rank(r) || !(alpha == alpha) || alpha > 3.0e38f || alpha < -3.0e38f) return QLORA_ERR_INVALID_ARG;
  if (w->rows > (1 << 30) || w->cols > (1 << 30)) return QLORA_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(B) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st) return st;
  launch_merge(w, A, B, r, alpha / (float)r, W_out, (cudaStream_t)stream);
  st = launch_status();
  if (!st) count_launches(1);
  return st;
}

static int fwd_impl(const nf4_weight* w, const void* X, int64_t M, const void* A, const void* B,
                    int r, float alpha, const Dropout* drop, void* Y, void* T_save, void* ws,
                    size_t ws_bytes, qlora_stream_t stream) {
  int st = validate_fwd_args(w, X, M, A, B, r, alpha, Y, T_save);
  if (st) return st;
  const int64_t N = w->rows, K = w->cols;
  // dropout applies to the adapter's input only: the decode kernel, which
  // reads X once for both, is left to the plain layer
  const bool gemm_path = drop != nullptr;
  const FwdWs lay = fwd_ws(M, N, K, r, gemm_path);
  if (!ws || ws_bytes < lay.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int RP = padded_rank(r);
  const float scale = alpha / (float)r;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  if (M <= kDecodeMaxTokens && !gemm_path) {
    // decode-sized call: HBM-bound GEMV on the warp-level tensor cores
    const int n = launch_qlora_gemv(w, X, (int)M, A, B, r, scale, Y, T_save,
                                    reinterpret_cast<float*>(wsb + lay.gemv), host_tables(w->quant_type).q,
                                    d->status, s, d->sms);
    if (n < 0) return QLORA_ERR_CUDA;
    st = launch_status();
    if (!st) count_launches(n);
    return st;
  }
  void* sT = wsb + lay.sT;
  const void* Bp = B;
  int n = 1;
  if (r < RP) {
    launch_pad_cols(B, (int)N, r, RP, wsb + lay.Bpad, s);
    Bp = wsb + lay.Bpad;
    ++n;
  }
  n += launch_lora_down(X, A, (int)M, (int)K, r, RP, scale, sT, T_save,
                        reinterpret_cast<float*>(wsb + lay.part), s, drop);
  GemmArgs a{};
  a.packed = w->packed;
  a.absmax = w->absmax;
  a.qabsmax = w->qabsmax;
  a.dq_scale = w->dq_scale;
  a.dq_mean = w->dq_mean;
  a.out = static_cast<__nv_bfloat16*>(Y);
  a.wad = static_cast<const __nv_bfloat16*>(Bp);
  a.RP = RP;
  a.Mtok = (int)M; a.Nout = (int)N; a.Kc = (int)K;
  a.na = RP / 64;
  a.double_quant = w->double_quant;
  a.status = d->status;
  for (int i = 0; i < 16; ++i) a.q[i] = host_tables(w->quant_type).q[i];
  cudaEvent_t e0, e1;
  take_gemm_events(&e0, &e1);
  if (e0) cudaEventRecord(e0, s);
  // paired-SM tiles (256 weight rows, two token tiles each) once there is
  // more than one 128-row block
  st = N > 128 ? launch_qlora_gemm_dual(a, X, sT, RP, s, d->sms)
               : launch_qlora_gemm(MODE_NF4, a, X, sT, Bp, nullptr, RP, s, d->sms);
  if (e1) cudaEventRecord(e1, s);
  if (st) return st;
  st = launch_status();
  if (!st) count_launches(n);
  return st;
}

static int bwd_impl(const nf4_weight* w, const void* X, const void* dY, int64_t M, const void* A,
                    const void* B, int r, float alpha, const Dropout* drop, const void* T, void* dX,
                    void* dA, void* dB, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  int st = check_weight(w);
  if (st) return st;
  if (!X || !dY || !A || !B || !dX || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!valid_rank(r) || !(alpha == alpha) || alpha > 3.0e38f || alpha < -3.0e38f) return QLORA_ERR_INVALID_ARG;
  const int64_t N = w->rows, K = w->cols;
  if (M < 1 || N % 8 || M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(A) || !aligned16(B) || !aligned16(dX) ||
      !aligned16(dA) || !aligned16(dB) || (T && !aligned16(T)))
    return QLORA_ERR_ALIGN;
  const BwdWs lay = bwd_ws(M, N, K, r);
  if (!ws || ws_bytes < lay.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int RP = padded_rank(r);
  const float scale = alpha / (float)r;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  void* Tw = wsb + lay.T;
  void* sU = wsb + lay.sU;
  void* Wt = wsb + lay.Wt;
  void* At = wsb + lay.At;
  int n = 7;   // dequant_t, transpose_pad, GEMM, 2 x (partials + reduce)
  if (!T) {
    n += launch_lora_down(X, A, (int)M, (int)K, r, RP, scale, nullptr, Tw,
                          reinterpret_cast<float*>(wsb + lay.pT), s, drop);
    T = Tw;
  }
  n += launch_lora_u(dY, B, (int)M, (int)N, r, RP, scale, sU, reinterpret_cast<float*>(wsb + lay.pU), s);
  launch_dequant_t(w, Wt, s);
  launch_transpose_pad(A, r, (int)K, RP, At, s);
  // dX[M, K] = dY Wt^T + sU At^T   (tokens = dY rows, outputs = K, contraction = N)
  GemmArgs a{};
  a.out = static_cast<__nv_bfloat16*>(dX);
  a.wad = static_cast<const __nv_bfloat16*>(At);
  a.RP = RP;
  a.Mtok = (int)M; a.Nout = (int)K; a.Kc = (int)N;
  // with dropout the adapter term needs the keep mask: the GEMM writes dY W'
  // alone and a rank-r pass adds D * c * (s U A)
  const bool dropping = drop && drop->on;
  a.na = dropping ? 0 : RP / 64;
  a.status = d->status;
  cudaEvent_t e0, e1;
  take_gemm_events(&e0, &e1);
  if (e0) cudaEventRecord(e0, s);
  st = K > 128 ? launch_qlora_gemm_pair(a, dY, sU, At, Wt, RP, s, d->sms)
               : launch_qlora_gemm(MODE_BF16, a, dY, sU, At, Wt, RP, s, d->sms);
  if (e1) cudaEventRecord(e1, s);
  if (st) return st;
  if (dropping) {
    launch_rank_add(sU, RP, A, r, (int)M, (int)K, dX, *drop, s);
    ++n;
  }
  // dA[r, K] = (s U)^T X ;  dB[N, r] = s dY^T T
  launch_atb(sU, RP, r, X, (int)K, (int)K, (int)M, 1.0f, dA, reinterpret_cast<float*>(wsb + lay.pA),
             d->sms, s, drop);
  launch_atb(dY, (int)N, (int)N, T, r, r, (int)M, scale, dB, reinterpret_cast<float*>(wsb + lay.pB),
             d->sms, s);
  st = launch_status();
  if (!st) count_launches(n);
  return st;
}

int qlora_linear_fwd(const nf4_weight* w, const void* X, int64_t M, const void* A, const void* B,
                     int r, float alpha, void* Y, void* T_save, void* ws, size_t ws_bytes,
                     qlora_stream_t stream) {
  return fwd_impl(w, X, M, A, B, r, alpha, nullptr, Y, T_save, ws, ws_bytes, stream);
}

int qlora_linear_bwd(const nf4_weight* w, const void* X, const void* dY, int64_t M, const void* A,
                     const void* B, int r, float alpha, const void* T, void* dX, void* dA,
                     void* dB, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  return bwd_impl(w, X, dY, M, A, B, r, alpha, nullptr, T, dX, dA, dB, ws, ws_bytes, stream);
}

// Dropout parameters -> the kernels' form; QLORA_OK with *on = 0 for p == 0.
static int make_dropout(const qlora_dropout* dp, Dropout* out) {
  if (!dp) return QLORA_ERR_INVALID_ARG;
  const float p = dp->p;
  if (!(p >= 0.0f && p < 1.0f)) return QLORA_ERR_INVALID_ARG;
  out->seed = dp->seed;
  out->thr = (uint32_t)std::floor((double)p * 16777216.0 + 0.5);
  out->scale = 1.0f / (1.0f - p);
  out->on = out->thr != 0 ? 1 : 0;
  return QLORA_OK;
}

int qlora_linear_fwd_dropout(const nf4_weight* w, const void* X, int64_t M, const void* A,
                             const void* B, int r, float alpha, const qlora_dropout* dropout,
                             void* Y, void* T_save, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  Dropout dr{};
  const int st = make_dropout(dropout, &dr);
  if (st) return st;
  return fwd_impl(w, X, M, A, B, r, alpha, &dr, Y, T_save, ws, ws_bytes, stream);
}

int qlora_linear_bwd_dropout(const nf4_weight* w, const void* X, const void* dY, int64_t M,
                             const void* A, const void* B, int r, float alpha,
                             const qlora_dropout* dropout, const void* T, void* dX, void* dA,
                             void* dB, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  Dropout dr{};
  const int st = make_dropout(dropout, &dr);
  if (st) return st;
  return bwd_impl(w, X, dY, M, A, B, r, alpha, &dr, T, dX, dA, dB, ws, ws_bytes, stream);
}

// Write one field of the current device's state block (synchronous).
static int write_state_field(size_t offset, const void* src, size_t bytes) {
  DeviceInfo* d = nullptr;
  int st = current_device(&d);
  if (st) return st;
  if (cudaMemcpy(reinterpret_cast<uint8_t*>(d->status) + offset, src, bytes, cudaMemcpyHostToDevice) !=
      cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

int qlora_set_wait_limit(uint64_t ns) {
  if (ns == 0) ns = kWaitLimitNs;
  if (ns < 1000000ull || ns > 60000000000ull) return QLORA_ERR_INVALID_ARG;
  const unsigned long long v = ns;
  return write_state_field(offsetof(DevState, wait_limit_ns), &v, sizeof(v));
}

int qlora_test_withhold_first_fill(int on) {
  const int v = on ? 1 : 0;
  return write_state_field(offsetof(DevState, withhold_first_fill), &v, sizeof(v));
}

int qlora_check_status(qlora_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  DeviceInfo* d = nullptr;
  int st = current_device(&d);
  if (st) return st;
  int v = 0;
  if (cudaMemcpy(&v, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(d->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
  }
  return v;
}

}  // extern "C"
