"""B200-native QLoRA NF4 linear layers.

Thin Python binding over libqlora_nf4.so (C ABI in include/qlora_nf4.h).
PyTorch supplies device memory and streams only; every step of the path runs
in the library's sm_100a kernels.  The functions named like the C entry
points (nf4_quantize, nf4_double_quantize, nf4_dequantize, qlora_linear_fwd,
qlora_linear_bwd, qlora_check_status) marshal tensors to pointers; `quantize`,
`dequantize`, `linear_fwd`, `linear_bwd` are conveniences that allocate the
outputs and the workspace with torch and call them.
"""

from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import QLoraError  # noqa: F401

BLOCKSIZE = 64
DQ_BLOCKSIZE = 256


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


@dataclass
class NF4Tensor:
    """A quantised weight: the buffers of `nf4_weight` plus its shape."""
    packed: torch.Tensor            # uint8 [rows*cols/2]
    rows: int
    cols: int
    absmax: torch.Tensor            # fp32 [rows*cols/64]
    qabsmax: torch.Tensor | None    # int8 [rows*cols/64]
    dq_scale: torch.Tensor | None   # fp32 [ceil(n_absmax/256)]
    dq_mean: torch.Tensor | None    # fp32 [1]
    double_quant: int = 1           # 0 none, 1 int8 codes, 2 E4M3 codes (True = 1)
    quant_type: int = _lib.QLORA_QUANT_NF4

    def c_struct(self) -> _lib.NF4Weight:
        return _lib.NF4Weight(
            packed=_ptr(self.packed), rows=self.rows, cols=self.cols, blocksize=BLOCKSIZE,
            double_quant=int(self.double_quant),
            absmax=_ptr(self.absmax), qabsmax=_ptr(self.qabsmax), dq_scale=_ptr(self.dq_scale),
            dq_mean=_ptr(self.dq_mean), dq_blocksize=DQ_BLOCKSIZE, quant_type=self.quant_type)

    def stored_bytes(self) -> int:
        """Bytes the quantised weight occupies (codes + constants in use)."""
        if self.double_quant:
            return (self.packed.numel() + self.qabsmax.numel() + 4 * self.dq_scale.numel()
                    + 4 * self.dq_mean.numel())
        return self.packed.numel() + 4 * self.absmax.numel()


# ---------------------------------------------------------------------------
# Entry points with the C names
# ---------------------------------------------------------------------------

def nf4_quantize(W: torch.Tensor, packed: torch.Tensor, absmax: torch.Tensor, stream=None):
    _need_cuda(W, packed, absmax)
    dt = {torch.float32: _lib.QLORA_F32, torch.bfloat16: _lib.QLORA_BF16}.get(W.dtype)
    if dt is None:
        raise ValueError("W must be fp32 or bf16")
    _lib.check(_lib.load().nf4_quantize(_ptr(W), dt, W.shape[0], W.shape[1], BLOCKSIZE,
                                        _ptr(packed), _ptr(absmax), _stream(stream)),
               "nf4_quantize")


def qlora_quantize_4bit(W: torch.Tensor, packed: torch.Tensor, absmax: torch.Tensor,
                        quant_type: int = _lib.QLORA_QUANT_NF4, dq_hist: torch.Tensor | None = None,
                        stream=None):
    """Quantise W (fp32/bf16 [rows, cols]); with dq_hist (int64 [256]) also
    write the exponent histogram of the block absmax values."""
    _need_cuda(W, packed, absmax, dq_hist)
    dt = {torch.float32: _lib.QLORA_F32, torch.bfloat16: _lib.QLORA_BF16}.get(W.dtype)
    if dt is None:
        raise ValueError("W must be fp32 or bf16")
    if dq_hist is not None and (dq_hist.dtype != torch.int64 or dq_hist.numel() != 256):
        raise ValueError("dq_hist must be int64 [256]")
    _lib.check(_lib.load().qlora_quantize_4bit(_ptr(W), dt, W.shape[0], W.shape[1], BLOCKSIZE,
                                               int(quant_type), _ptr(packed), _ptr(absmax),
                                               _ptr(dq_hist), _stream(stream)),
               "qlora_quantize_4bit")


def nf4_double_quantize_hist(absmax: torch.Tensor, dq_hist: torch.Tensor, n_total: int,
                             qabsmax: torch.Tensor, dq_scale: torch.Tensor, dq_mean: torch.Tensor,
                             stream=None, dq_type: int = _lib.QLORA_DQ_INT8):
    """Second double-quantisation pass from a complete histogram over n_total
    absmax values (summed over shards when the weight is sharded); dq_type
    picks int8 or E4M3 codes."""
    _need_cuda(absmax, dq_hist, qabsmax, dq_scale, dq_mean)
    _lib.check(_lib.load().qlora_double_quantize_hist(_ptr(absmax), absmax.numel(), _ptr(dq_hist),
                                                      int(n_total), DQ_BLOCKSIZE, int(dq_type),
                                                      _ptr(qabsmax), _ptr(dq_scale), _ptr(dq_mean),
                                                      _stream(stream)),
               "qlora_double_quantize_hist")


def workspace_bytes(op: int, M: int, N: int, K: int, r: int) -> int:
    return int(_lib.load().qlora_workspace_bytes(op, M, N, K, r))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def nf4_double_quantize(absmax: torch.Tensor, qabsmax: torch.Tensor, dq_scale: torch.Tensor,
                        dq_mean: torch.Tensor, ws: torch.Tensor | None = None, stream=None):
    _need_cuda(absmax, qabsmax, dq_scale, dq_mean)
    need = workspace_bytes(_lib.QLORA_OP_DOUBLE_QUANT, 0, absmax.numel(), 0, 0)
    if ws is None:
        ws = _workspace(need, absmax.device)
    _lib.check(_lib.load().nf4_double_quantize(_ptr(absmax), absmax.numel(), DQ_BLOCKSIZE,
                                               _ptr(qabsmax), _ptr(dq_scale), _ptr(dq_mean),
                                               _ptr(ws), ws.numel(), _stream(stream)),
               "nf4_double_quantize")


def nf4_dequantize(w: NF4Tensor, out: torch.Tensor, stream=None):
    _need_cuda(out)
    cw = w.c_struct()
    _lib.check(_lib.load().nf4_dequantize(C.byref(cw), _ptr(out), _stream(stream)),
               "nf4_dequantize")


def qlora_merge(w: NF4Tensor, A, B, alpha: float, out, stream=None):
    """out[N, K] bf16 = RNbf16(deq(W) + (alpha / r) B A)."""
    _need_cuda(A, B, out)
    cw = w.c_struct()
    _lib.check(_lib.load().qlora_merge(C.byref(cw), _ptr(A), _ptr(B), A.shape[0], float(alpha),
                                       _ptr(out), _stream(stream)),
               "qlora_merge")


def qlora_linear_fwd(w: NF4Tensor, X, A, B, alpha: float, Y, T_save=None, ws=None, stream=None):
    _need_cuda(X, A, B, Y, T_save)
    M, r = X.shape[0], A.shape[0]
    need = workspace_bytes(_lib.QLORA_OP_FWD, M, w.rows, w.cols, r)
    if ws is None:
        ws = _workspace(need, X.device)
    cw = w.c_struct()
    _lib.check(_lib.load().qlora_linear_fwd(C.byref(cw), _ptr(X), M, _ptr(A), _ptr(B), r,
                                            float(alpha), _ptr(Y), _ptr(T_save), _ptr(ws),
                                            ws.numel(), _stream(stream)),
               "qlora_linear_fwd")


def qlora_linear_bwd(w: NF4Tensor, X, dY, A, B, alpha: float, dX, dA, dB, T=None, ws=None,
                     stream=None):
    _need_cuda(X, dY, A, B, dX, dA, dB, T)
    M, r = X.shape[0], A.shape[0]
    need = workspace_bytes(_lib.QLORA_OP_BWD, M, w.rows, w.cols, r)
    if ws is None:
        ws = _workspace(need, X.device)
    cw = w.c_struct()
    _lib.check(_lib.load().qlora_linear_bwd(C.byref(cw), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B),
                                            r, float(alpha), _ptr(T), _ptr(dX), _ptr(dA),
                                            _ptr(dB), _ptr(ws), ws.numel(), _stream(stream)),
               "qlora_linear_bwd")


def qlora_linear_fwd_dropout(w: NF4Tensor, X, A, B, alpha: float, p: float, seed: int, Y,
                             T_save=None, ws=None, stream=None):
    """The forward with LoRA dropout (rate p, Philox seed) on the adapter input."""
    _need_cuda(X, A, B, Y, T_save)
    M, r = X.shape[0], A.shape[0]
    if ws is None:
        ws = _workspace(workspace_bytes(_lib.QLORA_OP_FWD_DROPOUT, M, w.rows, w.cols, r), X.device)
    cw = w.c_struct()
    dr = _lib.Dropout(p=float(p), reserved=0, seed=int(seed))
    _lib.check(_lib.load().qlora_linear_fwd_dropout(C.byref(cw), _ptr(X), M, _ptr(A), _ptr(B), r,
                                                    float(alpha), C.byref(dr), _ptr(Y), _ptr(T_save),
                                                    _ptr(ws), ws.numel(), _stream(stream)),
               "qlora_linear_fwd_dropout")


def qlora_linear_bwd_dropout(w: NF4Tensor, X, dY, A, B, alpha: float, p: float, seed: int, dX, dA,
                             dB, T=None, ws=None, stream=None):
    """The backward with LoRA dropout; the mask is regenerated from (p, seed)."""
    _need_cuda(X, dY, A, B, dX, dA, dB, T)
    M, r = X.shape[0], A.shape[0]
    if ws is None:
        ws = _workspace(workspace_bytes(_lib.QLORA_OP_BWD_DROPOUT, M, w.rows, w.cols, r), X.device)
    cw = w.c_struct()
    dr = _lib.Dropout(p=float(p), reserved=0, seed=int(seed))
    _lib.check(_lib.load().qlora_linear_bwd_dropout(C.byref(cw), _ptr(X), _ptr(dY), M, _ptr(A),
                                                    _ptr(B), r, float(alpha), C.byref(dr), _ptr(T),
                                                    _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                                                    ws.numel(), _stream(stream)),
               "qlora_linear_bwd_dropout")


def qlora_check_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(_lib.load().qlora_check_status(_stream(stream)))


def code_table(quant_type: int = _lib.QLORA_QUANT_NF4) -> list[float]:
    buf = (C.c_float * 16)()
    _lib.check(_lib.load().qlora_code_table(int(quant_type), buf), "qlora_code_table")
    return list(buf)


def code_thresholds(quant_type: int = _lib.QLORA_QUANT_NF4) -> list[float]:
    buf = (C.c_float * 15)()
    cnt = C.c_int(0)
    _lib.check(_lib.load().qlora_code_thresholds(int(quant_type), buf, C.byref(cnt)),
               "qlora_code_thresholds")
    return list(buf)[:cnt.value]


# ---------------------------------------------------------------------------
# Conveniences
# ---------------------------------------------------------------------------

def empty_quantized(rows: int, cols: int, device, double_quant: int = 1,
                    quant_type: int = _lib.QLORA_QUANT_NF4) -> NF4Tensor:
    """Buffers of a quantised [rows, cols] weight (absmax is kept either way:
    the quantise pass writes it)."""
    n = rows * cols
    na = n // BLOCKSIZE
    t = NF4Tensor(torch.empty(n // 2, dtype=torch.uint8, device=device), rows, cols,
                  torch.empty(na, dtype=torch.float32, device=device), None, None, None,
                  int(double_quant), quant_type)
    if double_quant:
        t.qabsmax = torch.empty(na, dtype=torch.int8, device=device)
        t.dq_scale = torch.empty((na + DQ_BLOCKSIZE - 1) // DQ_BLOCKSIZE, dtype=torch.float32,
                                 device=device)
        t.dq_mean = torch.empty(4, dtype=torch.float32, device=device)[:1]
    return t


def quantize(W: torch.Tensor, double_quant: int = 1, quant_type: int = _lib.QLORA_QUANT_NF4,
             stream=None) -> NF4Tensor:
    """Quantise W.  double_quant: 0 (or False) keeps fp32 block scales, 1 (or
    True) int8 codes, 2 E4M3 codes; the mean's histogram is built in the
    quantise pass and one more pass writes the 8-bit scales."""
    rows, cols = W.shape
    dq = int(double_quant)
    q = empty_quantized(rows, cols, W.device, dq, quant_type)
    if not dq:
        qlora_quantize_4bit(W, q.packed, q.absmax, quant_type, None, stream)
        return q
    hist = torch.empty(256, dtype=torch.int64, device=W.device)
    qlora_quantize_4bit(W, q.packed, q.absmax, quant_type, hist, stream)
    nf4_double_quantize_hist(q.absmax, hist, q.absmax.numel(), q.qabsmax, q.dq_scale, q.dq_mean,
                             stream, dq_type=dq)
    return q


def dequantize(w: NF4Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=w.packed.device)
    nf4_dequantize(w, out, stream)
    return out


def merge(w: NF4Tensor, A, B, alpha: float, stream=None) -> torch.Tensor:
    out = torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=w.packed.device)
    qlora_merge(w, A, B, alpha, out, stream)
    return out


def linear_fwd(w: NF4Tensor, X, A, B, alpha: float, save_T: bool = True, stream=None):
    M, r = X.shape[0], A.shape[0]
    Y = torch.empty(M, w.rows, dtype=torch.bfloat16, device=X.device)
    T = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if save_T else None
    qlora_linear_fwd(w, X, A, B, alpha, Y, T, stream=stream)
    return Y, T


def linear_fwd_dropout(w: NF4Tensor, X, A, B, alpha: float, p: float, seed: int,
                       save_T: bool = True, stream=None):
    M, r = X.shape[0], A.shape[0]
    Y = torch.empty(M, w.rows, dtype=torch.bfloat16, device=X.device)
    T = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if save_T else None
    qlora_linear_fwd_dropout(w, X, A, B, alpha, p, seed, Y, T, stream=stream)
    return Y, T


def linear_bwd_dropout(w: NF4Tensor, X, dY, A, B, alpha: float, p: float, seed: int, T=None,
                       stream=None):
    dX = torch.empty_like(X)
    dA = torch.empty_like(A)
    dB = torch.empty_like(B)
    qlora_linear_bwd_dropout(w, X, dY, A, B, alpha, p, seed, dX, dA, dB, T=T, stream=stream)
    return dX, dA, dB


def linear_bwd(w: NF4Tensor, X, dY, A, B, alpha: float, T=None, stream=None):
    dX = torch.empty_like(X)
    dA = torch.empty_like(A)
    dB = torch.empty_like(B)
    qlora_linear_bwd(w, X, dY, A, B, alpha, dX, dA, dB, T=T, stream=stream)
    return dX, dA, dB
