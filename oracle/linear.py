"""Oracle for the QLoRA linear layer, forward and input/adapter backward, fp64.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Page "LoRA vs QLoRA: Efficient Fine-Tuning Explained", section "How LoRA
Works: Low-Rank Adapters": a frozen W of shape d x k, B of shape d x r, A of
shape r x k, effective weight W + (alpha/r) * B @ A.  With PyTorch's Linear
convention (W stored [N, K] = [d, k], Y = X W^T) the layer is

    Y = X W'^T + s (X A^T) B^T,      s = alpha / r,

where W' is the dequantised bf16 NF4 weight (page "QLoRA Explained",
section "That is NF4": every matmul runs on values expanded back to bf16;
the adapter is bf16 throughout).  Section "How QLoRA Works: Quantized Base
Plus LoRA" of the LoRA-vs-QLoRA page: the base weights never receive
gradients, only the adapters do -- so the backward produces dX, dA, dB and
no dW.

All products are fp64 matmuls (NumPy) of the exact bf16 input values; no
blocking, no fusion.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def linear_fwd(X, Wdeq, A, B, alpha: float, r: int):
    """Y = X W'^T + s (X A^T) B^T in fp64.  Returns (Y, T) with T = X A^T."""
    X, W, A, B = _f64(X), _f64(Wdeq), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    T = X @ A.T                      # [M, r]
    Y = X @ W.T + s * (T @ B.T)      # [M, N]
    return Y, T


def linear_bwd(X, dY, Wdeq, A, B, alpha: float, r: int):
    """Gradients of sum(dY * Y) with respect to X, A and B (W is frozen).

      U  = dY B                 [M, r]
      dX = dY W' + s U A        [M, K]
      dA = s U^T X              [r, K]
      dB = s dY^T (X A^T)       [N, r]
    """
    X, dY, W, A, B = _f64(X), _f64(dY), _f64(Wdeq), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    U = dY @ B
    dX = dY @ W + s * (U @ A)
    dA = s * (U.T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dX, dA, dB


def linear_bwd_adapters(X, dY, A, B, alpha: float, r: int):
    """dA = s (dY B)^T X and dB = s dY^T (X A^T) alone (no dX), fp64.

    Same formulas as linear_bwd; split out so that the adapter gradients of a
    large layer can be checked in full without forming the M x N x K product
    that dX needs.
    """
    X, dY, A, B = _f64(X), _f64(dY), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    dA = s * ((dY @ B).T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dA, dB


def round_bf16_f64(x) -> np.ndarray:
    """fp64 -> bf16 round-to-nearest-even in one step (no fp32 in between);
    returns the bf16 values as fp64.  bf16 keeps 8 significand bits: the top
    1 + 7 of fp64's 53, so the low 45 bits of the fp64 pattern are dropped
    with half rounding up and exact halves to an even kept part.  Finite
    values of normal bf16 magnitude (>= 2^-126) or zero."""
    u = np.asarray(x, dtype=np.float64).view(np.uint64)
    keep = u >> np.uint64(45)
    rest = u & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rest > half) | ((rest == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    return ((keep + up.astype(np.uint64)) << np.uint64(45)).view(np.float64)


def merge(Wdeq, A, B, alpha: float, r: int) -> np.ndarray:
    """The merged weight for export: RNbf16(W' + s B A), the sum in fp64 and
    rounded once to bf16.

    Page "QLoRA Explained", section "Why a 16-bit adapter will not fold into a
    4-bit base": the adapter product is bf16 and cannot be added to 4-bit
    codes, so the base is dequantised first (W' = the bf16 values of
    dequantize) and the product added to it; page "LoRA vs QLoRA", section
    "How LoRA Works": W + (alpha/r) B A with B d x r, A r x k.  Reading: the
    result is stored in the compute type, bf16.
    """
    W, A, B = _f64(Wdeq), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    return round_bf16_f64(W + s * (B @ A))
