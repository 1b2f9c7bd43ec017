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
