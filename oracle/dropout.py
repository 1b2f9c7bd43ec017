"""Oracle for LoRA dropout on the adapter's input (CPU, NumPy, fp64 matmuls).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Page "QLoRA Explained", config walk-through: the adapter configuration sets
lora_dropout=0.05 -- dropout on the input of the adapter branch only; the
frozen base still sees every input.  With keep mask D (1 with probability
1 - p) and X' = D * X / (1 - p):

    Y  = X W'^T + s (X' A^T) B^T
    U  = dY B
    dX = dY W' + (D / (1 - p)) * (s U A)      (the dropout's gradient)
    dA = s U^T X'
    dB = s dY^T (X' A^T)

Readings (the page names only the rate):
* The mask is drawn from a counter-based generator so that the forward and
  the backward regenerate the same mask: Philox4x64-10 (Salmon, Moraes, Dror
  and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), key
  (seed, 0), counter (e // 8, 0, 0, 0) for element e = m * K + k of X.  One
  block's four 64-bit words serve eight elements: element e uses word
  (e % 8) // 2, bits 40..63 for even e and bits 16..39 for odd e, as a
  24-bit uniform u; the element is kept when u >= floor(p * 2^24 + 1/2).
* X' is rounded to bf16 like every adapter operand: X' = RNbf16(RN32(x * c))
  with c = RN32(1 / RN32(1 - p)); dropped elements are 0.
* The dropout gradient's factor is the same c: dX's adapter term is
  D * c * (s U A).
"""

from __future__ import annotations

import numpy as np

from .nf4 import round_bf16

_MASK64 = (1 << 64) - 1
# Philox4x64 multipliers and key increments (the published constants)
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15
PHILOX_W1 = 0xBB67AE8584CAA73B


def _mulhilo(a: int, b: int):
    p = a * b
    return p >> 64, p & _MASK64


def philox4x64_10(counter, key) -> tuple[int, int, int, int]:
    """Ten Philox rounds of the 4 x 64-bit counter under the 2 x 64-bit key.

    One round: (hi0, lo0) = M0 * c0, (hi1, lo1) = M1 * c2 (full 128-bit
    products), then c = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0); the key is
    bumped by (W0, W1) before every round after the first.
    """
    c0, c1, c2, c3 = (int(v) & _MASK64 for v in counter)
    k0, k1 = (int(v) & _MASK64 for v in key)
    for r in range(10):
        if r:
            k0 = (k0 + PHILOX_W0) & _MASK64
            k1 = (k1 + PHILOX_W1) & _MASK64
        hi0, lo0 = _mulhilo(PHILOX_M0, c0)
        hi1, lo1 = _mulhilo(PHILOX_M1, c2)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def keep_threshold(p: float) -> int:
    """floor(RN32(p) * 2^24 + 1/2) (exact in fp64): 24-bit uniforms below it
    are dropped."""
    return int(np.floor(float(np.float32(p)) * (1 << 24) + 0.5))


def keep_mask(M: int, K: int, p: float, seed: int) -> np.ndarray:
    """The [M, K] keep mask (bool) of the reading above (pure-Python Philox:
    for small shapes)."""
    thr = keep_threshold(p)
    n = M * K
    out = np.empty(n, dtype=bool)
    for blk in range((n + 7) // 8):
        words = philox4x64_10((blk, 0, 0, 0), (seed, 0))
        for i in range(8):
            e = 8 * blk + i
            if e < n:
                u = (words[i // 2] >> (40 if i % 2 == 0 else 16)) & 0xFFFFFF
                out[e] = u >= thr
    return out.reshape(M, K)


def keep_scale(p: float) -> np.float32:
    """c = RN32(1 / RN32(1 - p))."""
    return np.float32(np.float32(1.0) / np.float32(np.float32(1.0) - np.float32(p)))


def dropped_input(X, mask, p: float) -> np.ndarray:
    """X' = RNbf16(RN32(x * c)) where kept, 0 where dropped (fp32 values)."""
    x = np.asarray(X, dtype=np.float32)
    scaled = round_bf16((x * keep_scale(p)).astype(np.float32))
    return np.where(mask, scaled, np.float32(0)).astype(np.float32)


def linear_fwd_dropout(X, Wdeq, A, B, alpha: float, r: int, mask, p: float):
    """Y = X W'^T + s (X' A^T) B^T in fp64; returns (Y, T) with T = X' A^T."""
    X64 = np.asarray(X, dtype=np.float64)
    Xd = dropped_input(X, mask, p).astype(np.float64)
    W, A, B = (np.asarray(t, dtype=np.float64) for t in (Wdeq, A, B))
    s = float(alpha) / float(r)
    T = Xd @ A.T
    return X64 @ W.T + s * (T @ B.T), T


def linear_bwd_dropout(X, dY, Wdeq, A, B, alpha: float, r: int, mask, p: float):
    """(dX, dA, dB) of the layer with dropout on the adapter input, fp64."""
    Xd = dropped_input(X, mask, p).astype(np.float64)
    dY, W, A, B = (np.asarray(t, dtype=np.float64) for t in (dY, Wdeq, A, B))
    s = float(alpha) / float(r)
    c = float(keep_scale(p))
    U = dY @ B
    dX = dY @ W + np.where(mask, c, 0.0) * (s * (U @ A))
    dA = s * (U.T @ Xd)
    dB = s * (dY.T @ (Xd @ A.T))
    return dX, dA, dB
