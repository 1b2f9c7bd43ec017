"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This module holds no quantisation or layer arithmetic: it only draws
Gaussian tensors and names the workloads.

Recipe
------
* Generator: NumPy ``default_rng(seed)`` (PCG64), ``standard_normal`` in fp32,
  multiplied by sigma, then rounded to bf16 (round-to-nearest-even, via
  torch's dtype conversion) wherever the workload is bf16.
* Seed = 1000 * workload id + tensor id, tensor ids W=1, X=2, A=3, B=4, dY=5,
  outlier mask=6 (a second weight of the same workload uses +10, +20, ...).
* sigma: W 0.02, X and dY 1.0, A and B 0.02 -- trained weights are roughly
  normal (page "QLoRA Explained", section "What a trained model's weights
  actually look like"); no real model, dataset or checkpoint is used.
* Outlier variant: 1 % of the weight indices, chosen without replacement by
  the mask generator, are multiplied by 10 before rounding to bf16 (the
  "single freak weight" of section "Why the groups are small").
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

TID_W, TID_X, TID_A, TID_B, TID_DY, TID_MASK = 1, 2, 3, 4, 5, 6


def gaussian(shape, sigma: float, seed: int) -> np.ndarray:
    """fp32 N(0, sigma^2) samples from PCG64(seed)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=int(np.prod(shape)), dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return x.reshape(shape)


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """fp32 NumPy array -> CPU bf16 tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)


def weight(rows: int, cols: int, seed: int, dtype: str = "bf16",
           outliers: bool = False, sigma: float = 0.02) -> torch.Tensor:
    """A seeded weight matrix [rows, cols] in bf16 (or fp32)."""
    w = gaussian((rows, cols), sigma, seed)
    if outliers:
        n = rows * cols
        k = max(1, n // 100)
        rng = np.random.default_rng(seed - TID_W + TID_MASK)
        idx = rng.choice(n, size=k, replace=False)
        w.reshape(-1)[idx] *= np.float32(10.0)
    if dtype == "fp32":
        return torch.from_numpy(w)
    return to_bf16(w)


def activations(rows: int, cols: int, seed: int, sigma: float = 1.0) -> torch.Tensor:
    """A seeded bf16 activation (or upstream-gradient) matrix."""
    return to_bf16(gaussian((rows, cols), sigma, seed))


@dataclass
class Workload:
    """One named workload: weight shapes, token count, adapter rank and alpha."""
    wid: int
    name: str
    weights: list = field(default_factory=list)   # [(N, K), ...]
    M: int = 16
    r: int = 8
    alpha: float = 16.0
    w_dtype: str = "bf16"
    backward: bool = False
    decode_M: tuple = ()

    def seed(self, tid: int, which: int = 0) -> int:
        return 1000 * self.wid + tid + 10 * which


WORKLOADS = {
    "tiny_roundtrip": Workload(
        1, "W 1024x1024 fp32, X 16x1024, r=8 alpha=16",
        weights=[(1024, 1024)], M=16, r=8, alpha=16.0, w_dtype="fp32"),
    "attn_proj_4096": Workload(
        2, "W 4096x4096 bf16, X 4096x4096 (batch 4 x seq 1024), r=16 alpha=32",
        weights=[(4096, 4096)], M=4096, r=16, alpha=32.0),
    "mlp_7b": Workload(
        3, "7B-class MLP: gate/up W 18944x3584, down W 3584x18944, 8192 tokens, r=64 alpha=16",
        weights=[(18944, 3584), (18944, 3584), (3584, 18944)], M=8192, r=64, alpha=16.0),
    "bwd_4096": Workload(
        4, "backward on W 4096x4096, X and dY 8192x4096, r=64 alpha=128",
        weights=[(4096, 4096)], M=8192, r=64, alpha=128.0, backward=True),
    "decode_70b": Workload(
        5, "70B-class W 28672x8192 (also 1% outliers x10), decode M in {1,4,16}, r=16 alpha=32",
        weights=[(28672, 8192)], M=16, r=16, alpha=32.0, decode_M=(1, 4, 16)),
}


def layer_inputs(wl: Workload, which: int = 0, M: int | None = None,
                 outliers: bool = False):
    """(W, X, A, B) for weight `which` of a workload, all CPU tensors."""
    N, K = wl.weights[which]
    M = wl.M if M is None else M
    W = weight(N, K, wl.seed(TID_W, which), wl.w_dtype, outliers=outliers)
    X = activations(M, K, wl.seed(TID_X, which))
    A = activations(wl.r, K, wl.seed(TID_A, which), sigma=0.02)
    B = activations(N, wl.r, wl.seed(TID_B, which), sigma=0.02)
    return W, X, A, B


def upstream_grad(wl: Workload, which: int = 0, M: int | None = None) -> torch.Tensor:
    N, _ = wl.weights[which]
    M = wl.M if M is None else M
    return activations(M, N, wl.seed(TID_DY, which))
