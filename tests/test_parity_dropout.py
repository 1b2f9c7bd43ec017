"""GPU parity of the layer with LoRA dropout on the adapter input against the
oracle (oracle.dropout: Philox4x64-10 mask pinned against NumPy's Philox).

* The mask and the scaled kept values are checked bit for bit: with A a set
  of one-hot rows, T = X' A^T picks single columns of the dropped-out input
  X' exactly.
* Forward and backward are checked within the layer tolerance
  max|d| / max|ref| <= 1e-2 against the oracle's fp64 layer on the same mask.
* p = 0 is the plain layer, bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import dropout as OD
from qlora_linear_layers_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module")
def q():
    from qlora_linear_layers_b200.build import build
    build()
    import qlora_linear_layers_b200 as q
    return q


def rel_err(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(g - ref)) / np.max(np.abs(ref)))


def _oracle_weight(W_cpu):
    codes, a = oracle.quantize(W_cpu.float().numpy())
    qa, s, mu = oracle.double_quantize(a)
    return oracle.dequantize(oracle.pack(codes), oracle.dq_absmax(qa, s, mu), tuple(W_cpu.shape))


@pytest.mark.parametrize("p,seed", [(0.05, 1234), (0.5, 99), (0.3, 2 ** 63 + 5)])
def test_mask_and_scaling_exact(q, p, seed):
    """T = X' A^T with one-hot rows of A returns columns of X' exactly."""
    N, K, M, r = 256, 512, 300, 128
    W = synth.weight(N, K, 31, "bf16").cuda()
    X = synth.activations(M, K, 32)
    cols = np.random.default_rng(33).choice(K, r, replace=False)
    A = torch.zeros(r, K, dtype=torch.bfloat16)
    A[np.arange(r), cols] = 1.0
    B = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    wq = q.quantize(W)
    Y, T = q.linear_fwd_dropout(wq, X.cuda(), A.cuda(), B, 32.0, p, seed)
    assert q.qlora_check_status() == 0
    mask = OD.keep_mask(M, K, p, seed)
    Xd = OD.dropped_input(X.float().numpy(), mask, p)
    assert np.array_equal(T.float().cpu().numpy(), Xd[:, cols])
    # the base path sees every input: with B = 0, Y is the plain layer's
    Y0, _ = q.linear_fwd(wq, X.cuda(), A.cuda(), B, 32.0)
    assert torch.equal(Y.view(torch.int16), Y0.view(torch.int16))


@pytest.mark.parametrize("N,K,M,r,alpha,p", [
    (384, 512, 300, 16, 32.0, 0.05),
    (200, 192, 257, 64, 16.0, 0.1),
    (96, 256, 300, 8, 16.0, 0.05),          # single-SM GEMM engine
    (512, 1024, 8, 16, 32.0, 0.05),         # a decode-sized token count runs the GEMM path
])
def test_forward_backward_dropout(q, N, K, M, r, alpha, p):
    seed = 1000 + M
    W = synth.weight(N, K, seed + 1, "bf16")
    X = synth.activations(M, K, seed + 2)
    A = synth.activations(r, K, seed + 3, sigma=0.02)
    B = synth.activations(N, r, seed + 4, sigma=0.02)
    dY = synth.activations(M, N, seed + 5)
    wq = q.quantize(W.cuda())
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    Y, T = q.linear_fwd_dropout(wq, Xc, Ac, Bc, alpha, p, seed)
    dX, dA, dB = q.linear_bwd_dropout(wq, Xc, dYc, Ac, Bc, alpha, p, seed, T=T)
    dX2, dA2, dB2 = q.linear_bwd_dropout(wq, Xc, dYc, Ac, Bc, alpha, p, seed)     # T recomputed
    assert q.qlora_check_status() == 0
    mask = OD.keep_mask(M, K, p, seed)
    Wd = _oracle_weight(W)
    Xn, An, Bn, dYn = (t.float().numpy() for t in (X, A, B, dY))
    Yr, Tr = OD.linear_fwd_dropout(Xn, Wd, An, Bn, alpha, r, mask, p)
    dXr, dAr, dBr = OD.linear_bwd_dropout(Xn, dYn, Wd, An, Bn, alpha, r, mask, p)
    assert rel_err(Y, Yr) <= TOL and rel_err(T, Tr) <= TOL
    for got in ((dX, dA, dB), (dX2, dA2, dB2)):
        assert rel_err(got[0], dXr) <= TOL
        assert rel_err(got[1], dAr) <= TOL
        assert rel_err(got[2], dBr) <= TOL
    # the dropout matters: without it the adapter gradient is off the bar
    dAp, _ = oracle.linear_bwd_adapters(Xn, dYn, An, Bn, alpha, r)
    assert np.max(np.abs(dAp - dAr)) / np.max(np.abs(dAr)) > 2 * TOL


def test_p_zero_is_the_plain_layer(q):
    N, K, M, r, alpha = 256, 512, 300, 16, 32.0
    W = synth.weight(N, K, 41, "bf16").cuda()
    X = synth.activations(M, K, 42).cuda()
    A = synth.activations(r, K, 43, sigma=0.02).cuda()
    B = synth.activations(N, r, 44, sigma=0.02).cuda()
    dY = synth.activations(M, N, 45).cuda()
    wq = q.quantize(W)
    Y, T = q.linear_fwd_dropout(wq, X, A, B, alpha, 0.0, 7)
    Y0, T0 = q.linear_fwd(wq, X, A, B, alpha)
    g = q.linear_bwd_dropout(wq, X, dY, A, B, alpha, 0.0, 7, T=T)
    g0 = q.linear_bwd(wq, X, dY, A, B, alpha, T=T0)
    assert q.qlora_check_status() == 0
    assert torch.equal(Y, Y0) and torch.equal(T, T0)
    for a, b in zip(g, g0):
        assert torch.equal(a, b)
    with pytest.raises(q.QLoraError):
        q.linear_fwd_dropout(wq, X, A, B, alpha, 1.0, 7)
