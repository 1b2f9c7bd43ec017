"""GPU parity of qlora_merge (the adapter added to the dequantised base)
against the oracle.

The oracle sums in fp64 and rounds once to bf16; the kernel accumulates the
rank-r product in fp32 on tensor cores, adds the bf16 dequantised weight in
fp32 and rounds that to bf16.  The two differ only where the exact sum lies
within the kernel's fp32 error (about r * 2^-24 relative) of a halfway point
between two bf16 values, so the bar is: every element within one bf16 ulp of
the oracle, and at least 99 % of them equal bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from qlora_linear_layers_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from qlora_linear_layers_b200.build import build
    build()
    import qlora_linear_layers_b200 as q
    return q


def _oracle_deq(W_cpu, dq, qt):
    table = oracle.fp4_table() if qt == 1 else oracle.nf4_table()
    codes, a = oracle.quantize(W_cpu.float().numpy(), table)
    if dq:
        fmt = "fp8" if int(dq) == 2 else "int8"
        qa, s, mu = oracle.double_quantize(a, fmt=fmt)
        a = oracle.dq_absmax(qa, s, mu, fmt=fmt)
    return oracle.dequantize(oracle.pack(codes), a, tuple(W_cpu.shape), table=table)


def _check(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) * 2.0 ** 16
    ulp = np.maximum(ulp, 2.0 ** -133)
    assert np.all(np.abs(g - ref) <= ulp), float(np.max(np.abs(g - ref) / ulp))
    assert np.mean(g == ref) >= 0.99


@pytest.mark.parametrize("N,K,r,alpha,dq,qt", [
    (200, 192, 8, 16.0, True, 0),          # ragged rows and a 64-column last tile
    (384, 512, 64, 16.0, True, 0),
    (136, 320, 128, 64.0, False, 0),
    (1024, 1024, 16, 32.0, True, 0),
    (256, 640, 32, 8.0, True, 1),          # FP4 storage
    (384, 512, 64, 16.0, 2, 0),            # E4M3 block-scale codes
])
def test_merge_small(q, N, K, r, alpha, dq, qt):
    W = synth.weight(N, K, 600 + r, "bf16")
    A = synth.activations(r, K, 601 + r, sigma=0.02)
    B = synth.activations(N, r, 602 + r, sigma=0.02)
    wq = q.quantize(W.cuda(), double_quant=dq, quant_type=qt)
    Wm = q.merge(wq, A.cuda(), B.cuda(), alpha)
    assert q.qlora_check_status() == 0
    ref = oracle.merge(_oracle_deq(W, dq, qt), A.float().numpy(), B.float().numpy(), alpha, r)
    _check(Wm, ref)


def test_merge_zero_adapter_is_dequantize(q):
    """B = 0: the merged weight is the dequantised weight, bit for bit."""
    N, K, r = 384, 512, 16
    W = synth.weight(N, K, 650, "bf16").cuda()
    wq = q.quantize(W, double_quant=True)
    A = synth.activations(r, K, 651, sigma=0.02).cuda()
    B = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    Wm = q.merge(wq, A, B, 32.0)
    assert torch.equal(Wm.view(torch.int16), q.dequantize(wq).view(torch.int16))


@pytest.mark.slow
def test_merge_mlp_7b_gate_full_size_sampled(q):
    """The 7B-class gate projection (18944 x 3584, r = 64): merged on the
    GPU in full, compared on sampled rows (the oracle dequantises the sampled
    rows from the whole weight's double quantisation)."""
    wl = synth.WORKLOADS["mlp_7b"]
    N, K = wl.weights[0]
    W = synth.weight(N, K, wl.seed(synth.TID_W), "bf16")
    A = synth.activations(wl.r, K, wl.seed(synth.TID_A), sigma=0.02)
    B = synth.activations(N, wl.r, wl.seed(synth.TID_B), sigma=0.02)
    wq = q.quantize(W.cuda(), double_quant=True)
    Wm = q.merge(wq, A.cuda(), B.cuda(), wl.alpha)
    assert q.qlora_check_status() == 0
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.choice(N, 64, replace=False), [0, N - 1]]))
    Wn = W.float().numpy()
    a = oracle.block_absmax(Wn)
    qa, s, mu = oracle.double_quantize(a)
    ah = oracle.dq_absmax(qa, s, mu)
    nbr = K // 64
    deq = np.concatenate([
        oracle.dequantize(oracle.pack(oracle.quantize(Wn[r:r + 1])[0]), ah[r * nbr:(r + 1) * nbr], (1, K))
        for r in rows])
    ref = oracle.merge(deq, A.float().numpy(), B.float().numpy()[rows], wl.alpha, wl.r)
    _check(Wm[rows], ref)
