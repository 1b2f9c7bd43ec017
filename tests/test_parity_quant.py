"""GPU parity: NF4 quantise, double quantise and dequantise vs the oracle.

All results must be bit-exact: packed codes, fp32 absmax, int8 qabsmax, fp32
group scales, the fp32 mean and the dequantised bf16 weights.  Small
workloads are compared in full; the full-size weights are quantised whole on
the GPU and their absmax and double quantisation compared in full against the
oracle's own (computed from the weight), the codes and dequantised weights on
sampled blocks (quantise and dequantise are local to a block).
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
    assert torch.cuda.is_available()
    return q


def _np(t):
    return t.detach().cpu().numpy()


def _check_full(q, W_cpu, double_quant=True):
    Wd = W_cpu.cuda()
    wq = q.quantize(Wd, double_quant=double_quant)
    Wdeq = q.dequantize(wq)
    assert q.qlora_check_status() == 0
    Wnp = W_cpu.float().numpy()
    codes, a = oracle.quantize(Wnp)
    assert np.array_equal(_np(wq.packed), oracle.pack(codes))
    assert np.array_equal(_np(wq.absmax).view(np.uint32), a.view(np.uint32))
    if double_quant:
        qa, s, mu = oracle.double_quantize(a)
        assert np.array_equal(_np(wq.qabsmax), qa)
        assert np.array_equal(_np(wq.dq_scale).view(np.uint32), s.view(np.uint32))
        assert _np(wq.dq_mean)[0].view(np.uint32) == np.float32(mu).view(np.uint32)
        ah = oracle.dq_absmax(qa, s, mu)
    else:
        ah = a
    ref = oracle.dequantize(oracle.pack(codes), ah, Wnp.shape)
    got = Wdeq.float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    return wq


def test_tiny_roundtrip_fp32(q):
    wl = synth.WORKLOADS["tiny_roundtrip"]
    W = synth.weight(1024, 1024, wl.seed(synth.TID_W), "fp32")
    _check_full(q, W, True)
    _check_full(q, W, False)


def test_attn_proj_bf16(q):
    wl = synth.WORKLOADS["attn_proj_4096"]
    W = synth.weight(4096, 4096, wl.seed(synth.TID_W), "bf16")
    _check_full(q, W, True)


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 6400), (7, 192), (5, 64 * 257)])
def test_ragged_shapes(q, rows, cols):
    """Single block, partial last DQ group (300 and 1285 scales), odd rows."""
    W = synth.weight(rows, cols, 77 + rows, "bf16")
    _check_full(q, W, True)


def test_edge_values(q):
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    W[0, :64] = 0.0                        # all-zero block
    W[1, :64] = -0.0                       # all negative-zero block
    W[1, 64:128] = 0.0
    W[1, 70] = -0.0
    W[2, :64] = 0.01                       # absmax repeated in every element
    W[3, :64] = -0.01
    W[4, :64] *= 1e30                      # huge magnitudes
    W[5, :64] *= 1e-35                     # tiny (subnormal ratios)
    W[6, 3] = 3.0                          # outlier
    W[7, 64:128] = np.float32(1e-45)       # smallest subnormal
    for dt in ("fp32", "bf16"):
        Wt = torch.from_numpy(W) if dt == "fp32" else torch.from_numpy(W).to(torch.bfloat16)
        _check_full(q, Wt, True)
        _check_full(q, Wt, False)


def test_nonfinite_sets_status(q):
    W = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    W[2, 5] = float("nan")
    q.quantize(W, double_quant=False)
    assert q.qlora_check_status() == q._lib.QLORA_ERR_NONFINITE
    assert q.qlora_check_status() == 0     # cleared
    W[2, 5] = float("inf")
    q.quantize(W, double_quant=False)
    assert q.qlora_check_status() == q._lib.QLORA_ERR_NONFINITE


def _sampled(q, W_cpu, nsample=96, seed=0):
    """Quantise the whole matrix on the GPU.  The oracle computes every block
    absmax and the double quantisation of the whole tensor from the weight
    itself (never from a GPU output); both are compared in full, the codes
    and dequantised weights on sampled blocks (they are local to a block)."""
    wq = q.quantize(W_cpu.cuda(), double_quant=True)
    Wdeq = q.dequantize(wq)
    assert q.qlora_check_status() == 0
    Wnp = W_cpu.float().numpy()
    a = oracle.block_absmax(Wnp)
    absmax = _np(wq.absmax)
    assert np.array_equal(absmax.view(np.uint32), a.view(np.uint32))
    qa, s, mu = oracle.double_quantize(a)
    assert np.array_equal(_np(wq.qabsmax), qa)
    assert np.array_equal(_np(wq.dq_scale).view(np.uint32), s.view(np.uint32))
    assert _np(wq.dq_mean)[0].view(np.uint32) == np.float32(mu).view(np.uint32)
    ah = oracle.dq_absmax(qa, s, mu)
    nblk = a.size
    rng = np.random.default_rng(seed)
    blocks = np.unique(np.concatenate([rng.choice(nblk, nsample, replace=False), [0, nblk - 1]]))
    Wflat = Wnp.reshape(-1, 64)
    packed = _np(wq.packed).reshape(-1, 32)
    deq = Wdeq.reshape(-1, 64)
    for b in blocks:
        codes, ab = oracle.quantize(Wflat[b:b + 1])
        assert ab[0].view(np.uint32) == a[b].view(np.uint32)
        assert np.array_equal(packed[b], oracle.pack(codes))
        ref = oracle.dequantize(oracle.pack(codes), ah[b:b + 1], (1, 64))
        assert np.array_equal(deq[b].float().cpu().numpy().view(np.uint32),
                              ref.reshape(-1).view(np.uint32))


@pytest.mark.slow
def test_decode_70b_full_size_sampled(q):
    wl = synth.WORKLOADS["decode_70b"]
    for outliers in (False, True):
        W = synth.weight(28672, 8192, wl.seed(synth.TID_W), "bf16", outliers=outliers)
        _sampled(q, W, seed=int(outliers))


@pytest.mark.slow
def test_mlp_7b_full_size_sampled(q):
    wl = synth.WORKLOADS["mlp_7b"]
    for which, (N, K) in enumerate(wl.weights):
        W = synth.weight(N, K, wl.seed(synth.TID_W, which), "bf16")
        _sampled(q, W, seed=which)
