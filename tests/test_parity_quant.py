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


NF4, FP4 = 0, 1


def _table(qt):
    return oracle.nf4_table() if qt == NF4 else oracle.fp4_table()


def _check_full(q, W_cpu, double_quant=True, qt=NF4):
    Wd = W_cpu.cuda()
    wq = q.quantize(Wd, double_quant=double_quant, quant_type=qt)
    Wdeq = q.dequantize(wq)
    assert q.qlora_check_status() == 0
    Wnp = W_cpu.float().numpy()
    table = _table(qt)
    codes, a = oracle.quantize(Wnp, table)
    assert np.array_equal(_np(wq.packed), oracle.pack(codes))
    assert np.array_equal(_np(wq.absmax).view(np.uint32), a.view(np.uint32))
    if double_quant:
        fmt = "fp8" if int(double_quant) == 2 else "int8"
        qa, s, mu = oracle.double_quantize(a, fmt=fmt)
        assert np.array_equal(_np(wq.qabsmax), qa)
        assert np.array_equal(_np(wq.dq_scale).view(np.uint32), s.view(np.uint32))
        assert _np(wq.dq_mean)[0].view(np.uint32) == np.float32(mu).view(np.uint32)
        ah = oracle.dq_absmax(qa, s, mu, fmt=fmt)
    else:
        ah = a
    ref = oracle.dequantize(oracle.pack(codes), ah, Wnp.shape, table=table)
    got = Wdeq.float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    return wq


@pytest.mark.parametrize("qt", [NF4, FP4])
def test_tiny_roundtrip_fp32(q, qt):
    wl = synth.WORKLOADS["tiny_roundtrip"]
    W = synth.weight(1024, 1024, wl.seed(synth.TID_W), "fp32")
    _check_full(q, W, True, qt)
    _check_full(q, W, False, qt)


@pytest.mark.parametrize("qt", [NF4, FP4])
def test_attn_proj_bf16(q, qt):
    wl = synth.WORKLOADS["attn_proj_4096"]
    W = synth.weight(4096, 4096, wl.seed(synth.TID_W), "bf16")
    _check_full(q, W, True, qt)


@pytest.mark.parametrize("rows,cols,outliers", [(4096, 4096, False), (300, 4096, True), (5, 64 * 257, False)])
def test_fp8_double_quant(q, rows, cols, outliers):
    """8-bit float block-scale codes (double_quant = 2): codes, E4M3 scale
    bytes (signed zeros included), group scales, mean and the dequantised
    weights bit for bit."""
    W = synth.weight(rows, cols, 880 + rows, "bf16", outliers=outliers)
    _check_full(q, W, 2)
    _check_full(q, W, 2, FP4)


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 6400), (7, 192), (5, 64 * 257)])
def test_ragged_shapes(q, rows, cols):
    """Single block, partial last DQ group (300 and 1285 scales), odd rows."""
    W = synth.weight(rows, cols, 77 + rows, "bf16")
    _check_full(q, W, True)
    _check_full(q, W, True, FP4)


def test_standalone_double_quantize(q):
    """nf4_double_quantize on an absmax array (its own histogram pass) equals
    the oracle, and the fused quantise + histogram path."""
    W = synth.weight(300, 4096, 991, "bf16")
    wq = q.quantize(W.cuda(), double_quant=True)
    qa = torch.empty_like(wq.qabsmax)
    sc = torch.empty_like(wq.dq_scale)
    mu = torch.empty(4, dtype=torch.float32, device="cuda")[:1]
    q.nf4_double_quantize(wq.absmax, qa, sc, mu)
    assert q.qlora_check_status() == 0
    a = oracle.block_absmax(W.float().numpy())
    qa_r, s_r, mu_r = oracle.double_quantize(a)
    assert np.array_equal(_np(qa), qa_r) and np.array_equal(_np(qa), _np(wq.qabsmax))
    assert np.array_equal(_np(sc).view(np.uint32), s_r.view(np.uint32))
    assert _np(mu)[0].view(np.uint32) == np.float32(mu_r).view(np.uint32)


@pytest.mark.parametrize("splits", [(2, 4), (1, 3, 8)])
def test_row_sharded_quantise_matches_whole(q, splits):
    """A weight quantised in row shards -- each shard its own histogram, the
    histograms summed, each shard's DQ finalised from the sum over the whole
    count -- equals the whole weight's quantisation bit for bit (the shard
    boundaries fall on groups of 256 scales: 4 rows of 4096 columns)."""
    rows, cols = 8 * 4 + 3, 4096
    W = synth.weight(rows, cols, 515, "bf16").cuda()
    bounds = [0] + [4 * k for k in splits] + [rows]
    whole = q.quantize(W, double_quant=True)
    parts = []
    hist = torch.zeros(256, dtype=torch.int64, device="cuda")
    for r0, r1 in zip(bounds[:-1], bounds[1:]):
        t = q.empty_quantized(r1 - r0, cols, W.device)
        h = torch.empty(256, dtype=torch.int64, device="cuda")
        q.qlora_quantize_4bit(W[r0:r1].contiguous(), t.packed, t.absmax, 0, h)
        hist += h
        parts.append(t)
    n_total = rows * cols // 64
    for t in parts:
        q.nf4_double_quantize_hist(t.absmax, hist, n_total, t.qabsmax, t.dq_scale, t.dq_mean)
    assert q.qlora_check_status() == 0
    cat = lambda name: torch.cat([getattr(t, name) for t in parts])
    assert torch.equal(cat("packed"), whole.packed)
    assert torch.equal(cat("absmax"), whole.absmax)
    assert torch.equal(cat("qabsmax"), whole.qabsmax)
    assert torch.equal(cat("dq_scale"), whole.dq_scale)
    for t in parts:
        assert torch.equal(t.dq_mean, whole.dq_mean)
    a = oracle.block_absmax(W.float().cpu().numpy())
    assert np.float32(oracle.dq_mean(a)) == _np(whole.dq_mean)[0]


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
        _check_full(q, Wt, False, FP4)


@pytest.mark.parametrize("qt", [NF4, FP4])
def test_threshold_values_every_part(q, qt):
    # fp32 blocks whose absmax is exactly 1, with the weights T - 1 ulp, T and
    # T + 1 ulp (T a decision threshold of the table) placed in one of the
    # threads' parts of each block, part by part: the quotient lands within a
    # few ulp of T, so that part is coded by the exact (IEEE division) path
    # and the block's other parts by the fast path; ties go up.
    rng = np.random.default_rng(33)
    thr = oracle.thresholds(_table(qt))
    W = (rng.standard_normal((24, 512)) * 0.1).clip(-0.5, 0.5).astype(np.float32)
    nblk = W.size // 64
    Wb = W.reshape(nblk, 64)
    for b in range(nblk):
        Wb[b, 63 - (b % 7)] = 1.0 if b % 2 else -1.0          # the block's absmax
        T = thr[b % thr.size]
        part = b % 4                                            # a 16-weight part
        lo = part * 16 + 3
        Wb[b, lo] = np.nextafter(T, np.float32(-np.inf))
        Wb[b, lo + 1] = T
        Wb[b, lo + 2] = np.nextafter(T, np.float32(np.inf))
    Wt = torch.from_numpy(Wb.reshape(W.shape).copy())
    _check_full(q, Wt, True, qt)
    _check_full(q, Wt, False, qt)


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
