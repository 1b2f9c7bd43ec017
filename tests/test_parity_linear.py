"""GPU parity of the QLoRA linear layer (forward, backward) against the oracle.

Bar: max|GPU - oracle| / max|oracle| <= 1e-2 per output tensor (bf16 inputs,
fp32 accumulation, bf16 outputs; the oracle is fp64 on the same bf16 inputs
and the oracle's own dequantised weight, which the quantisation tests show
equals the GPU's bit for bit).  The bf16 rounding of the output alone is
2^-9 relative; a dropped adapter term is >= 4 % of max|Y| on these
workloads, so the bar separates right from wrong.

Two cases are exact: with X = identity and A = 0 the forward returns the
in-GEMM dequantised weights, which must equal nf4_dequantize bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
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
    g = got.float().cpu().numpy().astype(np.float64) if torch.is_tensor(got) else got
    return float(np.max(np.abs(g - ref)) / np.max(np.abs(ref)))


def _oracle_weight(wq, W_cpu):
    table = oracle.fp4_table() if wq.quant_type == 1 else oracle.nf4_table()
    codes, a = oracle.quantize(W_cpu.float().numpy(), table)
    if wq.double_quant:
        fmt = "fp8" if int(wq.double_quant) == 2 else "int8"
        qa, s, mu = oracle.double_quantize(a, fmt=fmt)
        a = oracle.dq_absmax(qa, s, mu, fmt=fmt)
    return oracle.dequantize(oracle.pack(codes), a, tuple(W_cpu.shape), table=table)


def _layer(q, N, K, M, r, alpha, seed, dq=True, wdtype="bf16", qt=0):
    W = synth.weight(N, K, seed + 1, wdtype)
    X = synth.activations(M, K, seed + 2)
    A = synth.activations(r, K, seed + 3, sigma=0.02)
    B = synth.activations(N, r, seed + 4, sigma=0.02)
    wq = q.quantize(W.cuda(), double_quant=dq, quant_type=qt)
    return W, X, A, B, wq


@pytest.mark.parametrize("N,K,M,r,alpha,dq", [
    (1024, 1024, 16, 8, 16.0, True),       # tiny round-trip workload
    (1024, 1024, 16, 8, 16.0, False),
    (200, 192, 300, 16, 32.0, True),       # ragged N and M tiles, 3 K steps
    (384, 512, 257, 32, 8.0, True),
    (256, 640, 513, 64, 16.0, True),
    (136, 256, 700, 128, 64.0, False),
    (96, 256, 300, 16, 32.0, True),        # N <= 128: the single-SM GEMM engine
    (128, 192, 257, 8, 16.0, False),
    (512, 1024, 1, 16, 32.0, True),        # decode-sized token counts
    (512, 1024, 4, 16, 32.0, True),
    (512, 1024, 17, 16, 32.0, True),
])
def test_forward_small(q, N, K, M, r, alpha, dq):
    W, X, A, B, wq = _layer(q, N, K, M, r, alpha, seed=100 * M + r, dq=dq, wdtype="bf16")
    Y, T = q.linear_fwd(wq, X.cuda(), A.cuda(), B.cuda(), alpha)
    assert q.qlora_check_status() == 0
    Wd = _oracle_weight(wq, W)
    Yr, Tr = oracle.linear_fwd(X.float().numpy(), Wd, A.float().numpy(), B.float().numpy(), alpha, r)
    assert rel_err(Y, Yr) <= TOL
    assert rel_err(T, Tr) <= TOL


@pytest.mark.parametrize("N,K,M,r,dq", [
    (1024, 1024, 16, 8, False),            # decode GEMV: fewer units than SMs
    (512, 1024, 1, 16, True),
    (64, 4096, 3, 8, True),                # one row group split over many CTAs
    (200, 192, 300, 16, True),             # tensor-core GEMM path
])
def test_forward_ignores_workspace_contents(q, N, K, M, r, dq):
    """Every workspace byte the forward reads is written earlier in the same
    call: a workspace full of NaN bytes changes nothing."""
    W, X, A, B, wq = _layer(q, N, K, M, r, 16.0, seed=7000 + M, dq=dq)
    ws = torch.full((q.workspace_bytes(1, M, N, K, r),), 0xFF, dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    T = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    q.qlora_linear_fwd(wq, X.cuda(), A.cuda(), B.cuda(), 16.0, Y, T, ws)
    assert q.qlora_check_status() == 0
    Yr, Tr = oracle.linear_fwd(X.float().numpy(), _oracle_weight(wq, W), A.float().numpy(),
                               B.float().numpy(), 16.0, r)
    assert torch.isfinite(Y.float()).all() and torch.isfinite(T.float()).all()
    assert rel_err(Y, Yr) <= TOL
    assert rel_err(T, Tr) <= TOL


@pytest.mark.parametrize("N,K,M,r,alpha,dq", [
    (1024, 1024, 16, 8, 16.0, True),
    (200, 192, 300, 16, 32.0, True),
    (256, 640, 513, 64, 16.0, False),
    (96, 256, 300, 16, 32.0, True),
    (512, 1024, 1, 16, 32.0, True),
    (512, 1024, 4, 16, 32.0, False),
])
def test_forward_small_fp4(q, N, K, M, r, alpha, dq):
    """The FP4 storage type through the same kernels (the table is the only
    difference)."""
    W, X, A, B, wq = _layer(q, N, K, M, r, alpha, seed=300 * M + r, dq=dq, qt=1)
    Y, T = q.linear_fwd(wq, X.cuda(), A.cuda(), B.cuda(), alpha)
    assert q.qlora_check_status() == 0
    Wd = _oracle_weight(wq, W)
    Yr, Tr = oracle.linear_fwd(X.float().numpy(), Wd, A.float().numpy(), B.float().numpy(), alpha, r)
    assert rel_err(Y, Yr) <= TOL
    assert rel_err(T, Tr) <= TOL


@pytest.mark.parametrize("N,K,M,r,alpha", [
    (384, 512, 300, 16, 32.0),
    (96, 256, 300, 16, 32.0),
    (512, 1024, 4, 16, 32.0),
])
def test_forward_backward_fp8_scales(q, N, K, M, r, alpha):
    """Block scales double-quantised to E4M3 codes (double_quant = 2) in the
    forward GEMM engines, the decode kernel and the backward."""
    W, X, A, B, wq = _layer(q, N, K, M, r, alpha, seed=500 + M + r, dq=2)
    dY = synth.activations(M, N, 511 + M)
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    Y, T = q.linear_fwd(wq, Xc, Ac, Bc, alpha)
    dX, dA, dB = q.linear_bwd(wq, Xc, dYc, Ac, Bc, alpha, T=T)
    assert q.qlora_check_status() == 0
    Wd = _oracle_weight(wq, W)
    Xn, An, Bn, dYn = (t.float().numpy() for t in (X, A, B, dY))
    Yr, Tr = oracle.linear_fwd(Xn, Wd, An, Bn, alpha, r)
    dXr, dAr, dBr = oracle.linear_bwd(Xn, dYn, Wd, An, Bn, alpha, r)
    assert rel_err(Y, Yr) <= TOL and rel_err(T, Tr) <= TOL
    assert rel_err(dX, dXr) <= TOL and rel_err(dA, dAr) <= TOL and rel_err(dB, dBr) <= TOL


@pytest.mark.parametrize("qt,dq", [(0, 1), (1, 1), (0, 2)])
def test_forward_identity_is_exact_dequant(q, qt, dq):
    """X = I, A = 0: Y[m, n] = W'[n, m] exactly (one nonzero product per sum)."""
    N, K = 384, 512
    W = synth.weight(N, K, 4242, "bf16")
    wq = q.quantize(W.cuda(), double_quant=dq, quant_type=qt)
    X = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")
    B = synth.activations(N, 16, 4243, sigma=0.02).cuda()
    Y, _ = q.linear_fwd(wq, X, A, B, 32.0)
    Wdeq = q.dequantize(wq)
    assert q.qlora_check_status() == 0
    assert torch.equal(Y.t().contiguous().view(torch.int16), Wdeq.view(torch.int16))
    Wd = _oracle_weight(wq, W)
    assert np.array_equal(Y.t().float().cpu().numpy(), Wd)


@pytest.mark.parametrize("qt,dq,M", [(0, 1, 1), (0, 1, 16), (1, 1, 9), (0, 2, 4), (0, 0, 8)])
def test_decode_onehot_tokens_exact(q, qt, dq, M):
    """Decode path (M <= 16) with one-hot token rows and A = 0: every output
    is one table value times one block scale, so Y equals, bit for bit, the
    decode path's reading of the weight, RNbf16(RN32(a^ * RNbf16(q[c]))) --
    which pins its row, block and column mapping and its scale decode."""
    N, K = 384, 1024
    W = synth.weight(N, K, 4300 + M, "bf16")
    wq = q.quantize(W.cuda(), double_quant=dq, quant_type=qt)
    cols = np.random.default_rng(M).choice(K, M, replace=False)
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[np.arange(M), torch.from_numpy(cols)] = 1.0
    A = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")
    B = synth.activations(N, 16, 4301, sigma=0.02).cuda()
    Y, _ = q.linear_fwd(wq, X.cuda(), A, B, 32.0)
    assert q.qlora_check_status() == 0
    table = oracle.fp4_table() if qt == 1 else oracle.nf4_table()
    codes, a = oracle.quantize(W.float().numpy(), table)
    if dq:
        fmt = "fp8" if dq == 2 else "int8"
        a = oracle.dq_absmax(*oracle.double_quantize(a, fmt=fmt), fmt=fmt)
    codes = np.asarray(codes).reshape(N, K)
    ah = np.asarray(a, dtype=np.float32).reshape(N, K // 64)
    qb = oracle.round_bf16(np.asarray(table, dtype=np.float32))
    Yg = Y.float().cpu().numpy()
    for m, k in enumerate(cols):
        expect = oracle.round_bf16((ah[:, k // 64] * qb[codes[:, k]]).astype(np.float32))
        assert np.array_equal(Yg[m], expect), (m, k)


def test_forward_adapter_only(q):
    """W = 0 quantises to the exact-zero row everywhere: Y = s (X A^T) B^T."""
    N, K, M, r, alpha = 256, 512, 300, 16, 32.0
    W = torch.zeros(N, K, dtype=torch.bfloat16)
    X = synth.activations(M, K, 5001)
    A = synth.activations(r, K, 5002, sigma=0.02)
    B = synth.activations(N, r, 5003, sigma=0.02)
    wq = q.quantize(W.cuda(), double_quant=True)
    Y, _ = q.linear_fwd(wq, X.cuda(), A.cuda(), B.cuda(), alpha)
    assert q.qlora_check_status() == 0
    Yr, _ = oracle.linear_fwd(X.float().numpy(), np.zeros((N, K)), A.float().numpy(),
                              B.float().numpy(), alpha, r)
    assert rel_err(Y, Yr) <= TOL


def _sampled_forward(q, W, X, A, B, alpha, r, nrows=48, seed=0):
    wq = q.quantize(W.cuda(), double_quant=True)
    Y, T = q.linear_fwd(wq, X.cuda(), A.cuda(), B.cuda(), alpha)
    assert q.qlora_check_status() == 0
    rng = np.random.default_rng(seed)
    M = X.shape[0]
    rows = np.unique(np.concatenate([rng.choice(M, nrows, replace=False), [0, M - 1]]))
    Wd = _oracle_weight(wq, W)
    Yr, _ = oracle.linear_fwd(X[rows].float().numpy(), Wd, A.float().numpy(), B.float().numpy(),
                              alpha, r)
    assert rel_err(Y[rows], Yr) <= TOL


@pytest.mark.slow
def test_forward_attn_proj_full_size_sampled(q):
    wl = synth.WORKLOADS["attn_proj_4096"]
    W, X, A, B = synth.layer_inputs(wl, 0)
    _sampled_forward(q, W, X, A, B, wl.alpha, wl.r)


@pytest.mark.slow
def test_forward_mlp_7b_full_size_sampled(q):
    wl = synth.WORKLOADS["mlp_7b"]
    for which in range(3):
        W, X, A, B = synth.layer_inputs(wl, which)
        _sampled_forward(q, W, X, A, B, wl.alpha, wl.r, seed=which)


# ---------------------------------------------------------------------------
# Backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,M,r,alpha,pass_T", [
    (256, 512, 300, 16, 32.0, True),
    (256, 512, 300, 16, 32.0, False),
    (200, 192, 257, 8, 16.0, True),        # N not a multiple of 64: partial contraction step
    (384, 256, 513, 64, 128.0, False),
    (136, 320, 100, 128, 64.0, True),
    (512, 128, 300, 16, 32.0, True),       # K <= 128: dX on the single-SM GEMM engine
    (256, 64, 100, 8, 16.0, False),
    (512, 1024, 1, 16, 32.0, False),       # decode-sized token counts
    (512, 1024, 4, 16, 32.0, True),
])
def test_backward_small(q, N, K, M, r, alpha, pass_T):
    W, X, A, B, wq = _layer(q, N, K, M, r, alpha, seed=7 * M + r)
    dY = synth.activations(M, N, 7 * M + r + 5)
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    _, T = q.linear_fwd(wq, Xc, Ac, Bc, alpha)
    dX, dA, dB = q.linear_bwd(wq, Xc, dYc, Ac, Bc, alpha, T=T if pass_T else None)
    assert q.qlora_check_status() == 0
    Wd = _oracle_weight(wq, W)
    dXr, dAr, dBr = oracle.linear_bwd(X.float().numpy(), dY.float().numpy(), Wd,
                                      A.float().numpy(), B.float().numpy(), alpha, r)
    assert rel_err(dX, dXr) <= TOL
    assert rel_err(dA, dAr) <= TOL
    assert rel_err(dB, dBr) <= TOL


@pytest.mark.parametrize("N,K,M,r,alpha,pass_T", [
    (256, 512, 300, 16, 32.0, True),
    (512, 128, 300, 16, 32.0, False),
])
def test_backward_small_fp4(q, N, K, M, r, alpha, pass_T):
    W, X, A, B, wq = _layer(q, N, K, M, r, alpha, seed=11 * M + r, qt=1)
    dY = synth.activations(M, N, 11 * M + r + 5)
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    _, T = q.linear_fwd(wq, Xc, Ac, Bc, alpha)
    dX, dA, dB = q.linear_bwd(wq, Xc, dYc, Ac, Bc, alpha, T=T if pass_T else None)
    assert q.qlora_check_status() == 0
    Wd = _oracle_weight(wq, W)
    dXr, dAr, dBr = oracle.linear_bwd(X.float().numpy(), dY.float().numpy(), Wd,
                                      A.float().numpy(), B.float().numpy(), alpha, r)
    assert rel_err(dX, dXr) <= TOL
    assert rel_err(dA, dAr) <= TOL
    assert rel_err(dB, dBr) <= TOL


def test_backward_adapter_gradients_only(q):
    """W = 0: dX = s U A only, dA and dB unchanged by the base weight."""
    N, K, M, r, alpha = 256, 384, 200, 32, 64.0
    W = torch.zeros(N, K, dtype=torch.bfloat16)
    X = synth.activations(M, K, 6001)
    A = synth.activations(r, K, 6002, sigma=0.02)
    B = synth.activations(N, r, 6003, sigma=0.02)
    dY = synth.activations(M, N, 6004)
    wq = q.quantize(W.cuda())
    dX, dA, dB = q.linear_bwd(wq, X.cuda(), dY.cuda(), A.cuda(), B.cuda(), alpha)
    assert q.qlora_check_status() == 0
    dXr, dAr, dBr = oracle.linear_bwd(X.float().numpy(), dY.float().numpy(), np.zeros((N, K)),
                                      A.float().numpy(), B.float().numpy(), alpha, r)
    assert rel_err(dX, dXr) <= TOL and rel_err(dA, dAr) <= TOL and rel_err(dB, dBr) <= TOL


@pytest.mark.slow
def test_backward_4096_full_size(q):
    """The full backward workload: dA, dB compared in full, dX on sampled rows."""
    wl = synth.WORKLOADS["bwd_4096"]
    W, X, A, B = synth.layer_inputs(wl, 0)
    dY = synth.upstream_grad(wl, 0)
    wq = q.quantize(W.cuda(), double_quant=True)
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    _, T = q.linear_fwd(wq, Xc, Ac, Bc, wl.alpha)
    dX, dA, dB = q.linear_bwd(wq, Xc, dYc, Ac, Bc, wl.alpha, T=T)
    assert q.qlora_check_status() == 0
    Xn, An, Bn, dYn = (t.float().numpy() for t in (X, A, B, dY))
    dAr, dBr = oracle.linear_bwd_adapters(Xn, dYn, An, Bn, wl.alpha, wl.r)
    assert rel_err(dA, dAr) <= TOL
    assert rel_err(dB, dBr) <= TOL
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([rng.choice(wl.M, 48, replace=False), [0, wl.M - 1]]))
    Wd = _oracle_weight(wq, W)
    dXr, _, _ = oracle.linear_bwd(Xn[rows], dYn[rows], Wd, An, Bn, wl.alpha, wl.r)
    assert rel_err(dX[rows], dXr) <= TOL


# ---------------------------------------------------------------------------
# Decode (M <= 16) at full size
# ---------------------------------------------------------------------------

def _oracle_weight_rows(W_cpu, rows):
    """Dequantised rows of a double-quantised weight, all by the oracle: the
    DQ constants come from every block's absmax, the codes of `rows` only
    (blocks never straddle rows)."""
    Wn = W_cpu.float().numpy()
    a = oracle.block_absmax(Wn)
    qa, s, mu = oracle.double_quantize(a)
    ah = oracle.dq_absmax(qa, s, mu)
    nbr = Wn.shape[1] // 64
    out = []
    for r in rows:
        codes, _ = oracle.quantize(Wn[r:r + 1])
        out.append(oracle.dequantize(oracle.pack(codes), ah[r * nbr:(r + 1) * nbr], (1, Wn.shape[1])))
    return np.concatenate(out, axis=0)


@pytest.mark.slow
@pytest.mark.parametrize("outliers", [False, True])
def test_decode_70b_full_size(q, outliers):
    wl = synth.WORKLOADS["decode_70b"]
    W = synth.weight(28672, 8192, wl.seed(synth.TID_W), "bf16", outliers=outliers)
    wq = q.quantize(W.cuda(), double_quant=True)
    rng = np.random.default_rng(5 + int(outliers))
    rows = np.unique(np.concatenate([rng.choice(28672, 96, replace=False), [0, 28671]]))
    Wd = _oracle_weight_rows(W, rows)
    A = synth.activations(wl.r, 8192, wl.seed(synth.TID_A), sigma=0.02)
    B = synth.activations(28672, wl.r, wl.seed(synth.TID_B), sigma=0.02)
    for M in wl.decode_M:
        X = synth.activations(M, 8192, wl.seed(synth.TID_X) + M)
        Y, _ = q.linear_fwd(wq, X.cuda(), A.cuda(), B.cuda(), wl.alpha)
        assert q.qlora_check_status() == 0
        Yr, _ = oracle.linear_fwd(X.float().numpy(), Wd, A.float().numpy(),
                                  B.float().numpy()[rows], wl.alpha, wl.r)
        assert rel_err(Y[:, rows], Yr) <= TOL
