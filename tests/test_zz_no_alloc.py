"""qlora_linear_fwd_noalloc: the forward for callers that cannot allocate.

Callers such as a plugin inside a host program that owns every device
allocation, code running under CUDA stream capture, or a loop that forbids
allocation after start-up cannot provide a workspace.  This entry point keeps
its scratch in a fixed array inside the library.  The test calls it through
the C ABI twice in a row, on different layers, and checks each result against
the regular qlora_linear_fwd within the layer tests' tolerance (so nothing
from the first call leaks into the second), then checks that a layer too big
for the fixed scratch is refused before anything runs.

This file is named so that pytest collects it last.
"""

import ctypes as C

import numpy as np
import pytest
import torch

from qlora_linear_layers_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module")
def q():
    from qlora_linear_layers_b200.build import build
    build()
    import qlora_linear_layers_b200 as q
    return q


def _noalloc_fwd(q, wq, X, A, B, alpha, Y, T):
    lib = q._lib.load()
    cw = wq.c_struct()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.qlora_linear_fwd_noalloc(C.byref(cw), X.data_ptr(), X.shape[0], A.data_ptr(),
                                        B.data_ptr(), A.shape[0], float(alpha), Y.data_ptr(),
                                        None if T is None else T.data_ptr(), stream)


def _rel(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("first,second", [
    ((384, 512, 300, 16, 32.0), (200, 192, 1000, 64, 16.0)),
])
def test_noalloc_matches_regular_forward_twice(q, first, second):
    for i, (N, K, M, r, alpha) in enumerate((first, second)):
        W = synth.weight(N, K, 8100 + i, "bf16").cuda()
        X = synth.activations(M, K, 8200 + i).cuda()
        A = synth.activations(r, K, 8300 + i, sigma=0.02).cuda()
        B = synth.activations(N, r, 8400 + i, sigma=0.02).cuda()
        wq = q.quantize(W, double_quant=True)
        Y_ref, T_ref = q.linear_fwd(wq, X, A, B, alpha)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        T = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc_fwd(q, wq, X, A, B, alpha, Y, T) == q._lib.QLORA_OK
        assert q.qlora_check_status() == 0
        assert _rel(Y, Y_ref) <= TOL
        assert _rel(T, T_ref) <= TOL


def test_noalloc_rejects_layers_beyond_the_fixed_scratch(q):
    lib = q._lib.load()
    N, K, r = 256, 512, 64
    W = synth.weight(N, K, 8500, "bf16").cuda()
    wq = q.quantize(W, double_quant=True)
    M_big = q._lib.QLORA_FWD_NOALLOC_SCRATCH_BYTES // (64 * 2) + 1
    assert q.workspace_bytes(q._lib.QLORA_OP_FWD, M_big, N, K, r) > \
        q._lib.QLORA_FWD_NOALLOC_SCRATCH_BYTES
    X = torch.zeros(1, K, dtype=torch.bfloat16, device="cuda")      # never read: refused first
    A = torch.zeros(r, K, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(1, N, dtype=torch.bfloat16, device="cuda")
    cw = wq.c_struct()
    launches = lib.qlora_kernel_launches()
    st = lib.qlora_linear_fwd_noalloc(C.byref(cw), X.data_ptr(), M_big, A.data_ptr(), B.data_ptr(),
                                      r, 16.0, Y.data_ptr(), None,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == q._lib.QLORA_ERR_WORKSPACE
    assert lib.qlora_kernel_launches() == launches
    assert q.qlora_check_status() == 0
