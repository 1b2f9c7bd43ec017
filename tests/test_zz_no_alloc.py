"""qlora_linear_fwd_noalloc: the forward for callers that cannot allocate.

Callers such as a plugin inside a host program that owns every device
allocation, code running under CUDA stream capture, or a loop that forbids
allocation after start-up cannot provide a workspace.  This entry point keeps
its scratch in a fixed array inside the library.  The tests call it through
the C ABI several times in a row -- the tensor-core GEMM path (M > 16), the
decode path (M <= 16, whose scratch holds the GEMV's partial sums) and rank
128 -- and require each result to equal the regular qlora_linear_fwd bit for
bit: both run the same kernels on the same inputs, so any difference would
be scratch left over from an earlier call.  A layer too big for the fixed
scratch is refused before anything runs, and a malformed argument is
reported exactly as qlora_linear_fwd reports it.

This file is named so that pytest collects it last.
"""

import ctypes as C

import pytest
import torch

from qlora_linear_layers_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from qlora_linear_layers_b200.build import build
    build()
    import qlora_linear_layers_b200 as q
    return q


def _noalloc_fwd(q, wq, X, A, B, alpha, Y, T, M=None):
    lib = q._lib.load()
    cw = wq.c_struct()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.qlora_linear_fwd_noalloc(C.byref(cw), X.data_ptr(), X.shape[0] if M is None else M,
                                        A.data_ptr(), B.data_ptr(), A.shape[0], float(alpha),
                                        Y.data_ptr(), None if T is None else T.data_ptr(), stream)


# (N, K, M, r, alpha): GEMM path, decode path, GEMM path again, decode with
# one token, rank 128 on both paths
LAYERS = [
    (384, 512, 300, 16, 32.0),
    (200, 192, 1000, 64, 16.0),
    (1024, 1024, 16, 8, 16.0),
    (512, 1024, 700, 32, 8.0),
    (4096, 1024, 1, 16, 32.0),
    (256, 640, 513, 128, 64.0),
    (512, 1024, 4, 128, 64.0),
]


def test_noalloc_equals_regular_forward_call_after_call(q):
    for i, (N, K, M, r, alpha) in enumerate(LAYERS):
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
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), (N, K, M, r)
        assert torch.equal(T.view(torch.int16), T_ref.view(torch.int16)), (N, K, M, r)


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
    launches = lib.qlora_kernel_launches()
    assert _noalloc_fwd(q, wq, X, A, B, 16.0, Y, None, M=M_big) == q._lib.QLORA_ERR_WORKSPACE
    # a malformed argument wins over the size: the same error as the regular entry point
    bad = torch.zeros(1, 8, dtype=torch.bfloat16, device="cuda")
    Abad = bad[:, 1:]                                                  # 2-byte aligned
    st = lib.qlora_linear_fwd_noalloc(C.byref(wq.c_struct()), X.data_ptr(), M_big, Abad.data_ptr(),
                                      B.data_ptr(), r, 16.0, Y.data_ptr(), None,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == q._lib.QLORA_ERR_ALIGN
    assert lib.qlora_kernel_launches() == launches
    assert q.qlora_check_status() == 0
