"""Failure detection: a bounded wait that runs out reports QLORA_ERR_TIMEOUT
and leaves the context usable.

The test switch qlora_test_withhold_first_fill makes the decode kernel's
first CTA leave its first pipeline stage unfilled -- a barrier that nothing
completes.  With the wait limit shortened to 20 ms, that CTA's consumer
warps give up, raise the CTA's abort flag, the producer stops and waits
(bounded) for its copies in flight, and the call's status is
QLORA_ERR_TIMEOUT.  No fault, trap or unbounded wait is involved.  With the
switch off and the default limit restored, the same call is correct.
"""

import time

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


def test_decode_wait_runs_out_then_recovers(q):
    lib = q._lib.load()
    N, K, M, r, alpha = 512, 1024, 4, 16, 32.0
    W = synth.weight(N, K, 7301, "bf16")
    X = synth.activations(M, K, 7302).cuda()
    A = synth.activations(r, K, 7303, sigma=0.02).cuda()
    B = synth.activations(N, r, 7304, sigma=0.02).cuda()
    wq = q.quantize(W.cuda(), double_quant=True)
    assert q.qlora_check_status() == 0
    assert lib.qlora_set_wait_limit(20_000_000) == 0
    assert lib.qlora_test_withhold_first_fill(1) == 0
    try:
        t0 = time.perf_counter()
        q.linear_fwd(wq, X, A, B, alpha, save_T=False)
        st = q.qlora_check_status()
        elapsed = time.perf_counter() - t0
    finally:
        assert lib.qlora_test_withhold_first_fill(0) == 0
        assert lib.qlora_set_wait_limit(0) == 0
    assert st == q._lib.QLORA_ERR_TIMEOUT
    assert 0.015 < elapsed < 5.0                       # the waits ran out, bounded
    assert q.qlora_check_status() == 0                  # the word was cleared
    # the context is usable: the same call again, checked against the oracle
    Y, T = q.linear_fwd(wq, X, A, B, alpha)
    assert q.qlora_check_status() == 0
    codes, a = oracle.quantize(W.float().numpy())
    qa, s, mu = oracle.double_quantize(a)
    Wd = oracle.dequantize(oracle.pack(codes), oracle.dq_absmax(qa, s, mu), (N, K))
    Yr, _ = oracle.linear_fwd(X.float().cpu().numpy(), Wd, A.float().cpu().numpy(),
                              B.float().cpu().numpy(), alpha, r)
    err = np.max(np.abs(Y.float().cpu().numpy() - Yr)) / np.max(np.abs(Yr))
    assert err <= 1e-2
