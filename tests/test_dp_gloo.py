"""The data-parallel host logic on CPU: two `gloo` ranks, each with its own
tokens and the same replicated weight and adapter factors, sum their adapter
gradients with ``dp.allreduce_adapter_grads``.  The result must be the same
on both ranks and equal the oracle's gradients of the concatenated batch (dA
and dB are sums over tokens: page "LoRA vs QLoRA: Efficient Fine-Tuning
Explained", section "How QLoRA Works" -- only the adapters are trained)."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

N, K, M, R, ALPHA = 96, 128, 24, 8, 16.0


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out) -> None:
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from qlora_linear_layers_b200 import dp, synth
        W = synth.weight(N, K, dp.replica_seed(11, rank), "bf16").float().numpy()
        A = synth.activations(R, K, dp.replica_seed(13, rank), sigma=0.02).float().numpy()
        B = synth.activations(N, R, dp.replica_seed(14, rank), sigma=0.02).float().numpy()
        X = synth.activations(M, K, dp.token_seed(12, rank)).float().numpy()
        dY = synth.activations(M, N, dp.token_seed(15, rank)).float().numpy()
        dA, dB = oracle.linear_bwd_adapters(X, dY, A, B, ALPHA, R)
        dA_t, dB_t = torch.from_numpy(dA.copy()), torch.from_numpy(dB.copy())
        dp.allreduce_adapter_grads(dA_t, dB_t)
        out.put((rank, dict(W=W, A=A, B=B, X=X, dY=dY, dA=dA_t.numpy(), dB=dB_t.numpy())))
    finally:
        dist.destroy_process_group()


def test_two_rank_adapter_gradient_sum():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rk, world, port, out)) for rk in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    r0, r1 = res[0], res[1]
    # replicas are identical, tokens are not
    for k in ("W", "A", "B"):
        assert np.array_equal(r0[k], r1[k]), k
    assert not np.array_equal(r0["X"], r1["X"])
    assert not np.array_equal(r0["dY"], r1["dY"])
    # both ranks hold the same summed gradients
    assert np.array_equal(r0["dA"], r1["dA"]) and np.array_equal(r0["dB"], r1["dB"])
    # ... equal to the gradients of the concatenated batch
    import oracle
    X = np.concatenate([r0["X"], r1["X"]])
    dY = np.concatenate([r0["dY"], r1["dY"]])
    dA_ref, dB_ref = oracle.linear_bwd_adapters(X, dY, r0["A"], r0["B"], ALPHA, R)
    np.testing.assert_allclose(r0["dA"], dA_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r0["dB"], dB_ref, rtol=1e-12, atol=1e-14)
    # and differ from one rank's own gradients (the exchange did something)
    dA_0, _ = oracle.linear_bwd_adapters(r0["X"], r0["dY"], r0["A"], r0["B"], ALPHA, R)
    assert np.max(np.abs(dA_0 - r0["dA"])) > 1e-3 * np.max(np.abs(dA_ref))
