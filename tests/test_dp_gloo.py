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


# ---------------------------------------------------------------------------
# Row-sharded quantisation: the histogram exchange and the gather
# ---------------------------------------------------------------------------

def _exp_hist(a: np.ndarray) -> np.ndarray:
    """Exponent histogram of fp32 absmax values: bin e = sum of the 24-bit
    significands of the values whose exponent field is e (test-side
    restatement of the exchanged quantity)."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.int64)
    e = u >> 23
    m = (u & 0x7FFFFF) | np.where(e > 0, 0x800000, 0)
    h = np.zeros(256, dtype=np.int64)
    np.add.at(h, e, m)
    return h


def test_shard_rows_cover_and_align():
    from qlora_linear_layers_b200 import dp
    for rows, cols in ((28672, 8192), (18944, 3584), (3584, 18944), (35, 4096), (7, 192)):
        align = dp.row_alignment(cols)
        assert (align * cols // 64) % 256 == 0
        for world in (1, 2, 3, 4, 8):
            b = [dp.shard_rows(rows, cols, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == rows
            assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))
            assert all(r0 % align == 0 for r0, _ in b)
            sizes = [r1 - r0 for r0, r1 in b]
            assert max(sizes) - min(sizes) <= align


def _hist_worker(rank: int, world: int, port: int, out) -> None:
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import ctypes as C
        import oracle
        import qlora_linear_layers_b200 as q
        from qlora_linear_layers_b200 import _lib, dp, synth
        from qlora_linear_layers_b200.build import build
        build()
        rows, cols = 70, 4096
        W = synth.weight(rows, cols, 4711, "bf16").float().numpy()
        r0, r1 = dp.shard_rows(rows, cols, world, rank)
        # this rank's histogram, summed over ranks through the dp helper
        h = torch.from_numpy(_exp_hist(oracle.block_absmax(W[r0:r1]) if r1 > r0 else np.zeros(0)))
        dp._allreduce_sum(h)
        mean = C.c_float(0.0)
        hp = h.numpy().ctypes.data_as(C.POINTER(C.c_int64))
        st = _lib.load().qlora_dq_mean_from_hist(hp, rows * cols // 64, C.byref(mean))
        # gather of the shards of the whole-tensor quantisation (oracle-made)
        codes, a = oracle.quantize(W)
        qa, s, mu = oracle.double_quantize(a)
        packed = oracle.pack(codes)
        nb = cols // 64
        sh = q.empty_quantized(r1 - r0, cols, torch.device("cpu"))
        sh.packed.copy_(torch.from_numpy(packed[r0 * cols // 2:r1 * cols // 2]))
        sh.absmax.copy_(torch.from_numpy(a[r0 * nb:r1 * nb]))
        sh.qabsmax.copy_(torch.from_numpy(qa[r0 * nb:r1 * nb]))
        g0, g1 = r0 * nb // 256, (r1 * nb + 255) // 256
        sh.dq_scale.copy_(torch.from_numpy(s[g0:g1]))
        sh.dq_mean.fill_(float(mu))
        full = dp.allgather_quantized(q, sh, rows, world)
        out.put((rank, dict(st=st, mean=mean.value, hist=h.numpy(),
                            ok_gather=bool(np.array_equal(full.packed.numpy(), packed)
                                           and np.array_equal(full.qabsmax.numpy(), qa)
                                           and np.array_equal(full.absmax.numpy(), a)
                                           and np.array_equal(full.dq_scale.numpy(), s)
                                           and float(full.dq_mean[0]) == float(mu)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_histogram_gives_the_whole_tensor_mean(world):
    """Ranks quantise row shards; their exponent histograms summed over ranks
    (gloo all-reduce) give, through the library's host finalisation, the
    oracle's mean of the whole tensor bit for bit; and the gather of the
    shards reassembles the whole quantised weight."""
    import oracle
    from qlora_linear_layers_b200 import synth
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_hist_worker, args=(rk, world, port, out)) for rk in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W = synth.weight(70, 4096, 4711, "bf16").float().numpy()
    a = oracle.block_absmax(W)
    mu = oracle.dq_mean(a)
    for rk in range(world):
        r = res[rk]
        assert r["st"] == 0
        assert np.array_equal(r["hist"], _exp_hist(a))
        assert np.float32(r["mean"]).view(np.uint32) == np.float32(mu).view(np.uint32)
        assert r["ok_gather"]
