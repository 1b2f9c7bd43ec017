"""The library under data parallelism on a GPU: two ranks (processes) share
cuda:0 and exchange through the gloo backend (host memory), so no kernel of
one rank ever waits on the other.

* Row-sharded quantisation: each rank quantises its rows with the histogram
  pass, the histograms are summed, each shard's 8-bit scales are finalised
  from the sum; the gathered weight equals the one-process quantisation bit
  for bit (page "QLoRA Explained", section "Shrink the scale factors too":
  the per-tensor mean is the one global quantity).
* Data-parallel training step: replicated weight and adapters, each rank its
  own tokens, forward and backward on the library, dA and dB summed over
  ranks; the sums match the oracle's gradients of the concatenated batch
  within the layer tolerance.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu
N, K, M, R, ALPHA = 384, 1024, 300, 16, 32.0
TOL = 1e-2


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
                            timeout=datetime.timedelta(seconds=120))
    try:
        import qlora_linear_layers_b200 as q
        from qlora_linear_layers_b200 import dp, synth
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        W = synth.weight(N, K, dp.replica_seed(901, rank), "bf16").to(dev)
        A = synth.activations(R, K, dp.replica_seed(903, rank), sigma=0.02).to(dev)
        B = synth.activations(N, R, dp.replica_seed(904, rank), sigma=0.02).to(dev)
        X = synth.activations(M, K, dp.token_seed(902, rank)).to(dev)
        dY = synth.activations(M, N, dp.token_seed(905, rank)).to(dev)
        r0, r1 = dp.shard_rows(N, K, world, rank)
        shard = dp.quantize_sharded(q, W[r0:r1].contiguous(), N, r0)
        full = dp.allgather_quantized(q, shard, N, world)
        whole = q.quantize(W, double_quant=True)
        same = all(torch.equal(getattr(full, k), getattr(whole, k))
                   for k in ("packed", "absmax", "qabsmax", "dq_scale", "dq_mean"))
        _, T = q.linear_fwd(full, X, A, B, ALPHA)
        _, dA, dB = q.linear_bwd(full, X, dY, A, B, ALPHA, T=T)
        dp.allreduce_adapter_grads(dA, dB)
        st = q.qlora_check_status()
        out.put((rank, dict(same=same, st=st, dA=dA.float().cpu().numpy(),
                            dB=dB.float().cpu().numpy(), bounds=(r0, r1))))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_quantise_and_sum_gradients():
    import oracle
    from qlora_linear_layers_b200 import dp, synth
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rk, world, port, out)) for rk in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0]["bounds"] != res[1]["bounds"] and res[0]["bounds"][1] == res[1]["bounds"][0]
    for rk in range(world):
        assert res[rk]["st"] == 0
        assert res[rk]["same"]
    assert np.array_equal(res[0]["dA"], res[1]["dA"]) and np.array_equal(res[0]["dB"], res[1]["dB"])
    Xs = [synth.activations(M, K, dp.token_seed(902, rk)).float().numpy() for rk in range(world)]
    dYs = [synth.activations(M, N, dp.token_seed(905, rk)).float().numpy() for rk in range(world)]
    A = synth.activations(R, K, 903, sigma=0.02).float().numpy()
    B = synth.activations(N, R, 904, sigma=0.02).float().numpy()
    dAr, dBr = oracle.linear_bwd_adapters(np.concatenate(Xs), np.concatenate(dYs), A, B, ALPHA, R)
    rel = lambda g, r: float(np.max(np.abs(g - r)) / np.max(np.abs(r)))
    assert rel(res[0]["dA"], dAr) <= TOL
    assert rel(res[0]["dB"], dBr) <= TOL
