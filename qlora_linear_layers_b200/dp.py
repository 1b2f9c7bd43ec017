"""Data-parallel plumbing of the QLoRA layer.

The layer is data-parallel: every rank holds the same frozen quantised weight
and the same adapter factors A, B, and takes its own tokens.  Two exchanges
exist on the path:

* the sum of the adapter gradients dA, dB over ranks (page "LoRA vs QLoRA:
  Efficient Fine-Tuning Explained", section "How QLoRA Works": only the
  adapters are trained, so only their gradients cross ranks).  Both are sums
  over tokens, so the sum over ranks equals the gradient of the concatenated
  batch;
* when the quantisation of the frozen weight is itself split over ranks (each
  rank quantises a range of rows), the double quantisation's per-tensor mean
  (page "QLoRA Explained", section "Shrink the scale factors too") is the one
  global quantity: each rank's exponent histogram of its block absmax values
  is summed with an integer all-reduce -- exact and order-free, so the mean
  is bit-identical to quantising on one device -- and the shards are then
  gathered so that every rank holds the whole quantised weight.

All collectives go through torch.distributed (NCCL on GPUs); with the gloo
backend, device tensors are staged through host memory.
"""

from __future__ import annotations

import math

RANK_SEED_STRIDE = 100000
BLOCKSIZE = 64
DQ_BLOCKSIZE = 256


def token_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own token-side tensor (X, dY): distinct per rank."""
    return seed + RANK_SEED_STRIDE * rank


def replica_seed(seed: int, rank: int) -> int:
    """Seed of a replicated tensor (W, A, B): the same on every rank."""
    del rank
    return seed


def _allreduce_sum(t, group=None) -> None:
    import torch
    import torch.distributed as dist
    if (t.is_cuda or t.dtype in (torch.bfloat16, torch.float16)) and dist.get_backend(group) == "gloo":
        # gloo: host staging; 16-bit values summed in fp32 and rounded once
        h = t.cpu()
        if h.dtype in (torch.bfloat16, torch.float16):
            h = h.float()
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
        t.copy_(h)
    else:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def allreduce_adapter_grads(dA, dB, group=None) -> None:
    """Sum dA and dB over the ranks of `group`, in place, in their own dtype."""
    _allreduce_sum(dA, group)
    _allreduce_sum(dB, group)


def row_alignment(cols: int) -> int:
    """Rows per whole number of DQ groups: a shard boundary on a multiple of
    this keeps every group of 256 block scales on one rank."""
    blocks_per_row = cols // BLOCKSIZE
    return DQ_BLOCKSIZE // math.gcd(DQ_BLOCKSIZE, blocks_per_row)


def shard_rows(rows: int, cols: int, world: int, rank: int) -> tuple[int, int]:
    """Row range [r0, r1) that `rank` quantises: contiguous, balanced to
    within one alignment unit, every boundary but the end of the matrix on a
    whole DQ group.  A rank may get an empty range when rows are few."""
    align = row_alignment(cols)
    units = -(-rows // align)
    u0, u1 = units * rank // world, units * (rank + 1) // world
    return min(rows, u0 * align), min(rows, u1 * align)


def quantize_sharded(q, W, rows_total: int, row0: int, group=None, quant_type: int = 0):
    """Quantise this rank's rows W = W_full[row0 : row0 + W.shape[0]] with
    double quantisation whose mean covers the whole matrix: the exponent
    histogram of this shard's absmax values is summed over ranks, then the
    shard's 8-bit scales are written from the summed histogram.  Returns the
    shard's quantised weight (an NF4Tensor of W.shape)."""
    import torch
    rows, cols = W.shape
    t = q.empty_quantized(rows, cols, W.device, True, quant_type)
    hist = torch.empty(256, dtype=torch.int64, device=W.device)
    if rows:
        q.qlora_quantize_4bit(W, t.packed, t.absmax, quant_type, hist)
    else:
        hist.zero_()
    _allreduce_sum(hist, group)
    if rows:
        q.nf4_double_quantize_hist(t.absmax, hist, rows_total * cols // BLOCKSIZE, t.qabsmax,
                                   t.dq_scale, t.dq_mean)
    return t


def allgather_quantized(q, shard, rows_total: int, world: int, group=None):
    """Every rank's shard (from quantize_sharded on shard_rows) gathered into
    the whole quantised weight on every rank: packed codes, 8-bit scales and
    group scales concatenated in rank order (the shards' means are equal)."""
    import torch
    import torch.distributed as dist
    cols = shard.cols
    bounds = [shard_rows(rows_total, cols, world, r) for r in range(world)]
    counts = [r1 - r0 for r0, r1 in bounds]
    full = q.empty_quantized(rows_total, cols, shard.packed.device, True, shard.quant_type)
    mean_src = None

    def gather(part, whole, per_row, groups=False):
        # pad every shard to the largest, gather, then cut each to its size
        dev = part.device
        sizes = [(c * cols // BLOCKSIZE + DQ_BLOCKSIZE - 1) // DQ_BLOCKSIZE if groups else c * per_row
                 for c in counts]
        mx = max(sizes) if sizes else 0
        buf = torch.zeros(mx, dtype=part.dtype, device=dev)
        buf[:part.numel()] = part
        outs = [torch.empty_like(buf) for _ in range(world)]
        if part.is_cuda and dist.get_backend(group) == "gloo":
            outs_h = [o.cpu() for o in outs]
            dist.all_gather(outs_h, buf.cpu(), group=group)
            outs = [o.to(dev) for o in outs_h]
        else:
            dist.all_gather(outs, buf, group=group)
        off = 0
        for o, n in zip(outs, sizes):
            whole[off:off + n] = o[:n]
            off += n

    gather(shard.packed, full.packed, cols // 2)
    gather(shard.absmax, full.absmax, cols // BLOCKSIZE)
    gather(shard.qabsmax, full.qabsmax, cols // BLOCKSIZE)
    gather(shard.dq_scale, full.dq_scale, 0, groups=True)
    for r, c in enumerate(counts):
        if c and mean_src is None:
            mean_src = r
    m = shard.dq_mean.clone()
    if mean_src is not None:
        import torch.distributed as dist2
        if m.is_cuda and dist2.get_backend(group) == "gloo":
            h = m.cpu()
            dist2.broadcast(h, src=mean_src, group=group)
            m.copy_(h)
        else:
            dist2.broadcast(m, src=mean_src, group=group)
    full.dq_mean.copy_(m)
    return full
