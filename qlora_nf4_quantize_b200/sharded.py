"""Quantization of one weight tensor split over ranks (one process per GPU).

"QLoRA: Mathematical Foundations ..." (llms.blog), section "Double
Quantization (DQ)": the second quantization level subtracts one mean per
tensor, so a tensor whose weights are spread over several GPUs needs one
exchange.  Everything else is independent per run of 256 blocks of 64
weights (16,384 weights):

  1. shard_range cuts the flattened tensor on run boundaries, so no 64-block
     and no second-level run straddles two ranks;
  2. each rank quantizes its shard (nf4_quantize) and computes the fp64 sum
     of each of its runs (nf4_dq_run_sums) -- quantize_shard_local;
  3. the run sums of all ranks are gathered in rank order (gather_run_sums:
     one all-gather of ceil(runs / world) doubles per rank);
  4. every rank double-quantizes its own constants with the mean built from
     the whole array (nf4_double_quantize_sharded) -- finish_shard.

Because every rank combines the same run sums in the same fixed order, mu,
c2 and every code are bit-identical to a one-rank quantization of the whole
tensor, for any world size.  Only the host-side plumbing lives here; every
arithmetic step runs in the library's kernels.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch

from . import nf4

RUN = nf4.BLOCKSIZE * nf4.DQ_BLOCKSIZE  # weights per second-level run


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Element range [e0, e1) of rank `rank` out of `world` for a flattened
    tensor of n weights: whole runs of 16,384 weights, as even as the run
    count allows (earlier ranks never hold fewer runs than later ones); the
    last non-empty range ends at n."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    runs = -(-n // RUN)
    base, extra = divmod(runs, world)
    r0 = rank * base + min(rank, extra)
    r1 = r0 + base + (1 if rank < extra else 0)
    return min(r0 * RUN, n), min(r1 * RUN, n)


def run_counts(n_total: int, world: int):
    """Runs (second-level blocks) each rank's shard holds."""
    out = []
    for r in range(world):
        e0, e1 = shard_range(n_total, world, r)
        out.append(-(-(-(-(e1 - e0) // nf4.BLOCKSIZE)) // nf4.DQ_BLOCKSIZE))
    return out


def gather_run_sums(local: torch.Tensor, world: int, group=None, counts=None) -> torch.Tensor:
    """All-gather the ranks' fp64 run sums, concatenated in rank order.

    Shards hold different run counts: each rank pads its sums to the largest
    count, takes part in one all-gather and drops the padding.  `counts`
    (each rank's run count, e.g. run_counts()) saves a first all-gather that
    learns them (and its host synchronisation)."""
    import torch.distributed as dist
    if world == 1:
        return local
    dev = local.device
    if counts is None:
        count = torch.tensor([local.numel()], dtype=torch.int64, device=dev)
        cl = [torch.zeros_like(count) for _ in range(world)]
        dist.all_gather(cl, count, group=group)
        counts = [int(c.item()) for c in cl]
    width = max(max(counts), 1)
    padded = torch.zeros(width, dtype=torch.float64, device=dev)
    padded[:local.numel()] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)])


def quantize_shard_local(w_shard: torch.Tensor, stream=None):
    """Step 2: NF4 codes and fp32 constants of this shard, and its runs'
    fp64 sums.  Returns (packed, absmax, run_sums)."""
    packed, absmax = nf4.nf4_quantize(w_shard.reshape(-1), stream=stream)
    sums = nf4.nf4_dq_run_sums(absmax, stream=stream)
    return packed, absmax, sums


def finish_shard(absmax: torch.Tensor, run_sums_all: torch.Tensor, n_total: int, stream=None):
    """Step 4: this shard's double quantization with the tensor-wide mean.
    Returns (absmax_q, absmax2, offset)."""
    nb_total = -(-n_total // nf4.BLOCKSIZE)
    return nf4.nf4_double_quantize_sharded(absmax, run_sums_all, nb_total, stream=stream)


def quantize_sharded(w_shard: torch.Tensor, n_total: int, world: int, group=None,
                     gather: Optional[Callable[[torch.Tensor], torch.Tensor]] = None, stream=None):
    """Quantize this rank's shard (the range shard_range gives it) of a tensor
    of n_total weights, with double quantization centred on the mean of the
    whole tensor.  ``gather`` replaces the all-gather (default:
    gather_run_sums over ``group``).  Returns the shard's QuantState (shape
    (numel,))."""
    packed, absmax, sums = quantize_shard_local(w_shard, stream=stream)
    all_sums = gather(sums) if gather is not None else gather_run_sums(sums, world, group,
                                                                        run_counts(n_total, world))
    q8, c2, off = finish_shard(absmax, all_sums, n_total, stream=stream)
    return nf4.QuantState(packed, q8, c2, off, (w_shard.numel(), 1))
