"""Sharded quantization of one tensor over ranks, host side, on the CPU
("QLoRA: Mathematical Foundations ...", section "Double Quantization (DQ)":
one mean per tensor, so ranks holding parts of a tensor must exchange one
thing).  The split (qlora_nf4_quantize_b200.sharded.shard_range) and the
all-gather of the runs' fp64 sums (gather_run_sums, over gloo with world
sizes 2 and 3) are the library's host code; the per-shard arithmetic is the
CPU oracle's.  Done this way on every rank, the mean, the second-level
scales, the 8-bit codes and the NF4 codes are bit-identical to the oracle's
one-rank quantization of the whole tensor."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

RUN = 64 * 256


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("n", [0, 2, RUN - 2, RUN, RUN + 64, 7 * RUN + 64 * 5 + 6, 300 * RUN])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_ranges_cover_the_tensor_on_run_boundaries(n, world):
    from qlora_nf4_quantize_b200.sharded import shard_range
    ranges = [shard_range(n, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    runs_held = []
    for (a, b), (c, _) in zip(ranges, ranges[1:] + [(n, n)]):
        assert a <= b and b == c              # contiguous, in rank order
        assert a % RUN == 0 or a == n         # starts on a run boundary
        assert b % RUN == 0 or b == n         # ends on one, or at the end
        runs_held.append(-(-(b - a) // RUN))
    assert max(runs_held) - min(runs_held) <= 1
    assert runs_held == sorted(runs_held, reverse=True)


def test_shard_range_rejects_bad_ranks():
    from qlora_nf4_quantize_b200.sharded import shard_range
    with pytest.raises(ValueError):
        shard_range(100, 2, 2)
    with pytest.raises(ValueError):
        shard_range(100, 0, 0)


def _tensor(n):
    g = torch.Generator().manual_seed(31)
    w = torch.randn(n, generator=g) * 0.02
    w[::997] *= 10.0
    w[3 * RUN:3 * RUN + 64] = 0.0  # an all-zero block
    return w.to(torch.bfloat16)


def _bits(w):
    return w.contiguous().view(torch.int16).numpy().view(np.uint16).ravel()


def _rank(rank, world, port, n, out):
    import torch.distributed as dist

    import oracle
    from qlora_nf4_quantize_b200.sharded import gather_run_sums, shard_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        e0, e1 = shard_range(n, world, rank)
        packed, c1 = oracle.quantize(_bits(_tensor(n))[e0:e1])
        local = torch.from_numpy(oracle.dq_run_sums(c1))
        all_sums = gather_run_sums(local, world)
        mu = oracle.dq_mean_from_run_sums(all_sums.numpy(), -(-n // 64))
        codes, c2 = oracle.double_quantize_with_mean(c1, mu)
        out[rank] = (packed.tobytes(), c1.tobytes(), codes.tobytes(), c2.tobytes(), float(mu),
                     all_sums.numpy().tobytes())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n", [(2, 9 * RUN + 64 * 3 + 10), (3, 4 * RUN), (3, 2 * RUN + 2)])
def test_sharded_quantization_bit_identical_to_one_rank(world, n):
    import oracle
    oracle.lib()
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank, args=(r, world, port, n, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    packed, c1 = oracle.quantize(_bits(_tensor(n)))
    codes, c2, mu = oracle.double_quantize(c1)
    parts = [out[r] for r in range(world)]
    assert b"".join(p[0] for p in parts) == packed.tobytes()
    assert b"".join(p[1] for p in parts) == c1.tobytes()
    assert b"".join(p[2] for p in parts) == codes.tobytes()
    assert b"".join(p[3] for p in parts) == c2.tobytes()
    for p in parts:
        assert np.float32(p[4]).view(np.uint32) == np.float32(mu).view(np.uint32)
        assert p[5] == oracle.dq_run_sums(c1).tobytes()  # every rank gathered every run, in order
