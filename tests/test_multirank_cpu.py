"""The multi-rank path of bench.py on the CPU: two gloo ranks agree on the
slowest rank's time and on the whole-job throughput (weak scaling: every rank
runs its own contiguous slice of one global batch; sequences are independent,
so no data moves between ranks), and the per-rank shards of a ragged global
batch, each run through the oracle, concatenate to the whole batch's result."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank             # rank 1 is the slow one
        got = bench.max_over_ranks(my_ms, world)
        rate = bench.whole_job_rate(1000, world, 4, got)
        dist.barrier()
        out[rank] = (got, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:      # no fork after other tests started threads
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 1000 tokens per rank per step, 4 steps, 2 ranks, 15 ms -> 533,333 tokens/s
    assert res[0][1] == res[1][1] == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(32768, 1, 10, 25.0) == pytest.approx(32768 * 10 / 0.025)


def _shard_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    from reverse_selective_ssm_b200 import synthetic as S
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = S.make_case(4, B=3, L=80, shard=(rank, world))     # lengths U{64..80}, NaN padding
        w = S.weights_f64(case.weights[0])
        got = O.sidecar_forward(S.to_f64(case.h), w, case.s[0], case.lengths.numpy(), "bf16")
        parts = [None] * world
        dist.all_gather_object(parts, (case.meta["first_sequence"], case.h, case.lengths, got))
        if rank == 0:
            out["parts"] = parts
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_partition_a_ragged_batch():
    """Rank r takes sequences [3r, 3r + 3) of a global batch of 6: its inputs
    are bit for bit those rows of the global batch, and the concatenated
    per-rank oracle outputs equal the whole batch's oracle output bit for bit
    (padding, NaN-poisoned, included)."""
    import numpy as np
    import oracle as O
    from reverse_selective_ssm_b200 import synthetic as S
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        parts = list(out["parts"])
    whole = S.make_case(4, B=6, L=80)
    assert [p[0] for p in parts] == [0, 3]
    h = torch.cat([p[1] for p in parts])
    lens = torch.cat([p[2] for p in parts])
    assert torch.equal(h.view(torch.int16), whole.h.view(torch.int16))
    assert torch.equal(lens, whole.lengths)
    assert len(set(lens.tolist())) > 1                      # genuinely ragged
    want = O.sidecar_forward(S.to_f64(whole.h), S.weights_f64(whole.weights[0]), whole.s[0],
                             whole.lengths.numpy(), "bf16")
    got = np.concatenate([p[3] for p in parts])
    assert np.array_equal(got, want, equal_nan=True)
