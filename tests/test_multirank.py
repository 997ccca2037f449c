"""The multi-rank path of bench.py on CPU: two gloo ranks (world size 2).

The decode path shards by sequence with no data-path exchange (replicas:
each rank decodes its own batch), so the only cross-rank steps are the
barrier and the max of the ranks' device times; both run here over gloo."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import synth
        dev = torch.device("cpu")
        torch.distributed.barrier()
        got = bench.max_over_ranks(1.5 + rank, world, dev)          # rank times 1.5 and 2.5
        inp = synth.make_decode_inputs("tiny", seed=bench.rank_seed(rank), device=dev)
        out[rank] = (got, float(inp["q"].float().sum()))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_time_and_draw_their_own_batches():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5                 # every rank reports the slowest rank's time
    assert res[0][1] != res[1][1]                        # independent batches per rank
    import synth
    same = synth.make_decode_inputs("tiny", seed=0, device="cpu")["q"].float().sum()
    assert float(same) == res[0][1]                      # rank 0's batch is the seed-0 batch


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
