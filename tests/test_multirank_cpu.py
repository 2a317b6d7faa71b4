"""The multi-GPU path is replicas only: N independent decoders, no data-path
collective.  Its host logic -- process group from the launcher's environment,
barriers around the timed region, the timed region's maximum over ranks and
the whole-job ms per token -- runs here as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup(world, backend="gloo")
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    # rank r's timed region took 100 + 10 r ms for 16 steps
    total = bench.max_over_ranks(100.0 + 10.0 * r, w)
    out[rank] = (total, bench.per_token_ms(total, 16, w))
    bench.barrier(w)
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_take_the_slowest_rank():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1]
    total, per_tok = out[0]
    assert total == 110.0                  # the slowest rank
    assert per_tok == 110.0 / (16 * 2)     # tokens of both replicas over that time


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.per_token_ms(32.0, 16, 1) == 2.0
