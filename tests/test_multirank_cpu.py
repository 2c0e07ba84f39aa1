"""Host-side logic of the multi-GPU benchmark on CPU: two gloo ranks.

Sequences are independent, so N GPUs run N replicas on their own batches
(weak scaling) with no data-path collective; the only cross-rank steps are the
timing reductions.  This checks them with world size 2 over gloo."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    from datetime import timedelta
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    import synth
    wl = synth.WORKLOADS["b256_T128"]
    ids, mask, L = synth.make_batch(wl, seed=bench.rank_batch_seed(wl.seed, rank))
    local_ms = [3.0, 5.0][rank]
    local_tok = float(L.sum())
    out = dict(rank=rank, ids_sum=int(ids.sum()), tok=local_tok,
               max_ms=bench.max_over_ranks(local_ms, dist), sum_tok=bench.sum_over_ranks(local_tok, dist),
               value=bench.job_throughput(local_tok, local_ms, dist))
    dist.barrier()
    dist.destroy_process_group()
    q.put(out)


def test_two_rank_timing_reductions_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda d: d["rank"])
    total_tok = res[0]["tok"] + res[1]["tok"]
    for d in res:
        assert d["max_ms"] == 5.0                      # the slowest rank sets the job time
        assert d["sum_tok"] == total_tok
        assert d["value"] == pytest.approx(total_tok / 5e-3)
    assert res[0]["ids_sum"] != res[1]["ids_sum"]      # each rank encodes its own batch


def test_single_process_reductions_are_identity():
    import bench
    assert bench.max_over_ranks(2.5) == 2.5 and bench.sum_over_ranks(7.0) == 7.0
    assert bench.job_throughput(1000.0, 2.0) == pytest.approx(5e5)
