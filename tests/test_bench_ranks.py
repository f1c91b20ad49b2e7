"""The multi-rank host logic of bench.py on CPU: two `gloo` ranks (world size
2) reduce their device-timed values to the slowest rank's and compute the
whole-job rate from it, as `bench.py --gpus N` does under torchrun with NCCL.
Replicas only: no collective on the data path, so the timing reduction is the
only exchange to cover."""

import importlib.util
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# per-rank (total, prefill sum, decode sum) in ms, and the e2e sum
TIMES = {0: [35.9, 8.6, 27.1, 36.8], 1: [35.2, 8.9, 26.7, 37.4]}
UNITS = 128 * 10   # decode tokens per rank (128 steps x 10 timed steps)


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        dist.barrier()
        total, pre, dec = b.max_over_ranks(dist, TIMES[rank][:3], "cpu")
        (e2e,) = b.max_over_ranks(dist, TIMES[rank][3:], "cpu")
        dist.barrier()
        res = {"max": [total, pre, dec, e2e], "value": b.whole_job_rate(world, UNITS, dec),
               "e2e": b.whole_job_rate(world, UNITS, e2e)}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_single_process_is_the_identity():
    b = _bench()
    assert b.max_over_ranks(None, [1.5, 2.25], "cpu") == [1.5, 2.25]
    assert b.whole_job_rate(1, 1280, 27.1) == pytest.approx(1280 / 0.0271)


def test_two_gloo_ranks_take_the_slowest_rank(tmp_path):
    world = 2
    mp.spawn(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    expect = [max(TIMES[0][i], TIMES[1][i]) for i in range(4)]
    for r in res:
        # every rank holds the same maxima: each column's slowest rank
        assert r["max"] == pytest.approx(expect, rel=0, abs=1e-12)
        # the whole job's units over the slowest rank's decode time
        assert r["value"] == pytest.approx(world * UNITS / (expect[2] / 1e3))
        assert r["e2e"] == pytest.approx(world * UNITS / (expect[3] / 1e3))
    # a rank's own (faster) time would overstate the rate
    assert res[0]["value"] < world * UNITS / (TIMES[1][2] / 1e3)
