"""The multi-process plumbing of bench.py on CPU: two gloo ranks.

On one GPU the virtual ranks of the ring are a loop, so ``bench.py --gpus N``
runs N independent replicas (no collective on the data path).  What the
processes share is host logic: the rendezvous, the barriers around the timed
region, the max over ranks of the device time, the whole-job rate (units of
all ranks over the slowest rank's time), and the rule that only rank 0 runs
and prints the reference arm.  All of that is exercised here with world size
2 over gloo; nothing touches a GPU.  The reference arm's JSON line (the CPU
oracle on a bounded sample) is checked against the contract too.
"""

import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, local = bench.dist_init(backend="gloo")
    bench.barrier(w)
    # rank r's own "device time": rank 1 is the slow one
    own_ms = 10.0 + 5.0 * r
    slowest = bench.max_over_ranks(own_ms, w)
    rate = bench.whole_job_rate(2.0e12, 4, w, slowest)

    class Args:  # the reference arm's arguments; ranks other than 0 must not run it
        steps, warmup, ref_sample_queries = 1, 3, 64

    ref = bench.bench_reference(Args, w, r) if r != 0 else "not run"
    bench.barrier(w)
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "local": local, "slowest": slowest, "rate": rate,
                   "ref_is_none": ref is None}, f)
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_replicas(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["world"] == world and d["rank"] == r and d["local"] == r
        # every rank sees the slowest rank's time
        assert d["slowest"] == 15.0
        # both replicas' units over the slowest time: 2 ranks x 4 steps x 2e12 / 15 ms
        assert d["rate"] == pytest.approx(2 * 4 * 2.0e12 / 15e-3)
    assert res[1]["ref_is_none"]  # only rank 0 runs the reference arm


def test_single_process_rate():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1.0e12, 10, 1, 20.0) == pytest.approx(1.0e12 * 10 / 20e-3)


def test_reference_line_contract():
    """The reference arm (the CPU oracle on a bounded sample) prints the same
    metric and units as the GPU arm, marked impl = reference, with its own
    cpu_baseline and an e2e that moves no bytes over the host link."""
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps, warmup, ref_sample_queries = 1, 3, 64

    line = bench.bench_reference(Args, 1, 0)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["value"] > 0 and line["higher_is_better"]
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "last 64 queries" in cb["sample"] and "query head 0" in cb["sample"]
    assert line["config"]["workload"] == bench.HEADLINE_NAME
    assert line["config"]["seq_len"] == 262144
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["h2d_bytes_per_step"] == 0
    assert e2e["d2h_bytes_per_step"] == 0
