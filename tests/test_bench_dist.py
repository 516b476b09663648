"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The scan path shards by replicas with no collective on the data path, so the
only cross-rank steps are the barriers and the max-over-ranks timing. These
tests run them as two real processes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slower one
    m = bench.max_over_ranks(local_ms, w)
    s = bench.sum_over_ranks(1.0, w)
    value, slowest = bench.weak_scaling_value(4096.0, local_ms, w)
    out[rank] = (m, s, value, slowest)
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_weak_scaling_aggregation_two_ranks(world):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        m, s, value, slowest = out[rank]
        assert m == 15.0 and s == 2.0 and slowest == 15.0
        # every rank processed 4096 units; the job time is the slowest rank's
        assert value == pytest.approx(4096.0 * world / 0.015)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(100.0, 50.0, 1) == (2000.0, 50.0)


def test_measured_traffic_only_for_the_profiled_sources(monkeypatch):
    import bench
    for step in ("prefill", "decode"):
        v = bench.measured_traffic(step)
        assert v is None or v == bench.MEASURED_TRAFFIC[step]["bytes"]
        changed = dict(bench.MEASURED_TRAFFIC[step], sha256="0" * 64)
        monkeypatch.setitem(bench.MEASURED_TRAFFIC, step, changed)
        assert bench.measured_traffic(step) is None


def test_source_digest_ignores_comments_not_code(tmp_path, monkeypatch):
    # the traffic records stay valid across a change of comments or blank space, not across a change of code
    import bench
    csrc = tmp_path / "gated_delta_rule_bounded_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = csrc / "k.cu"
    f.write_text("// kernel\nint f(int x) {\n  return x + 1;  /* one */\n}\n")
    d0 = bench.source_digest(["k.cu"])
    f.write_text("/* a longer\n   comment */\nint f(int x) {\n\n    return x + 1;   // one more\n}\n")
    assert bench.source_digest(["k.cu"]) == d0
    f.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.source_digest(["k.cu"]) != d0
