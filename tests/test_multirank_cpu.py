"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): process-group
set-up from the torchrun environment, barrier, and the max-over-ranks timing
that turns per-rank step times into the whole-job number."""

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


def _rank_main(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
        import bench

        r, lr, w = bench.dist_env()
        dist = bench.dist_init(w, "gloo")
        dev = torch.device("cpu")
        bench.barrier(dist, dev)
        ms = 10.0 + 5.0 * r  # rank 1 is slower
        mx = bench.reduce_max(ms, dist, dev)
        bench.barrier(dist, dev)
        dist.destroy_process_group()
        q.put((r, lr, w, mx))
    except Exception as e:  # report instead of hanging the parent
        q.put(("error", repr(e)))


def test_two_rank_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[0] != "error" for r in res), res
    res.sort()
    assert [r[:3] for r in res] == [(0, 0, 2), (1, 1, 2)]
    assert all(r[3] == 15.0 for r in res)  # both ranks see the slowest rank's time


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.dist_init(1, "gloo") is None
    assert bench.reduce_max(3.5, None, torch.device("cpu")) == 3.5
    bench.barrier(None, torch.device("cpu"))


def test_reference_arm_prints_on_rank0_only(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0",
                       "--workload", "tiny"]) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0",
                       "--workload", "tiny"]) == 0
    import json

    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_of_every_path(capsys, monkeypatch):
    """The reference arm (the oracle on the host) prints one valid line for
    the layer, each variant and the backward pass, with that path's metric."""
    sys.path.insert(0, ROOT)
    import json

    import bench

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    seen = set()
    for extra in (["--variant", "rope"], ["--variant", "gdn"], ["--variant", "softmax"],
                  ["--mode", "backward"]):
        assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0",
                           "--workload", "tiny"] + extra) == 0
        line = json.loads(capsys.readouterr().out.strip())
        assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
        assert line["metric"] == bench.metric_for(*(("backward", "plain") if "--mode" in extra
                                                    else ("forward", extra[1])))
        seen.add(line["metric"])
    assert len(seen) == 4


def test_anchor_pair_count_matches_the_oracle_key_ranges():
    """The softmax anchor's roofline counts 4 d flops per (query, key) pair;
    the pair count agrees with the oracle's key ranges summed frame by frame."""
    sys.path.insert(0, ROOT)
    import bench
    from oracle.gla_softmax_oracle import anchor_key_ranges
    from workloads import WORKLOADS

    for name, window, n_sink in (("720p-5s", 2, 3680), ("tiny", 3, 5), ("480p-5s", 1, 0)):
        w = WORKLOADS[name]
        T = w.tokens_per_frame
        per_bh = 0
        for f in range(w.frames):
            (s0, s1), (w0, w1) = anchor_key_ranges(f, T, window, n_sink)
            per_bh += T * ((s1 - s0) + (w1 - w0))
        assert bench.anchor_pairs(w, window, n_sink) == per_bh * w.B * w.H
