"""Multi-rank host logic of bench.py on CPU with gloo (world size 2): each
rank gets its own sequence (weak scaling, no data exchange) and the reported
time is the max over ranks."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


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
    import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        cfg = bench.rank_config(synth.CONFIGS[2], rank)
        # every rank draws a different sequence of the same shape
        stats = synth.make_stats(cfg)
        digest = float(stats[0][0, 0, 0])
        t = bench.max_over_ranks(1.0 + rank * 2.5, dist, "cpu")
        gathered = [None] * world
        dist.all_gather_object(gathered, (cfg.seed, cfg.n_layers, digest))
        out.put((rank, t, gathered))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, gathered in res:
        assert t == pytest.approx(3.5)  # max of 1.0 and 3.5
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == 2                      # distinct sequences
        assert gathered[0][1] == gathered[1][1] == 64    # same shape
        assert gathered[0][2] != gathered[1][2]          # different draws


def test_reference_arm_rank_gating(capsys, monkeypatch):
    import bench

    class A:
        steps, warmup, config = 1, 0, 0

    # a non-zero rank prints nothing and exits 0 without work
    assert bench.run_reference(A(), 1, 2) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank0(capsys):
    """Rank 0 times the oracle (one process per host core, one unit each per
    step) and prints the contract's JSON line with the GPU arm's config (the
    tiny configuration keeps this to seconds)."""
    import json

    import bench

    class A:
        steps, warmup, config = 2, 1, 0

    assert bench.run_reference(A(), 0, 1) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    import synth
    assert line["config"] == bench.config_desc(synth.CONFIGS[0])
    assert line["cpu_baseline"]["cores"] == bench.host_cores()


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """bench.py reports the score kernel's DRAM traffic only while the
    committed ncu record was taken on the current kernel source."""
    import json

    import bench

    rec = {"score_kernel": {"source_hash": bench.kernel_source_hash(),
                            "bytes_per_launch_full_size": 123}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    real_root = bench.ROOT
    src = os.path.join(real_root, "key_retention_scoring_b200")
    os.symlink(src, tmp_path / "key_retention_scoring_b200")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("score_kernel") == 123
    rec["score_kernel"]["source_hash"] = "0" * 16
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("score_kernel") is None
    assert bench.recorded_traffic("other_kernel") is None
