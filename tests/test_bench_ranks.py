"""The multi-GPU bench path (independent replicas, one per rank) on CPU with
the gloo backend: the whole-job value is all ranks' frames over the slowest
rank's device time, and every rank sees the same numbers.  Also: the
reference arm does no work on ranks other than 0."""

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


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r processed 100*(r+1) frames in 10*(r+1) ms of device time
        value, max_ms = bench.replica_throughput(100 * (rank + 1), 10.0 * (rank + 1), "cpu")
        results[rank] = (value, max_ms)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replica_throughput_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        got = dict(results)
    frames = sum(100 * (r + 1) for r in range(world))
    slowest = 10.0 * world
    for r in range(world):
        value, max_ms = got[r]
        assert max_ms == pytest.approx(slowest)
        assert value == pytest.approx(frames / (slowest / 1e3))


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not torch.distributed.is_initialized()
    value, max_ms = bench.replica_throughput(50, 25.0, "cpu")
    assert max_ms == 25.0 and value == pytest.approx(2000.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """Rank 0 of the reference arm (the oracle on host cores) prints one JSON
    line with the contract's keys, the metric of the headline arm and an e2e
    object with zero copies."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_peaks_file_read_with_fallback_for_missing_keys(tmp_path):
    """The measured peaks are used when present; missing, malformed or
    non-positive entries fall back to the stated fallback figures."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    full = tmp_path / "full.json"
    full.write_text(json.dumps({"hbm_gbs": 6541.0, "bf16_tflops": 1654.5, "bf16_tflops_sustained": 1420.0,
                                "clocks": {"sm_mhz": 1965}}))
    peaks, src = bench.load_peaks(str(full))
    assert src == "measured" and peaks["bf16_tflops"] == 1654.5 and peaks["hbm_gbs"] == 6541.0
    part = tmp_path / "part.json"
    part.write_text(json.dumps({"hbm_gbs": 6541.0, "bf16_tflops": "n/a"}))
    peaks, src = bench.load_peaks(str(part))
    assert src == "measured+fallback" and peaks["hbm_gbs"] == 6541.0
    assert peaks["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    bad = tmp_path / "bad.json"
    bad.write_text("{not json")
    peaks, src = bench.load_peaks(str(bad))
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    peaks, src = bench.load_peaks(str(tmp_path / "absent.json"))
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
