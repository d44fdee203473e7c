"""bench.py's steps across ranks, as two gloo processes on the CPU.

With N GPUs every rank decodes its own batch of the workload (weak scaling, no
collective on the data path); the ranks meet only at barriers and at the
max-over-ranks reduction of their device times, and rank 0 alone prints the
line and runs the oracle arm.  These tests run that host logic with the gloo
backend: each rank reports different times, every rank must see the slowest,
and the whole-job value must count every rank's batch at that time."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ranks = bench.Ranks(dist, "cpu")
        ranks.barrier()
        # rank r's device times: the decode total and the sum of per-launch times
        ms_total, dec_sum = ranks.max(100.0 + 7.0 * rank, 90.0 - 3.0 * rank)
        e2e, = ranks.max(50.0 * (rank + 1))
        ranks.barrier()
        out.put((rank, ms_total, dec_sum, e2e, bench.whole_job_value(world, 64, ms_total / 10)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_total, dec_sum, e2e, value in res:
        assert ms_total == 107.0          # the slower rank's total
        assert dec_sum == 90.0            # each value reduced on its own
        assert e2e == 100.0
        # both ranks' batches (2 x 64 query tokens) per 10.7 ms step
        assert value == pytest.approx(2 * 64 / 10.7e-3)


def test_ranks_without_a_process_group_are_identity():
    r = bench.Ranks()
    r.barrier()
    assert r.max(3.0, 1.5) == (3.0, 1.5)
    assert bench.whole_job_value(1, 32, 2.0) == pytest.approx(16000.0)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank, monkeypatch, capsys):
    calls = []
    monkeypatch.setattr(bench, "run_reference", lambda args, w: calls.append(w.name) or {"impl": "reference"})
    monkeypatch.setenv("RANK", str(rank))
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--config", "C0"])
    bench.main()
    printed = capsys.readouterr().out.strip()
    if rank == 0:
        assert calls == ["C0"] and json.loads(printed) == {"impl": "reference"}
    else:
        assert calls == [] and printed == ""


def test_recorded_traffic_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    """The committed DRAM traffic is reported only while the decode sources hash to the digest
    stored with it; any edit of those sources turns it into null (a re-capture is due)."""
    csrc = tmp_path / "rank_compressed_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in bench.DECODE_SOURCES:
        (csrc / n).write_text(f"// {n}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    rec = {"decode:C2": {"bytes_per_launch": 12345, "sources_sha256_16": bench.sources_digest()}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("decode", "C2") == 12345
    assert bench.recorded_traffic("decode", "C3") is None          # no record for this workload
    (csrc / bench.DECODE_SOURCES[0]).write_text("// edited\n")
    assert bench.recorded_traffic("decode", "C2") is None          # sources changed since the capture
