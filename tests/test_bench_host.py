"""Host-side checks of bench.py that need no GPU: the max-over-ranks timing
reduction on two gloo ranks, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT

sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(1.5 + rank * 2.25, world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 3.75, 1: 3.75}


def test_max_over_ranks_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "KV tokens/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["higher_is_better"] is True and d["warmup"] >= 3


def test_traffic_record_is_dropped_when_the_kernel_changes(tmp_path, monkeypatch):
    """The roofline's measured DRAM traffic is reported only while the kernel
    sources still hash to the value recorded with the ncu capture."""
    import hashlib
    import json
    import bench
    src = ["common.cuh"]
    path = os.path.join(bench.ROOT, "attention_decode_b200", "csrc", "common.cuh")
    good = hashlib.sha256(open(path, "rb").read()).hexdigest()
    rec = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    rec.write_text(json.dumps({"k": {"sources": src, "source_sha256": good, "bytes_per_launch": 123}}))
    assert bench.measured_traffic("k") == 123
    rec.write_text(json.dumps({"k": {"sources": src, "source_sha256": "0" * 64, "bytes_per_launch": 123}}))
    assert bench.measured_traffic("k") is None
    assert bench.measured_traffic("missing") is None
