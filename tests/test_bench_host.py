"""Host logic of bench.py, without a GPU: the replica (N > 1) plumbing on two
gloo ranks (barrier, max over ranks, whole-job aggregation, inputs generated
once per node and shared), the packed layouts, and the per-layer grouping."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from synth import workloads as W  # noqa: E402


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, tag, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = bench.Dist(world, "gloo")
    d.barrier()
    m = d.max(1.0 + 2.0 * rank)
    v = bench.aggregate(1_000_000_000, 10, world, m)
    specs = W.small()
    lay = bench.Layout(specs)
    # one rank generates, every rank reads the same bytes
    host, path = bench.host_inputs(specs, lay, 0 if rank == 0 else 1, d, tag)
    digest = int(np.frombuffer(host, dtype=np.uint8).astype(np.uint64).sum())
    d.barrier()
    if rank == 0:
        for p in (path, path + ".done"):
            os.remove(p)
    q.put((rank, m, v, digest))
    d.close()


def test_two_gloo_ranks_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    tag = f"test{os.getpid()}"
    procs = [ctx.Process(target=_worker, args=(r, 2, port, tag, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, d0), (r1, m1, v1, d1) = res
    assert m0 == m1 == 3.0                       # the slowest rank's time
    assert v0 == v1 == pytest.approx(1e9 * 10 * 2 / 3.0 / 1e9)
    assert d0 == d1 and d0 > 0                   # both ranks saw the same generated inputs
    x = W.materialize(W.small()[0])
    assert d0 == int(x.view(np.uint8).astype(np.uint64).sum())


def test_layout_and_layer_groups():
    specs = W.qwen3_8b_model(layers=3)
    lay = bench.Layout(specs)
    assert len(lay.x_off) == 21
    assert all(o % 256 == 0 for o in lay.x_off + lay.y_off + lay.s_off)
    for i in range(20):
        assert lay.x_off[i + 1] - lay.x_off[i] >= specs[i].numel * 2
        assert lay.y_off[i + 1] - lay.y_off[i] >= specs[i].numel
    groups = bench.layers_of(specs)
    assert groups == [list(range(7 * k, 7 * k + 7)) for k in range(3)]
    assert bench.layers_of(W.small()) == [[0]]


def test_aggregate_is_whole_job_throughput():
    assert bench.aggregate(20_838_998_016, 50, 1, 0.2) == pytest.approx(20_838_998_016 * 50 / 0.2 / 1e9)
    assert bench.aggregate(10, 1, 8, 1.0) == pytest.approx(80 / 1e9)


def test_reference_arm_prints_one_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "small", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=300, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--workload", "small", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_shape_workload():
    """`shape:` builds one tensor of the given shape (the launch counts the
    bench reports come from the library's own plan, checked on the GPU)."""
    (sp,), _ = bench.workload("shape:128x1536x2048")
    assert (sp.batch, sp.M, sp.N, sp.dtype) == (128, 1536, 2048, "bf16")
    (sp,), _ = bench.workload("shape:4000x4100:f32")
    assert (sp.batch, sp.M, sp.N, sp.dtype) == (1, 4000, 4100, "f32")


def test_traffic_record_lookup(tmp_path, monkeypatch):
    """roofline.traffic comes from a record taken on the current TMA kernel
    sources only, per launch, with the record's note on how it was obtained."""
    dig = bench.kernel_digest()
    f = tmp_path / "traffic.txt"
    f.write_text("# comment line\n"
                 f"qwen3_8b_model auto {dig} 2000000000 scaled from qwen3_8b_layer x 36.0\n"
                 f"moe_layer auto {dig} 1800000000\n"
                 "qwen3_8b_layer auto 0123456789abcdef 579000000 captured\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.traffic_for("qwen3_8b_model", "auto", 2) == (1e9, "scaled from qwen3_8b_layer x 36.0")
    assert bench.traffic_for("moe_layer", "auto", 1) == (1.8e9, "captured")
    assert bench.traffic_for("qwen3_8b_layer", "auto", 1) == (None, None)   # other sources
    assert bench.traffic_for("qwen3_8b_model", "tma", 2) == (None, None)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.traffic_for("qwen3_8b_model", "auto", 2) == (None, None)
