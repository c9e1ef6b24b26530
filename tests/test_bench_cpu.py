"""bench.py pieces that need no GPU: the reference arm's JSON line (alone and
under a two-rank torchrun launch) and the staleness rule of the recorded ncu
traffic."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["metric"] == bench.METRIC and line["unit"] == "elem/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.WORKLOAD
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["nproc"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_two_ranks():
    """Launched as the driver launches N > 1 (torchrun, one process per
    rank): the ranks meet over gloo, rank 0 alone prints one line, every
    rank exits 0."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def _fake_tree(tmp_path, monkeypatch, traffic=123456789):
    csrc = tmp_path / bench.CSRC
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("int kernel_v1;  // a comment\n")
    (csrc / "pwq_device.cuh").write_text("/* helpers */ int helpers;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.source_sha256("k.cu")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k.md").write_text(
        "# k\n\n| metric | value |\n\ntraffic_bytes_per_launch: %d\nsource_sha256: `%s` (note)\n" % (traffic, sha))


def test_recorded_traffic_fresh_and_stale(tmp_path, monkeypatch):
    _fake_tree(tmp_path, monkeypatch)
    monkeypatch.setattr(bench, "PROFILES", {"op": ("profiles/k.md", "k.cu")})
    t, note = bench.recorded_traffic("op")
    assert t == 123456789, note
    # a comment edit leaves the figure valid, a code edit makes it stale
    (tmp_path / bench.CSRC / "k.cu").write_text("int kernel_v1;  // another comment\n\n")
    assert bench.recorded_traffic("op")[0] == 123456789
    (tmp_path / bench.CSRC / "k.cu").write_text("int kernel_v2;\n")
    t, note = bench.recorded_traffic("op")
    assert t is None and "changed" in note
    assert bench.recorded_traffic("other")[0] is None


def test_every_profile_summary_parses():
    # each committed summary names its traffic and the source hash it was taken on
    for op, (md, src) in bench.PROFILES.items():
        if not os.path.exists(os.path.join(ROOT, md)):
            continue
        text = open(os.path.join(ROOT, md)).read()
        assert "traffic_bytes_per_launch:" in text and "source_sha256:" in text, md
        assert os.path.exists(os.path.join(ROOT, bench.CSRC, src)), src


class _Recorder:
    """Stands in for the binding: records the tensor lists of every call."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args, **kw):
            self.calls.append((name, args, kw))
        return f


def _flat(x):
    if isinstance(x, (list, tuple)):
        for y in x:
            yield from _flat(y)
    else:
        yield x


@pytest.mark.parametrize("per_call", [1, 2])
def test_grouped_calls_cover_every_layer_once(per_call):
    # small stand-in layers with the workload's tensor names
    import torch
    import workloads as W
    names = [n for g in W.QWEN3_4B_GROUPS for n in g]
    layers = [{n: torch.zeros(32, 64, dtype=torch.bfloat16) for n in names} for _ in range(3)]
    rec = _Recorder()
    buf = bench.Buffers(layers, rec, torch, per_call)
    for op in bench.QWEN_OPS:
        rec.calls.clear()
        calls = bench.op_calls(op, layers, buf, rec, True, per_call)
        assert len(calls) == -(-3 // per_call)
        for c in calls:
            c()
        inputs, outputs = [], []
        for name, args, kw in rec.calls:
            inputs += [id(t) for t in _flat(args[:1])]
            outputs += [id(t) for t in _flat(kw.get("out"))]
        if op in ("fp8_block_quant", "mxfp8_quant", "nvfp4_quant", "nvfp4_fake_quant"):
            # every tensor of every layer is an input exactly once
            assert sorted(inputs) == sorted(id(t) for lay in layers for t in lay.values()), op
        # no output appears twice within one call (the API rejects overlaps)
        for j, (name, args, kw) in enumerate(rec.calls):
            outs = [id(t) for t in _flat(kw.get("out"))]
            assert len(outs) == len(set(outs)), op
            assert len(outs) == 7 * min(per_call, 3 - j * per_call), op
