"""Benchmark: the whole block-scaled quantisation path on the Qwen3-4B-shaped
weight sweep (36 decoder layers x 7 BF16 weight tensors, 3.633 G elements,
seeded synthetic N(0, 0.02) weights), on N GPUs of one node.

One step takes every element of the sweep through every row of the path:
  fp8_block_quant -> fp8_block_dequant         (128x128 tiles, FP32 scales)
  mxfp8_quant     -> mxfp8_dequant             (1x32, UE8M0)
  nvfp4_quant (q/k/v and gate/up siblings share the global amax) -> nvfp4_dequant
  nvfp4_fake_quant (siblings; the straight-through backward needs no kernel)
Each op kind is captured once in a CUDA graph (one node per call, 36 layers)
and the step replays the graphs back to back on one stream; CUDA events
between them give the per-op device times.  Inputs (7.3 GB) are larger than
the 126 MB L2, so no flush is needed between steps.

`value` = elements of the sweep taken through the whole path per second,
summed over ranks (weak scaling: every rank sweeps its own seeded layers; the
path needs no collective).  `e2e` = the same metric through the public Python
API with the BF16 weights in pinned host memory, one layer at a time: H2D
copy, every op, and a D2H read of the quantised artefacts (codes + scales of
the three formats) inside the timed region.

`next_rows` times the FP8 block-wise re-quantisation ops (FP8 block-wise
codes + scales -> FP8 block-wise / MXFP8 / NVFP4 in one pass) on the step's
FP8 outputs over the same sweep, each in its own graph after the timed
steps; they are not part of `value`.  FP8 -> FP8 is timed twice: on the
quantiser's codes (every tile holds a +-448 code, so its code map is the
identity and the kernel copies the codes) and, as
`fp8_block_requant_general`, on seeded random codes whose magnitudes stop
below 448 with the same scales (every tile's codes change).

`--impl reference` times the CPU oracle (single thread, as it stands) on a
bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized elements/s and achieved HBM GB/s (% of B200 peak) per format"
WORKLOAD = "qwen3_4b_weight_sweep_36x7"
FALLBACK_HBM_GBS = 6650.0

# algorithmic HBM bytes per element: one read of every input, one write of
# every output, plus, for NVFP4 quantise / fake-quantise, the read of the
# amax pass (the method reads a sibling group twice: once for its amax, once
# to encode; the second read is not provably served on chip)
BYTES_PER_ELEM = {
    "fp8_block_quant": 2 + 1 + 4 / 16384,
    "fp8_block_dequant": 1 + 4 / 16384 + 2,
    "mxfp8_quant": 2 + 1 + 1 / 32,
    "mxfp8_dequant": 1 + 1 / 32 + 2,
    "nvfp4_quant": 2 + 2 + 0.5 + 1 / 16,
    "nvfp4_dequant": 0.5 + 1 / 16 + 2,
    "nvfp4_fake_quant": 2 + 2 + 2,
}
# the stricter one-pass ideal of the two-pass ops: the input read once
ONE_PASS_BYTES_PER_ELEM = {
    "nvfp4_quant": 2 + 0.5 + 1 / 16,
    "nvfp4_fake_quant": 2 + 2,
}
# our kernels launched per call (memsets are not counted)
# (NVFP4 quantise / fake-quantise is one single-pass kernel after a memset)
KERNELS_PER_CALL = {"fp8_block_quant": 1, "fp8_block_dequant": 1, "mxfp8_quant": 1, "mxfp8_dequant": 1,
                    "nvfp4_quant": 1, "nvfp4_dequant": 1, "nvfp4_fake_quant": 1}
OPS = list(BYTES_PER_ELEM)

# ncu DRAM traffic of one launch (one layer) for the kernels with a committed
# summary under profiles/: the summary records the bytes and the sha256 of
# the sources the capture ran on; once a source has changed the figure is
# stale and `traffic` is reported as null.
CSRC = "precision_weight_quantization_b200/csrc/"
PROFILES = {
    "nvfp4_fake_quant": ("profiles/nvfp4_flow_fake_quant_qwen3_4b_layer.md", "nvfp4.cu"),
    "nvfp4_quant": ("profiles/nvfp4_flow_quant_qwen3_4b_layer.md", "nvfp4.cu"),
    "fp8_block_quant": ("profiles/fp8_block_quant_qwen3_4b_layer.md", "fp8_block.cu"),
    "fp8_block_dequant": ("profiles/fp8_block_dequant_qwen3_4b_layer.md", "fp8_block.cu"),
    "mxfp8_quant": ("profiles/mxfp8_quant_qwen3_4b_layer.md", "mxfp8.cu"),
    "mxfp8_dequant": ("profiles/mxfp8_dequant_qwen3_4b_layer.md", "mxfp8.cu"),
    "nvfp4_dequant": ("profiles/nvfp4_dequant_qwen3_4b_layer.md", "nvfp4.cu"),
}


def source_sha256(kernel_file):
    """sha256 of the code of a kernel file and the shared device header, with
    comments and blank space left out (a comment edit is no kernel change)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in (kernel_file, "pwq_device.cuh"):
        with open(os.path.join(ROOT, CSRC, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("\n".join(line.strip() for line in text.splitlines() if line.strip()).encode())
    return h.hexdigest()


def recorded_traffic(op):
    """(bytes per launch, note) from the op's committed ncu summary."""
    if op not in PROFILES:
        return None, "no committed ncu summary for this kernel"
    md, src = PROFILES[op]
    try:
        text = open(os.path.join(ROOT, md)).read()
    except OSError:
        return None, "summary %s missing" % md
    import re
    vals = {}
    for key, pat in (("traffic_bytes_per_launch", r"^traffic_bytes_per_launch:\s*(\d+)"),
                     ("source_sha256", r"^source_sha256:\s*`?([0-9a-f]{64})")):
        m = re.search(pat, text, re.M)
        if m:
            vals[key] = m.group(1)
    if "traffic_bytes_per_launch" not in vals or "source_sha256" not in vals:
        return None, "summary %s records no traffic" % md
    if vals["source_sha256"] != source_sha256(src):
        return None, "kernel source changed since the capture in %s" % md
    return int(vals["traffic_bytes_per_launch"]), "ncu dram read+write of one launch, %s" % md


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="pwq", choices=["pwq", "reference"])
    ap.add_argument("--layers", type=int, default=36)
    ap.add_argument("--layers-per-call", type=int, default=2,
                    help="layers per grouped call (2: 14 tensors, the most one launch takes)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next", action="store_true",
                    help="skip timing the FP8 block-wise re-quantisation ops (reported under next_rows)")
    ap.add_argument("--per-tensor", action="store_true",
                    help="one call per tensor / sibling group instead of one grouped call per layer")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks

class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        load = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ workload

def bench_config(args, grouped, world):
    return {"workload": WORKLOAD, "layers": args.layers, "elements_per_rank": layer_elems() * args.layers,
            "tensors": "q 4096x2560, k/v 1024x2560, o 2560x4096, gate/up 9728x2560, down 2560x9728",
            "path": "fp8_block q+dq, mxfp8 q+dq, nvfp4 q (qkv, gate/up siblings)+dq, "
                    "nvfp4 fake-quant (siblings)",
            "l2": "inputs larger than L2 (7.3 GB per rank), no flush",
            "launch": ("one grouped call (one launch) per op per %d layers (%d tensors)"
                       % (args.layers_per_call, 7 * args.layers_per_call) if grouped else "one call per tensor") +
                      "; one CUDA graph per op kind, replayed back to back",
            "parallelism": "dp%d (independent sweeps)" % world}


def make_layers(n_layers, device, rank):
    import workloads as W
    layers = []
    for L in range(n_layers):
        # every rank sweeps its own seeded layers (weak scaling)
        layers.append(W.qwen3_4b_layer(L + 1000 * rank, device=device))
    return layers


def layer_elems():
    import workloads as W
    return sum(r * c for _, (r, c) in W.QWEN3_4B_LAYER)


class Buffers:
    """Pre-allocated outputs for every op of every layer."""

    def __init__(self, layers, P, torch, per_call=1):
        import workloads as W
        self.fp8 = []
        self.mx = []
        self.nv = []
        self.y = []
        self.ws = []
        dev = layers[0]["q_proj"].device
        for lay in layers:
            self.fp8.append({n: (torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=dev),
                                 torch.empty((-(-x.shape[0] // 128), -(-x.shape[1] // 128)),
                                             dtype=torch.float32, device=dev)) for n, x in lay.items()})
            self.mx.append({n: (torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=dev),
                                torch.empty((x.shape[0], x.shape[1] // 32), dtype=torch.uint8, device=dev))
                            for n, x in lay.items()})
            nv = {}
            for g in W.QWEN3_4B_GROUPS:
                nv[g] = ([torch.empty((lay[n].shape[0], lay[n].shape[1] // 2), dtype=torch.uint8, device=dev)
                          for n in g],
                         [torch.empty((lay[n].shape[0], lay[n].shape[1] // 16), dtype=torch.float8_e4m3fn,
                                      device=dev) for n in g],
                         torch.empty(1, dtype=torch.float32, device=dev))
            self.nv.append(nv)
        # BF16 output sets shared by every dequant / fake-quant, one per layer
        # position within a call (the layers of one call need distinct outputs)
        self.y = [{n: torch.empty(x.shape, dtype=torch.bfloat16, device=dev) for n, x in layers[0].items()}
                  for _ in range(min(per_call, len(layers)))]


def op_calls(op, layers, buf, P, grouped=True, per_call=1):
    """Closures for every call of one op kind over all layers: one grouped
    call per `per_call` consecutive layers (all their tensors / sibling
    groups in one launch), or with grouped=False one call per tensor / per
    group."""
    import workloads as W
    if not grouped:
        return op_calls_per_tensor(op, layers, buf, P)
    G = W.QWEN3_4B_GROUPS
    calls = []
    for i0 in range(0, len(layers), per_call):
        idx = list(range(i0, min(i0 + per_call, len(layers))))
        ts = [(i, k, n) for k, i in enumerate(idx) for n in layers[i]]       # (layer, position, name)
        gts = [(i, k, g) for k, i in enumerate(idx) for g in G]
        if op == "fp8_block_quant":
            calls.append(lambda xs=[layers[i][n] for i, k, n in ts], q=[buf.fp8[i][n][0] for i, k, n in ts],
                         s=[buf.fp8[i][n][1] for i, k, n in ts]: P.fp8_block_quant_grouped(xs, out=q, scale=s))
        elif op == "fp8_block_dequant":
            calls.append(lambda q=[buf.fp8[i][n][0] for i, k, n in ts], s=[buf.fp8[i][n][1] for i, k, n in ts],
                         y=[buf.y[k][n] for i, k, n in ts]: P.fp8_block_dequant_grouped(q, s, out=y))
        elif op == "mxfp8_quant":
            calls.append(lambda xs=[layers[i][n] for i, k, n in ts], q=[buf.mx[i][n][0] for i, k, n in ts],
                         e=[buf.mx[i][n][1] for i, k, n in ts]: P.mxfp8_quant_grouped(xs, out=q, scale=e))
        elif op == "mxfp8_dequant":
            calls.append(lambda q=[buf.mx[i][n][0] for i, k, n in ts], e=[buf.mx[i][n][1] for i, k, n in ts],
                         y=[buf.y[k][n] for i, k, n in ts]: P.mxfp8_dequant_grouped(q, e, out=y))
        elif op == "nvfp4_quant":
            calls.append(lambda xs=[[layers[i][n] for n in g] for i, k, g in gts],
                         pk=[buf.nv[i][g][0] for i, k, g in gts], sb=[buf.nv[i][g][1] for i, k, g in gts],
                         gsc=[buf.nv[i][g][2] for i, k, g in gts]:
                         P.nvfp4_quant_grouped(xs, out=pk, sb=sb, global_scale=gsc))
        elif op == "nvfp4_dequant":
            pk, sb, gs, ys = [], [], [], []
            for i, k, g in gts:
                for j, n in enumerate(g):
                    pk.append(buf.nv[i][g][0][j])
                    sb.append(buf.nv[i][g][1][j])
                    gs.append(buf.nv[i][g][2])
                    ys.append(buf.y[k][n])
            calls.append(lambda pk=pk, sb=sb, gs=gs, ys=ys: P.nvfp4_dequant_grouped(pk, sb, gs, out=ys))
        elif op == "nvfp4_fake_quant":
            calls.append(lambda xs=[[layers[i][n] for n in g] for i, k, g in gts],
                         ys=[[buf.y[k][n] for n in g] for i, k, g in gts]:
                         P.nvfp4_fake_quant_grouped(xs, out=ys))
    return calls


def op_calls_per_tensor(op, layers, buf, P):
    import workloads as W
    calls = []
    for i, lay in enumerate(layers):
        if op == "fp8_block_quant":
            for n, x in lay.items():
                q, s = buf.fp8[i][n]
                calls.append(lambda x=x, q=q, s=s: P.fp8_block_quant(x, out=q, scale=s))
        elif op == "fp8_block_dequant":
            for n in lay:
                q, s = buf.fp8[i][n]
                calls.append(lambda q=q, s=s, y=buf.y[0][n]: P.fp8_block_dequant(q, s, out=y))
        elif op == "mxfp8_quant":
            for n, x in lay.items():
                q, e = buf.mx[i][n]
                calls.append(lambda x=x, q=q, e=e: P.mxfp8_quant(x, out=q, scale=e))
        elif op == "mxfp8_dequant":
            for n in lay:
                q, e = buf.mx[i][n]
                calls.append(lambda q=q, e=e, y=buf.y[0][n]: P.mxfp8_dequant(q, e, out=y))
        elif op == "nvfp4_quant":
            for g in W.QWEN3_4B_GROUPS:
                pk, sb, gs = buf.nv[i][g]
                xs = [lay[n] for n in g]
                calls.append(lambda xs=xs, pk=pk, sb=sb, gs=gs: P.nvfp4_quant(xs, out=pk, sb=sb, global_scale=gs))
        elif op == "nvfp4_dequant":
            for g in W.QWEN3_4B_GROUPS:
                pk, sb, gs = buf.nv[i][g]
                for k, n in enumerate(g):
                    calls.append(lambda p=pk[k], s=sb[k], gs=gs, y=buf.y[0][n]: P.nvfp4_dequant(p, s, gs, out=y))
        elif op == "nvfp4_fake_quant":
            for g in W.QWEN3_4B_GROUPS:
                xs = [lay[n] for n in g]
                ys = [buf.y[0][n] for n in g]
                calls.append(lambda xs=xs, ys=ys: P.nvfp4_fake_quant(xs, out=ys))
    return calls


def capture(calls, torch):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in calls:           # warm up outside the graph (workspace pool, attributes)
            c()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    torch.cuda.synchronize()
    return g


# ------------------------------------------------------------------ the FP8 block-wise re-quantisation row

# FP8 block-wise codes + tile scales (the step's fp8_block_quant outputs)
# straight into a rollout format; algorithmic bytes: one read of the codes
# and scales (two for NVFP4: the amax pass and the encode pass), one write
# of each output
NEXT_BYTES_PER_ELEM = {
    "fp8_block_requant": 1 + 4 / 16384 + 1 + 4 / 16384,
    "fp8_block_requant_general": 1 + 4 / 16384 + 1 + 4 / 16384,
    "fp8_block_requant_mxfp8": 1 + 4 / 16384 + 1 + 1 / 32,
    "fp8_block_requant_nvfp4": 1 + 4 / 16384 + 1 + 4 / 16384 + 0.5 + 1 / 16,
}
NEXT_ONE_PASS_BYTES_PER_ELEM = {"fp8_block_requant_nvfp4": 1 + 4 / 16384 + 0.5 + 1 / 16}


def next_calls(op, layers, buf, P, torch, per_call=1):
    """One grouped call per `per_call` layers (their tensors; for NVFP4 their
    sibling groups in one single-pass launch), reading the FP8 codes and
    scales the step wrote; every layer writes its own outputs (no call
    writes over lines a previous call left in L2)."""
    import workloads as W
    lay0 = layers[0]
    dev = lay0["q_proj"].device
    names = list(lay0)
    G = W.QWEN3_4B_GROUPS
    npos = len(layers)
    nv = op == "fp8_block_requant_nvfp4"

    def per_layer(make, want):
        return [{n: make(x) for n, x in lay0.items()} for _ in range(npos)] if want else None

    out_q = per_layer(lambda x: torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=dev), not nv)
    out_s = [{n: torch.empty_like(buf.fp8[0][n][1]) for n in names} for _ in range(npos)]
    out_e = per_layer(lambda x: torch.empty((x.shape[0], x.shape[1] // 32), dtype=torch.uint8, device=dev),
                      op == "fp8_block_requant_mxfp8")
    pk = per_layer(lambda x: torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device=dev), nv)
    sb = per_layer(lambda x: torch.empty((x.shape[0], x.shape[1] // 16), dtype=torch.float8_e4m3fn, device=dev), nv)
    gsc = [[torch.empty(1, dtype=torch.float32, device=dev) for _ in G] for _ in range(npos)]
    general = None
    if op == "fp8_block_requant_general":
        general = [{n: W.random_code_bytes(tuple(x.shape), seed=9000 + 16 * i + t, max_mag=0x7D, device=dev)
                    for t, (n, x) in enumerate(layers[i].items())} for i in range(len(layers))]
    calls = []
    for i0 in range(0, len(layers), per_call):
        idx = list(range(i0, min(i0 + per_call, len(layers))))
        ts = [(i, k, n) for k, i in enumerate(idx) for n in names]
        gts = [(i, k, j) for k, i in enumerate(idx) for j in range(len(G))]
        qs = [buf.fp8[i][n][0] for i, k, n in ts]
        ss = [buf.fp8[i][n][1] for i, k, n in ts]
        if op == "fp8_block_requant_general":
            qs = [general[i][n] for i, k, n in ts]
        if op in ("fp8_block_requant", "fp8_block_requant_general"):
            calls.append(lambda qs=qs, ss=ss, o=[out_q[i][n] for i, k, n in ts], so=[out_s[i][n] for i, k, n in ts]:
                         P.fp8_block_requant_grouped(qs, ss, out=o, scale_out=so))
        elif op == "fp8_block_requant_mxfp8":
            calls.append(lambda qs=qs, ss=ss, o=[out_q[i][n] for i, k, n in ts], eo=[out_e[i][n] for i, k, n in ts]:
                         P.fp8_block_requant_mxfp8_grouped(qs, ss, out=o, scale_out=eo))
        else:
            calls.append(lambda gq=[[buf.fp8[i][n][0] for n in G[j]] for i, k, j in gts],
                         gs=[[buf.fp8[i][n][1] for n in G[j]] for i, k, j in gts],
                         o=[[pk[i][n] for n in G[j]] for i, k, j in gts],
                         so=[[sb[i][n] for n in G[j]] for i, k, j in gts],
                         gso=[gsc[i][j] for i, k, j in gts]:
                         P.fp8_block_requant_nvfp4_grouped(gq, gs, out=o, sb=so, global_scale=gso))
    return calls


def one_pass_fields(op, table, elems, ms, hbm_peak, peak_kind):
    """The one-pass figures of a two-pass op (empty for the others)."""
    if op not in table:
        return {}
    gbs = elems * table[op] / (ms / 1e3) / 1e9
    return {"alg_gbs_one_pass": round(gbs, 1), "frac_of_%s_hbm_one_pass" % peak_kind: round(gbs / hbm_peak, 4),
            "bytes_per_elem_one_pass": round(table[op], 5)}


def time_next_rows(args, layers, buf, P, torch, hbm_peak, peak_kind):
    """Device time of each re-quantisation op over the sweep (its own CUDA
    graph, replayed after the step's timing; not part of `value`)."""
    elems = layer_elems() * args.layers
    stream = torch.cuda.current_stream()
    out = {}
    for op, bpe in NEXT_BYTES_PER_ELEM.items():
        calls = next_calls(op, layers, buf, P, torch, max(1, args.layers_per_call))
        g = capture(calls, torch)
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.steps
        gbs = elems * bpe / (ms / 1e3) / 1e9
        out[op] = {"ms": round(ms, 4), "elem_per_s": elems / (ms / 1e3), "alg_gbs": round(gbs, 1),
                   "frac_of_%s_hbm" % peak_kind: round(gbs / hbm_peak, 4), "calls": len(calls),
                   "kernels_per_call": 1,
                   "bytes_per_elem": round(bpe, 5)}
        out[op].update(one_pass_fields(op, NEXT_ONE_PASS_BYTES_PER_ELEM, elems, ms, hbm_peak, peak_kind))
        del g
    return out


# ------------------------------------------------------------------ CPU oracle timing

def cpu_sample_elems():
    import workloads as W
    return sum(r * c for n, (r, c) in W.QWEN3_4B_LAYER if n in ("q_proj", "k_proj", "v_proj", "o_proj"))


def run_oracle_path(xs_bits, O):
    """The oracle over the same path for a list of member tensors (one
    sibling group)."""
    for x in xs_bits:
        q, s = O.fp8_block_quant(x)
        O.fp8_block_dequant(q, s)
        q, e = O.mxfp8_quant(x)
        O.mxfp8_dequant(q, e)
    A = O.nvfp4_group_amax(xs_bits)
    for x in xs_bits:
        pk, sb, gs = O.nvfp4_quant(x, A)
        O.nvfp4_dequant(pk, sb, gs, x.shape[-1])
        O.nvfp4_fake_quant(x, A)


def cpu_baseline(layer_cpu_bits):
    from oracle import oracle as O
    groups = [["q_proj", "k_proj", "v_proj"], ["o_proj"]]
    n = cpu_sample_elems()
    t0 = time.perf_counter()
    for g in groups:
        run_oracle_path([layer_cpu_bits[k] for k in g], O)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "elem/s", "cores": 1, "kind": "oracle",
            "sample": "layer 0 q/k/v (one NVFP4 sibling group) + o_proj: %d elements through every op "
                      "of the path, single-threaded scalar C oracle, %.1f s" % (n, dt)}


# ------------------------------------------------------------------ main

def main():
    args = parse()
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import datetime
    if args.impl == "reference":
        # the reference arm runs on the host alone: its ranks meet over gloo
        # (no GPU or NCCL involved), rank 0 times the oracle
        if world > 1:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=900))
        return main_reference(args, rank, world, torch, dist)
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import precision_weight_quantization_b200 as P
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_peak, peak_kind = peaks()

    layers = make_layers(args.layers, dev, rank)
    lpc = max(1, args.layers_per_call)
    buf = Buffers(layers, P, torch, lpc)
    elems_per_step = layer_elems() * args.layers
    grouped = not args.per_tensor
    graphs = {op: capture(op_calls(op, layers, buf, P, grouped, lpc), torch) for op in OPS}
    ncalls = {op: len(op_calls(op, layers, buf, P, grouped, lpc)) for op in OPS}
    launches_per_step = sum(ncalls[op] * KERNELS_PER_CALL[op] for op in OPS)

    stream = torch.cuda.current_stream()

    def step(evs=None):
        for k, op in enumerate(OPS):
            if evs is not None:
                evs[k].record(stream)
            graphs[op].replay()
        if evs is not None:
            evs[len(OPS)].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    per_op_ms = {op: 0.0 for op in OPS}
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(len(OPS) + 1)] for _ in range(args.steps)]
    with Clocks(local) as clk:
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            step(evsets[i])
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    for evs in evsets:
        for k, op in enumerate(OPS):
            per_op_ms[op] += evs[k].elapsed_time(evs[k + 1]) / args.steps
    ms_per_step = total_ms / args.steps
    t = torch.tensor([ms_per_step], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    value = elems_per_step * world / (ms_max / 1e3)

    per_op = {}
    for op in OPS:
        ms = per_op_ms[op]
        gbs = elems_per_step * BYTES_PER_ELEM[op] / (ms / 1e3) / 1e9
        per_op[op] = {"ms": round(ms, 4), "elem_per_s": elems_per_step / (ms / 1e3), "alg_gbs": round(gbs, 1),
                      "frac_of_%s_hbm" % peak_kind: round(gbs / hbm_peak, 4), "calls": ncalls[op],
                      "bytes_per_elem": round(BYTES_PER_ELEM[op], 5)}
        per_op[op].update(one_pass_fields(op, ONE_PASS_BYTES_PER_ELEM, elems_per_step, ms, hbm_peak, peak_kind))
    dom = max(OPS, key=lambda o: per_op_ms[o])
    dom_gbs = per_op[dom]["alg_gbs"]
    traffic, traffic_note = recorded_traffic(dom) if grouped else (None, "per-tensor launches")
    roofline = {"bound": "hbm", "kernel": dom, "achieved": dom_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": round(dom_gbs / hbm_peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                "alg_bytes_per_launch": int(round(elems_per_step / ncalls[dom] * BYTES_PER_ELEM[dom])),
                "avg_launch_us": round(per_op_ms[dom] * 1e3 / ncalls[dom], 2),
                "note": "achieved = algorithmic bytes of one launch / the average launch "
                        "duration (CUDA events around the graph of all %d launches of the step); traffic: %s"
                        % (ncalls[dom], traffic_note)}
    if dom in ONE_PASS_BYTES_PER_ELEM:
        one = per_op[dom]["alg_gbs_one_pass"]
        roofline.update({"achieved_one_pass": one, "frac_one_pass": round(one / hbm_peak, 4),
                         "alg_bytes_per_launch_one_pass":
                             int(round(elems_per_step / ncalls[dom] * ONE_PASS_BYTES_PER_ELEM[dom]))})
        roofline["note"] += ("; achieved counts the amax pass's read of the input (two reads, as the method "
                             "is defined); *_one_pass counts a single read, the stricter ideal")

    line = {"metric": METRIC, "value": value, "unit": "elem/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": bench_config(args, grouped, world),
            "per_op": per_op, "roofline": roofline, "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary() if rank == 0 else None}

    del graphs
    if not args.no_next:
        line["next_rows"] = time_next_rows(args, layers, buf, P, torch, hbm_peak, peak_kind)
    if not args.no_e2e:
        line["e2e"] = e2e(args, layers, P, torch, dev, world, dist, elems_per_step)
    if rank == 0 and not args.no_cpu_baseline:
        import workloads as W
        lay0 = {n: W.bits(x) for n, x in layers[0].items() if n in ("q_proj", "k_proj", "v_proj", "o_proj")}
        line["cpu_baseline"] = cpu_baseline(lay0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def e2e(args, layers, P, torch, dev, world, dist, elems_per_step):
    """Same path through the public API, host-resident weights: per layer an
    H2D copy from pinned memory, every op (one grouped call each), and a D2H
    read of the codes and scales of the three formats.  Three streams
    (copy in, compute, copy out) and two device buffer sets pipeline the
    layers, so the two copy directions and the kernels overlap.  A layer's
    tensors of one kind sit in one contiguous slab on both sides, so a
    layer moves in one H2D copy and six D2H copies."""
    import workloads as W
    names = list(layers[0])
    shapes = {n: tuple(layers[0][n].shape) for n in names}
    G = W.QWEN3_4B_GROUPS

    def slab(kind_shapes, dtype, device=None, pinned=False):
        """One contiguous buffer holding a tensor per name (row-major, in
        order), so a layer's tensors of one kind move in one copy."""
        numel = [int(torch.Size(sh).numel()) for sh in kind_shapes.values()]
        if device is None:
            flat = torch.empty(sum(numel), dtype=dtype)
            if pinned:
                flat = flat.pin_memory()
        else:
            flat = torch.empty(sum(numel), dtype=dtype, device=device)
        views, o = {}, 0
        for (n, sh), k in zip(kind_shapes.items(), numel):
            views[n] = flat[o:o + k].view(sh)
            o += k
        return flat, views

    tile_sh = {n: (-(-shapes[n][0] // 128), -(-shapes[n][1] // 128)) for n in names}
    mxs_sh = {n: (shapes[n][0], shapes[n][1] // 32) for n in names}
    pk_sh = {n: (shapes[n][0], shapes[n][1] // 2) for n in names}
    sb_sh = {n: (shapes[n][0], shapes[n][1] // 16) for n in names}
    host_x, hx = slab(shapes, torch.bfloat16, pinned=True)
    for n in names:
        hx[n].copy_(layers[0][n].cpu())
    # host images of a layer's outputs, one pinned slab per kind
    kinds = (("q", shapes, torch.uint8), ("s", tile_sh, torch.float32), ("mq", shapes, torch.uint8),
             ("me", mxs_sh, torch.uint8), ("pk", pk_sh, torch.uint8), ("sb", sb_sh, torch.uint8))
    host_out = {k: slab(sh, dt, pinned=True)[0] for k, sh, dt in kinds}

    def device_set():
        d = {}
        d["x_flat"], d["x"] = slab(shapes, torch.bfloat16, device=dev)
        for k, sh, dt in kinds:
            d[k + "_flat"], views = slab(sh, dt, device=dev)
            d[k] = views
        d["gs"] = [torch.empty(1, dtype=torch.float32, device=dev) for _ in G]
        return d

    sets = [device_set(), device_set()]
    y = [torch.empty(shapes[n], dtype=torch.bfloat16, device=dev) for n in names]   # dequant / QDQ outputs
    yg = [[y[names.index(n)] for n in g] for g in G]
    out_bytes = sum(t.numel() * t.element_size() for t in host_out.values())
    in_bytes = host_x.numel() * 2
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "comp", "out")}
    started = {k: [False, False] for k in ("comp", "out")}

    def one_layer(i):
        b = i % 2
        d = sets[b]
        with torch.cuda.stream(s_in):
            if started["comp"][b]:
                s_in.wait_event(ev["comp"][b])        # the layer that last read this input set is done
            d["x_flat"].copy_(host_x, non_blocking=True)
            ev["in"][b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["in"][b])
            if started["out"][b]:
                s_comp.wait_event(ev["out"][b])       # this output set has been read back
            xs = [d["x"][n] for n in names]
            q = [d["q"][n].view(torch.float8_e4m3fn) for n in names]
            sc = [d["s"][n] for n in names]
            mq = [d["mq"][n].view(torch.float8_e4m3fn) for n in names]
            me = [d["me"][n] for n in names]
            P.fp8_block_quant_grouped(xs, out=q, scale=sc)
            P.fp8_block_dequant_grouped(q, sc, out=y)
            P.mxfp8_quant_grouped(xs, out=mq, scale=me)
            P.mxfp8_dequant_grouped(mq, me, out=y)
            groups = [[d["x"][n] for n in g] for g in G]
            pk = [[d["pk"][n] for n in g] for g in G]
            sbg = [[d["sb"][n].view(torch.float8_e4m3fn) for n in g] for g in G]
            P.nvfp4_quant_grouped(groups, out=pk, sb=sbg, global_scale=d["gs"])
            P.nvfp4_dequant_grouped([p_ for g in pk for p_ in g], [t for g in sbg for t in g],
                                    [d["gs"][gi] for gi, g in enumerate(G) for _ in g], out=y)
            P.nvfp4_fake_quant_grouped(groups, out=yg)
            ev["comp"][b].record(s_comp)
            started["comp"][b] = True
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            for k, _, _ in kinds:
                host_out[k].copy_(d[k + "_flat"], non_blocking=True)
            ev["out"][b].record(s_out)
            started["out"][b] = True

    def run(n_layers):
        for i in range(n_layers):
            one_layer(i)
        cur = torch.cuda.current_stream()
        cur.wait_stream(s_in)
        cur.wait_stream(s_comp)
        cur.wait_stream(s_out)

    steps = max(1, min(args.steps, 3))
    run(args.layers)                                  # warm-up pass
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    stream = torch.cuda.current_stream()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    s_comp.wait_stream(stream)
    s_out.wait_stream(stream)
    for _ in range(steps):
        run(args.layers)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    return {"value": elems_per_step * world / (ms / 1e3), "unit": "elem/s",
            "h2d_bytes_per_step": in_bytes * args.layers, "d2h_bytes_per_step": out_bytes * args.layers,
            "ms_per_step": ms, "steps": steps,
            "note": "public Python API (one grouped call per op per layer), one layer at a time from "
                    "pinned host memory (the same host buffer feeds every layer), codes+scales of the "
                    "three formats read back; copy-in, compute and copy-out on three streams with two "
                    "device buffer sets, so layers overlap; a layer's tensors of one kind sit in one "
                    "contiguous slab on both sides (one H2D copy and six D2H copies per layer)"}


def main_reference(args, rank, world, torch, dist):
    """The CPU oracle, as it stands, on a bounded sample of the same workload."""
    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    import workloads as W
    from oracle import oracle as O
    lay = W.qwen3_4b_layer(0, device="cpu")
    # per step: a 256-row slice of each q/k/v member (one sibling group) = 1.57 M elements
    sample = [W.bits(lay[n][:256]) for n in ("q_proj", "k_proj", "v_proj")]
    n = sum(x.size for x in sample)
    for _ in range(args.warmup):
        run_oracle_path(sample, O)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_path(sample, O)
    dt = (time.perf_counter() - t0) / args.steps
    value = n / dt
    line = {"metric": METRIC, "value": value, "unit": "elem/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "reference",
            "config": dict(bench_config(args, not args.per_tensor, world),
                           sample_per_step="256 rows of q/k/v of layer 0 (%d elements)" % n),
            "cpu_baseline": {"value": value, "unit": "elem/s", "cores": 1, "kind": "oracle",
                             "sample": "256-row slices of q/k/v (one sibling group) through every op, "
                                       "single-threaded scalar C oracle"},
            "e2e": {"value": value, "unit": "elem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
