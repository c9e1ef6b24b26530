"""Benchmark of the block-scaled quantisation path on N GPUs of one node.

Headline step (the largest workload that fits one GPU): a DeepSeek-V3-shaped
MoE layer -- 256 routed experts, gate/up [256][2048][7168] and down
[256][7168][2048], BF16 N(0, 0.01), 11.27 G elements -- quantised and
dequantised in the three formats, plus the W4A4 NVFP4 fake-quantisation of
a 16384 x 7168 BF16 activation (N(0, 1), 8 outlier channels x 20):
  fp8_block_quant -> fp8_block_dequant        (128x128 tiles, FP32 scales)
  mxfp8_quant     -> mxfp8_dequant            (1x32, UE8M0)
  nvfp4_quant (gate/up of each expert share one global amax, down alone)
                  -> nvfp4_dequant
  nvfp4_fake_quant of the activation (its own dynamic amax; the
                  straight-through backward needs no kernel)
Every op is one grouped call over the three batched expert tensors (one
kernel launch); the pages quantise these experts in FP8 block-wise and
NVFP4, and MXFP8 is added so that one step takes the experts through every
row of the path.  Each op is captured once in a CUDA graph and a step
replays the seven graphs back to back on one stream; CUDA events between
them give the per-op device times.  Inputs (22.5 GB) are larger than the
126 MB L2, so no flush is needed between steps.

`value` = elements taken through the step (experts + activation) per
second, summed over ranks (weak scaling: every rank draws its own seeded
experts; the path needs no collective).  `e2e` = the same metric through
the public Python API from pinned host memory, 16 experts at a time (plus
the activation): the H2D copy of the BF16 inputs, every op, and the D2H
read of every result -- codes and scales of the three formats and the BF16
outputs of the three dequantisers and of the fake-quantisation.

`per_config` times every workload of the benchmark set with its own launch
shape: the 256 x 512 matrix (all ops; alone and as a batch of 64), the
Qwen3-4B weight sweep (36 layers, one grouped call per two layers), the
Qwen3-30B-A3B expert layer (128 experts, MXFP8, one call per layer over 48
layers), the 2048-hidden QAT block (NVFP4 fake-quant of its sibling groups
in one launch) and the two parts of the headline.  Workloads smaller than
L2 are timed call by call with a 256 MB write between calls (L2 flushed).
`next_rows` times the FP8 block-wise re-quantisation ops, the NVFP4
"4over6" variant and NVFP4 with a given group amax on the Qwen3-4B sweep,
and the W4A4 activation observer on the headline's activation shape.  `--impl reference` times the CPU oracle (all host threads) on a
bounded sample of the headline workload.
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
WORKLOAD = "dsv3_moe_layer_256_experts_and_w4a4_activation"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20

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
QWEN_OPS = list(BYTES_PER_ELEM)
# the spec bar: every quantise / QDQ kernel at 70 % of the HBM roofline
BAR_FRAC = 0.70

# ncu DRAM traffic of one launch of a kernel in the headline launch shape,
# from its committed summary under profiles/ (the summary records the bytes
# and the sha256 of the sources the capture ran on; once a source has
# changed the figure is stale and `traffic` is reported as null)
CSRC = "precision_weight_quantization_b200/csrc/"
PROFILES = {
    "nvfp4_quant": ("profiles/nvfp4_flow_quant_dsv3_experts.md", "nvfp4.cu"),
    "nvfp4_fake_quant": ("profiles/nvfp4_flow_fake_quant_dsv3_activation.md", "nvfp4.cu"),
    "fp8_block_quant": ("profiles/fp8_block_quant_dsv3_experts.md", "fp8_block.cu"),
    "fp8_block_dequant": ("profiles/fp8_block_dequant_dsv3_experts.md", "fp8_block.cu"),
    "mxfp8_quant": ("profiles/mxfp8_quant_dsv3_experts.md", "mxfp8.cu"),
    "mxfp8_dequant": ("profiles/mxfp8_dequant_dsv3_experts.md", "mxfp8.cu"),
    "nvfp4_dequant": ("profiles/nvfp4_dequant_dsv3_experts.md", "nvfp4.cu"),
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


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="pwq", choices=["pwq", "reference"])
    ap.add_argument("--experts", type=int, default=256,
                    help="routed experts of the headline layer (256 = the DeepSeek-V3 shape)")
    ap.add_argument("--layers", type=int, default=36, help="layers of the Qwen3-4B sweep (per_config)")
    ap.add_argument("--moe-layers", type=int, default=48, help="layers of the Qwen3-30B-A3B workload (per_config)")
    ap.add_argument("--layers-per-call", type=int, default=2,
                    help="Qwen3-4B layers per grouped call (2: 14 tensors, the most one launch takes)")
    ap.add_argument("--e2e-experts", type=int, default=16, help="experts per host round trip in e2e")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--configs", default="1,2,3,4",
                    help="per_config workloads to time besides the headline (1 small, 2 Qwen3-4B, 3 Qwen3-30B, 4 QAT block)")
    ap.add_argument("--no-next", action="store_true",
                    help="skip timing the FP8 block-wise re-quantisation ops (reported under next_rows)")
    ap.add_argument("--per-tensor", action="store_true",
                    help="Qwen3-4B sweep: one call per tensor / sibling group instead of one grouped call")
    return ap.parse_args(argv)


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


# ------------------------------------------------------------------ ops and workloads

class Op:
    """One op of a workload: its calls (closures over pre-allocated inputs
    and outputs, one kernel launch each), the elements they process and the
    algorithmic bytes per element of its kind."""

    def __init__(self, name, kind, calls, elems, kernels_per_call=1):
        self.name, self.kind, self.calls, self.elems = name, kind, calls, int(elems)
        self.kernels_per_call = kernels_per_call
        self.bpe = BYTES_PER_ELEM[kind]
        self.one_pass = ONE_PASS_BYTES_PER_ELEM.get(kind)

    @property
    def launches(self):
        return len(self.calls) * self.kernels_per_call

    def run(self):
        for c in self.calls:
            c()


class Workload:
    def __init__(self, name, ops, elems, config, tensors=None):
        self.name, self.ops, self.elems, self.config = name, ops, int(elems), config
        self.tensors = tensors or {}


def op_fields(op, ms, hbm_peak, peak_kind):
    gbs = op.elems * op.bpe / (ms / 1e3) / 1e9
    d = {"ms": round(ms, 5), "elements": op.elems, "elem_per_s": op.elems / (ms / 1e3),
         "alg_gbs": round(gbs, 1), "frac_of_%s_hbm" % peak_kind: round(gbs / hbm_peak, 4),
         "launches": op.launches, "bytes_per_elem": round(op.bpe, 5)}
    if op.one_pass is not None:
        g1 = op.elems * op.one_pass / (ms / 1e3) / 1e9
        d.update({"alg_gbs_one_pass": round(g1, 1), "frac_of_%s_hbm_one_pass" % peak_kind: round(g1 / hbm_peak, 4),
                  "bytes_per_elem_one_pass": round(op.one_pass, 5)})
    return d


def dsv3_workload(P, torch, dev, rank=0, experts=256):
    """The headline: DeepSeek-V3 expert layer (three batched tensors) and
    the W4A4 activation.  One grouped call (one launch) per op."""
    import workloads as W
    ex = W.dsv3_experts(device=dev, experts=experts, seed=5000 + 1000 * rank)
    names = [n for n, _ in W.DSV3_EXPERT_SHAPES]
    xs = [ex[n] for n in names]
    f8 = torch.float8_e4m3fn
    q = [torch.empty(x.shape, dtype=f8, device=dev) for x in xs]
    s = [torch.empty((x.shape[0], -(-x.shape[1] // 128), -(-x.shape[2] // 128)), dtype=torch.float32, device=dev)
         for x in xs]
    mq = [torch.empty(x.shape, dtype=f8, device=dev) for x in xs]
    me = [torch.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=torch.uint8, device=dev) for x in xs]
    pk = [torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device=dev) for x in xs]
    sb = [torch.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=f8, device=dev) for x in xs]
    gs = [torch.empty(experts, dtype=torch.float32, device=dev) for _ in range(2)]   # {gate, up}, {down}
    y = [torch.empty_like(x) for x in xs]      # BF16 output shared by the three dequantisers
    act = W.dsv3_activation(device=dev, seed=5100 + 1000 * rank)
    yact = torch.empty_like(act)
    act_amax = torch.empty(1, dtype=torch.float32, device=dev)
    E = sum(x.numel() for x in xs)
    groups = [[xs[0], xs[1]], [xs[2]]]
    ops = [
        Op("fp8_block_quant", "fp8_block_quant", [lambda: P.fp8_block_quant_grouped(xs, out=q, scale=s)], E),
        Op("fp8_block_dequant", "fp8_block_dequant", [lambda: P.fp8_block_dequant_grouped(q, s, out=y)], E),
        Op("mxfp8_quant", "mxfp8_quant", [lambda: P.mxfp8_quant_grouped(xs, out=mq, scale=me)], E),
        Op("mxfp8_dequant", "mxfp8_dequant", [lambda: P.mxfp8_dequant_grouped(mq, me, out=y)], E),
        Op("nvfp4_quant", "nvfp4_quant",
           [lambda: P.nvfp4_quant_grouped(groups, out=[pk[:2], pk[2:]], sb=[sb[:2], sb[2:]], global_scale=gs)], E),
        Op("nvfp4_dequant", "nvfp4_dequant",
           [lambda: P.nvfp4_dequant_grouped(pk, sb, [gs[0], gs[0], gs[1]], out=y)], E),
        Op("nvfp4_fake_quant", "nvfp4_fake_quant",
           [lambda: P.nvfp4_fake_quant(act, out=yact, amax_out=act_amax)], act.numel()),
    ]
    config = {"workload": WORKLOAD, "experts": experts,
              "tensors": "gate/up [%d][2048][7168], down [%d][7168][2048] BF16 N(0, 0.01); activation "
                         "16384x7168 BF16 N(0, 1) with 8 channels x20" % (experts, experts),
              "elements_per_rank": E + act.numel(),
              "path": "experts: fp8_block q+dq, mxfp8 q+dq, nvfp4 q (gate/up siblings per expert)+dq; "
                      "activation: nvfp4 fake-quant (W4A4, dynamic amax)",
              "launch": "one grouped call (one launch) per op; one CUDA graph per op, replayed back to back",
              "l2": "inputs larger than L2 (22.7 GB per rank), no flush"}
    tensors = dict(xs=xs, q=q, s=s, mq=mq, me=me, pk=pk, sb=sb, gs=gs, y=y, act=act, yact=yact, act_amax=act_amax,
                   names=names)
    return Workload("5_dsv3_experts_and_w4a4_activation", ops, E + act.numel(), config, tensors)


# ---- Qwen3-4B weight sweep (36 layers x 7 tensors)

def make_layers(n_layers, device, rank):
    import workloads as W
    return [W.qwen3_4b_layer(L + 1000 * rank, device=device) for L in range(n_layers)]


def layer_elems():
    import workloads as W
    return sum(r * c for _, (r, c) in W.QWEN3_4B_LAYER)


class Buffers:
    """Pre-allocated outputs for every op of every Qwen3-4B layer."""

    def __init__(self, layers, P, torch, per_call=1):
        import workloads as W
        self.fp8 = []
        self.mx = []
        self.nv = []
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


def qwen3_4b_workload(P, torch, dev, rank=0, layers=36, per_call=2, grouped=True):
    lays = make_layers(layers, dev, rank)
    buf = Buffers(lays, P, torch, per_call)
    E = layer_elems() * layers
    ops = [Op(op, op, op_calls(op, lays, buf, P, grouped, per_call), E) for op in QWEN_OPS]
    config = {"workload": "qwen3_4b_weight_sweep_%dx7" % layers, "layers": layers,
              "tensors": "q 4096x2560, k/v 1024x2560, o 2560x4096, gate/up 9728x2560, down 2560x9728",
              "path": "fp8_block q+dq, mxfp8 q+dq, nvfp4 q (qkv, gate/up siblings)+dq, nvfp4 fake-quant (siblings)",
              "launch": ("one grouped call (one launch) per op per %d layers (%d tensors)" % (per_call, 7 * per_call)
                         if grouped else "one call per tensor"),
              "l2": "inputs larger than L2 (%.1f GB per rank), no flush" % (2 * E / 1e9)}
    return Workload("2_qwen3_4b_weight_sweep", ops, E, config, dict(layers=lays, buf=buf, per_call=per_call))


def qwen3_30b_workload(P, torch, dev, rank=0, layers=48, layer_index=None):
    """128 batched experts per tensor kind, MXFP8 quant and dequant of all
    of them in one grouped call per layer; one layer's buffers serve all
    layers (1.2 GB of BF16, larger than L2).  layer_index picks the seeded
    layer drawn (default: one per rank)."""
    import workloads as W
    lay = W.qwen3_30b_moe_layer(1000 * rank if layer_index is None else layer_index, device=dev)
    xs = [lay[n] for n, _ in W.QWEN3_30B_EXPERT_SHAPES]
    q = [torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=dev) for x in xs]
    e = [torch.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=torch.uint8, device=dev) for x in xs]
    y = [torch.empty_like(x) for x in xs]
    E1 = sum(x.numel() for x in xs)
    ops = [Op("mxfp8_quant", "mxfp8_quant", [lambda: P.mxfp8_quant_grouped(xs, out=q, scale=e)] * layers, E1 * layers),
           Op("mxfp8_dequant", "mxfp8_dequant", [lambda: P.mxfp8_dequant_grouped(q, e, out=y)] * layers, E1 * layers)]
    config = {"workload": "qwen3_30b_a3b_moe_mxfp8_%d_layers" % layers,
              "tensors": "128 experts: gate/up [128][768][2048], down [128][2048][768] BF16 N(0, 0.02) x "
                         "per-expert LogUniform(0.5, 2)",
              "launch": "one grouped call (one launch) per layer and op, %d layers, one layer's buffers reused"
                        % layers,
              "l2": "inputs larger than L2 (1.2 GB per layer), no flush"}
    return Workload("3_qwen3_30b_a3b_moe_mxfp8", ops, E1 * layers, config, dict(xs=xs, q=q, e=e, y=y))


def block2048_workload(P, torch, dev):
    """The 2048-hidden QAT block: its three sibling groups fake-quantised in
    one single-pass launch (W4A16); the straight-through backward is the
    identity and launches nothing."""
    import workloads as W
    blk = W.block2048(device=dev)
    groups = [[blk[n] for n in g] for g in W.BLOCK2048_GROUPS]
    ys = [[torch.empty_like(x) for x in g] for g in groups]
    amax = [torch.empty(1, dtype=torch.float32, device=dev) for _ in groups]
    E = sum(x.numel() for g in groups for x in g)
    ops = [Op("nvfp4_fake_quant", "nvfp4_fake_quant",
              [lambda: P.nvfp4_fake_quant_grouped(groups, out=ys, amax_out=amax)], E)]
    config = {"workload": "block2048_nvfp4_qat_w4a16",
              "tensors": "q 4096x2048, k/v 512x2048 (siblings), gate/up 6144x2048 (siblings), down 2048x6144; "
                         "N(0, 0.02) + 0.05%% x100",
              "launch": "one grouped call (one launch) over the three sibling groups; STE backward: identity, "
                        "no kernel",
              "l2": "flushed before every timed call (inputs 96 MB, smaller than L2)"}
    return Workload("4_block2048_nvfp4_qat", ops, E, config, dict(blk=blk, groups=groups, ys=ys, amax=amax))


def small_workload(P, torch, dev, batch=1):
    """The 256 x 512 matrix through every op (batch > 1: that many copies as
    one batched tensor, each copy its own NVFP4 group)."""
    import workloads as W
    x = W.small_matrix(device="cpu").to(dev)
    if batch > 1:
        x = x.unsqueeze(0).repeat(batch, 1, 1).contiguous()
    f8 = torch.float8_e4m3fn
    M, N = x.shape[-2:]
    lead = tuple(x.shape[:-2])
    q = torch.empty(x.shape, dtype=f8, device=dev)
    s = torch.empty(lead + (-(-M // 128), -(-N // 128)), dtype=torch.float32, device=dev)
    mq = torch.empty(x.shape, dtype=f8, device=dev)
    me = torch.empty(x.shape[:-1] + (N // 32,), dtype=torch.uint8, device=dev)
    pk = torch.empty(x.shape[:-1] + (N // 2,), dtype=torch.uint8, device=dev)
    sb = torch.empty(x.shape[:-1] + (N // 16,), dtype=f8, device=dev)
    gs = torch.empty(batch, dtype=torch.float32, device=dev)
    y = torch.empty_like(x)
    E = x.numel()
    ops = [Op("fp8_block_quant", "fp8_block_quant", [lambda: P.fp8_block_quant(x, out=q, scale=s)], E),
           Op("fp8_block_dequant", "fp8_block_dequant", [lambda: P.fp8_block_dequant(q, s, out=y)], E),
           Op("mxfp8_quant", "mxfp8_quant", [lambda: P.mxfp8_quant(x, out=mq, scale=me)], E),
           Op("mxfp8_dequant", "mxfp8_dequant", [lambda: P.mxfp8_dequant(mq, me, out=y)], E),
           Op("nvfp4_quant", "nvfp4_quant", [lambda: P.nvfp4_quant(x, out=[pk], sb=[sb], global_scale=gs)], E),
           Op("nvfp4_dequant", "nvfp4_dequant", [lambda: P.nvfp4_dequant(pk, sb, gs, out=y)], E),
           Op("nvfp4_fake_quant", "nvfp4_fake_quant", [lambda: P.nvfp4_fake_quant(x, out=y)], E)]
    config = {"workload": "small_256x512" + ("_batch%d" % batch if batch > 1 else ""),
              "tensors": "256x512 BF16 N(0, 0.02), 131 entries x50" + (", %d copies as one batch" % batch
                                                                        if batch > 1 else ""),
              "launch": "one call (one launch) per op",
              "l2": "flushed before every timed call"}
    return Workload("1_small_256x512" + ("_batch%d" % batch if batch > 1 else ""), ops, E, config,
                    dict(x=x, q=q, s=s, mq=mq, me=me, pk=pk, sb=sb, gs=gs, y=y))


# ------------------------------------------------------------------ timing

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


def time_back_to_back(ops, torch, steps, warmup, barrier=None, clocks=None):
    """Each op in its own graph, the graphs of a step replayed back to back;
    returns (ms per step, {op name: ms per step}, clock summary)."""
    graphs = [capture(op.calls, torch) for op in ops]
    stream = torch.cuda.current_stream()

    def step(evs=None):
        for k, g in enumerate(graphs):
            if evs is not None:
                evs[k].record(stream)
            g.replay()
        if evs is not None:
            evs[len(graphs)].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clk = Clocks(torch.cuda.current_device()) if clocks else None
    if clk:
        clk.__enter__()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        step(evsets[i])
    end.record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.__exit__()
    if barrier:
        barrier()
    per = {op.name: sum(evs[k].elapsed_time(evs[k + 1]) for evs in evsets) / steps for k, op in enumerate(ops)}
    del graphs
    return start.elapsed_time(end) / steps, per, (clk.summary() if clk else None)


def time_flushed(ops, torch, iters, warmup):
    """Each op's graph replayed `iters` times, a write of L2_FLUSH_BYTES
    before every replay; the replay alone is timed (median)."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    out = {}
    for op in ops:
        g = capture(op.calls, torch)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        for i in range(warmup + iters):
            flush.zero_()
            if i >= warmup:
                evs[i - warmup][0].record(stream)
            g.replay()
            if i >= warmup:
                evs[i - warmup][1].record(stream)
        torch.cuda.synchronize()
        out[op.name] = statistics.median(a.elapsed_time(b) for a, b in evs)
        del g
    return out


def bars(per_op, peak_kind):
    """Which quantise / QDQ kernels meet the 70 % bar."""
    key = "frac_of_%s_hbm" % peak_kind
    return {op: d[key] >= BAR_FRAC for op, d in per_op.items() if key in d}


def config_entry(w, per_ms, hbm_peak, peak_kind, extra=None):
    per_op = {op.name: op_fields(op, per_ms[op.name], hbm_peak, peak_kind) for op in w.ops}
    d = dict(w.config)
    d["ops"] = per_op
    d["meets_%d_pct_bar" % int(BAR_FRAC * 100)] = bars(per_op, peak_kind)
    if extra:
        d.update(extra)
    return d


# ------------------------------------------------------------------ the FP8 block-wise re-quantisation row

# FP8 block-wise codes + tile scales (the sweep's fp8_block_quant outputs)
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
    scales the sweep wrote; every layer writes its own outputs (no call
    writes over lines a previous call left in L2).  Returns the calls and
    their outputs per layer."""
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
    return calls, {"q": out_q, "s": out_s, "e": out_e, "pk": pk, "sb": sb, "gs": gsc, "codes": general}


# NVFP4 "4over6" (E4M3 maximum 256) of the BF16 sweep, one grouped call per
# `per_call` layers (their sibling groups): the group amax launch and the
# encode launch that evaluates both block candidates; algorithmic bytes as
# for NVFP4 (two reads of the input)
FOUR_SIX_BYTES_PER_ELEM = {"nvfp4_4over6_quant": 2 + 2 + 0.5 + 1 / 16, "nvfp4_4over6_fake_quant": 2 + 2 + 2}
FOUR_SIX_ONE_PASS_BYTES_PER_ELEM = {"nvfp4_4over6_quant": 2 + 0.5 + 1 / 16, "nvfp4_4over6_fake_quant": 2 + 2}


def four_six_calls(op, layers, P, torch, per_call=1):
    """One grouped call per `per_call` layers, every layer writing its own
    outputs.  Returns the calls and, per call, its groups and outputs."""
    import workloads as W
    calls, outs = [], []
    for i0 in range(0, len(layers), per_call):
        groups = [[lay[n] for n in grp] for lay in layers[i0:i0 + per_call] for grp in W.QWEN3_4B_GROUPS]
        dev = groups[0][0].device
        if op == "nvfp4_4over6_quant":
            pk = [[torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device=dev) for x in g] for g in groups]
            sb = [[torch.empty((x.shape[0], x.shape[1] // 16), dtype=torch.float8_e4m3fn, device=dev) for x in g]
                  for g in groups]
            gs = [torch.empty(1, dtype=torch.float32, device=dev) for _ in groups]
            calls.append(lambda groups=groups, pk=pk, sb=sb, gs=gs:
                         P.nvfp4_4over6_quant_grouped(groups, 256, out=pk, sb=sb, global_scale=gs))
            outs.append((groups, pk, sb, gs))
        else:
            ys = [[torch.empty_like(x) for x in g] for g in groups]
            calls.append(lambda groups=groups, ys=ys: P.nvfp4_4over6_fake_quant_grouped(groups, 256, out=ys))
            outs.append((groups, ys))
    return calls, outs


# NVFP4 with the group amax given (the path of a sibling group sharded over
# data-parallel ranks, after the all-reduce of its amax): one call per
# sibling group of the sweep, each with its amax computed before timing; one
# read of the input.  The W4A4 activation observer: observe the activation
# (one read), then fake-quantise it with the observed amax.
AMAX_IN_BYTES_PER_ELEM = {"nvfp4_quant_amax_in": 2 + 0.5 + 1 / 16, "nvfp4_fake_quant_amax_in": 2 + 2}
OBSERVER_BYTES_PER_ELEM = 2 + 2 + 2
OBSERVER_ONE_PASS_BYTES_PER_ELEM = 2 + 2


def amax_in_calls(op, layers, P, torch):
    """One call per sibling group of every layer, with its precomputed amax."""
    import workloads as W
    calls = []
    for lay in layers:
        for grp in W.QWEN3_4B_GROUPS:
            xs = [lay[n] for n in grp]
            dev = xs[0].device
            amax = P.nvfp4_group_amax(xs)
            if op == "nvfp4_quant_amax_in":
                pk = [torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device=dev) for x in xs]
                sb = [torch.empty((x.shape[0], x.shape[1] // 16), dtype=torch.float8_e4m3fn, device=dev) for x in xs]
                gs = torch.empty(1, dtype=torch.float32, device=dev)
                calls.append(lambda xs=xs, amax=amax, pk=pk, sb=sb, gs=gs:
                             P.nvfp4_quant(xs, amax=amax, out=pk, sb=sb, global_scale=gs))
            else:
                ys = [torch.empty_like(x) for x in xs]
                calls.append(lambda xs=xs, amax=amax, ys=ys: P.nvfp4_fake_quant(xs, amax=amax, out=ys))
    return calls


def time_graph(calls, args, torch):
    """ms per replay of one CUDA graph of `calls` (warm-up replays first)."""
    stream = torch.cuda.current_stream()
    g = capture(calls, torch)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    n = max(1, min(args.steps, 10))
    a.record(stream)
    for _ in range(n):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / n


def row_entry(ms, elems, bpe, one_pass, launches, hbm_peak, peak_kind):
    gbs = elems * bpe / (ms / 1e3) / 1e9
    e = {"ms": round(ms, 4), "elem_per_s": elems / (ms / 1e3), "alg_gbs": round(gbs, 1),
         "frac_of_%s_hbm" % peak_kind: round(gbs / hbm_peak, 4), "launches": launches,
         "bytes_per_elem": round(bpe, 5)}
    if one_pass is not None:
        g1 = elems * one_pass / (ms / 1e3) / 1e9
        e.update({"alg_gbs_one_pass": round(g1, 1), "frac_of_%s_hbm_one_pass" % peak_kind: round(g1 / hbm_peak, 4)})
    return e


def time_next_rows(args, w, P, torch, hbm_peak, peak_kind):
    """Device time of each re-quantisation op, of the NVFP4 4over6 variant
    and of NVFP4 with a given amax over the Qwen3-4B sweep, and of the W4A4
    activation observer (each its own CUDA graph, replayed after the sweep's
    timing)."""
    import workloads as W
    layers, buf = w.tensors["layers"], w.tensors["buf"]
    elems = layer_elems() * len(layers)
    out = {}
    one_pass = dict(NEXT_ONE_PASS_BYTES_PER_ELEM)
    one_pass.update(FOUR_SIX_ONE_PASS_BYTES_PER_ELEM)
    for op, bpe in NEXT_BYTES_PER_ELEM.items():
        calls, _ = next_calls(op, layers, buf, P, torch, w.tensors["per_call"])
        out[op] = row_entry(time_graph(calls, args, torch), elems, bpe, one_pass.get(op), len(calls), hbm_peak,
                            peak_kind)
    for op, bpe in FOUR_SIX_BYTES_PER_ELEM.items():
        calls, _ = four_six_calls(op, layers, P, torch, w.tensors["per_call"])
        out[op] = row_entry(time_graph(calls, args, torch), elems, bpe, one_pass.get(op), 2 * len(calls), hbm_peak,
                            peak_kind)
    for op, bpe in AMAX_IN_BYTES_PER_ELEM.items():
        calls = amax_in_calls(op, layers, P, torch)
        out[op] = row_entry(time_graph(calls, args, torch), elems, bpe, None, len(calls), hbm_peak, peak_kind)
    # the W4A4 activation observer (static_minmax) on the 16384 x 7168 activation
    x = W.dsv3_activation(device=layers[0]["q_proj"].device)
    y = torch.empty_like(x)
    obs = P.NVFP4ActivationObserver("static_minmax", device=x.device)
    ms = time_graph([lambda: obs.fake_quant(x, out=y)], args, torch)
    out["nvfp4_w4a4_observer_fake_quant"] = row_entry(ms, x.numel(), OBSERVER_BYTES_PER_ELEM,
                                                      OBSERVER_ONE_PASS_BYTES_PER_ELEM, 3, hbm_peak, peak_kind)
    out["nvfp4_w4a4_observer_fake_quant"]["workload"] = "16384x7168 activation, observe (2 launches) + fake-quantise"
    del x, y
    return out


# ------------------------------------------------------------------ CPU oracle timing

def oracle_path(xs_bits, PO, threads):
    """The oracle (threaded driver) through the headline path for one expert:
    FP8 block-wise and MXFP8 quantise + dequantise of each tensor, NVFP4 of
    the {gate, up} group and of down, quantise + dequantise."""
    for x in xs_bits:
        q, s = PO.fp8_block_quant(x, threads)
        PO.fp8_block_dequant(q, s, threads)
        q, e = PO.mxfp8_quant(x, threads)
        PO.mxfp8_dequant(q, e, threads)
    for grp in (xs_bits[:2], xs_bits[2:]):
        A = PO.nvfp4_group_amax(grp, threads)
        for x in grp:
            pk, sb, gs = PO.nvfp4_quant(x, A, threads)
            PO.nvfp4_dequant(pk, sb, gs, x.shape[-1], threads)


def cpu_baseline(expert_bits):
    """The oracle as it stands on expert 0 of the headline layer, once on
    one thread and once on every host thread."""
    from oracle import parallel as PO
    n = sum(x.size for x in expert_bits)
    nthreads = PO.host_threads()
    rates = {}
    for th in (1, nthreads):
        t0 = time.perf_counter()
        oracle_path(expert_bits, PO, th)
        rates[th] = (n / (time.perf_counter() - t0), time.perf_counter() - t0)
    return {"value": rates[nthreads][0], "unit": "elem/s", "cores": nthreads, "kind": "oracle",
            "single_thread_value": rates[1][0], "host_threads": nthreads, "nproc": os.cpu_count(),
            "sample": "expert 0 of the headline layer (gate/up 2048x7168 as one NVFP4 sibling group, down "
                      "7168x2048): %d elements through fp8_block q+dq, mxfp8 q+dq, nvfp4 q+dq; scalar C oracle, "
                      "%.1f s on 1 thread, %.1f s on %d threads (rows split evenly)"
                      % (n, rates[1][1], rates[nthreads][1], nthreads)}


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
    barrier = dist.barrier if world > 1 else None

    # ---- headline: DeepSeek-V3 expert layer + W4A4 activation
    w5 = dsv3_workload(P, torch, dev, rank, args.experts)
    ms_step, per_ms, clocks = time_back_to_back(w5.ops, torch, args.steps, args.warmup, barrier, clocks=True)
    t = torch.tensor([ms_step], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    value = w5.elems * world / (ms_max / 1e3)
    per_op = {op.name: op_fields(op, per_ms[op.name], hbm_peak, peak_kind) for op in w5.ops}
    dom = max(w5.ops, key=lambda o: per_ms[o.name])
    avg_launch_ms = per_ms[dom.name] / dom.launches
    alg_bytes = dom.elems * dom.bpe / dom.launches
    achieved = alg_bytes / (avg_launch_ms / 1e3) / 1e9
    traffic, traffic_note = recorded_traffic(dom.name)
    roofline = {"bound": "hbm", "kernel": dom.name, "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                "alg_bytes_per_launch": int(round(alg_bytes)), "avg_launch_us": round(avg_launch_ms * 1e3, 2),
                "note": "achieved = algorithmic bytes of one launch / its duration (CUDA events around the op's "
                        "graph in every timed step); traffic: %s" % traffic_note}
    if dom.one_pass is not None:
        one = dom.elems * dom.one_pass / dom.launches / (avg_launch_ms / 1e3) / 1e9
        roofline.update({"achieved_one_pass": round(one, 1), "frac_one_pass": round(one / hbm_peak, 4)})
        roofline["note"] += ("; achieved counts the amax pass's read of the input (two reads, as the method is "
                             "defined); *_one_pass counts a single read, the stricter ideal")
    launches_per_step = sum(op.launches for op in w5.ops)
    line = {"metric": METRIC, "value": value, "unit": "elem/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(w5.config, parallelism="dp%d (independent experts per rank)" % world),
            "per_op": per_op, "roofline": roofline, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks if rank == 0 else None}
    per_config = {}
    per_config["5a_dsv3_experts"] = config_entry(
        Workload("5a", [o for o in w5.ops if o.name != "nvfp4_fake_quant"], 0,
                 {"workload": "dsv3_experts_%d" % args.experts}), per_ms, hbm_peak, peak_kind,
        {"source": "the headline step"})
    per_config["5b_dsv3_w4a4_activation"] = config_entry(
        Workload("5b", [o for o in w5.ops if o.name == "nvfp4_fake_quant"], 0,
                 {"workload": "dsv3_w4a4_activation_16384x7168"}), per_ms, hbm_peak, peak_kind,
        {"source": "the headline step"})
    expert0 = None
    if rank == 0 and not args.no_cpu_baseline:
        import workloads as W
        expert0 = [W.bits(w5.tensors["xs"][i][0]) for i in range(3)]
    if not args.no_e2e:
        line["e2e"] = e2e(args, w5, P, torch, dev, world, dist)
    del w5
    torch.cuda.empty_cache()

    if not args.no_per_config:
        per_config.update(time_per_config(args, P, torch, dev, rank, hbm_peak, peak_kind, line))
    line["per_config"] = per_config
    if expert0 is not None:
        line["cpu_baseline"] = cpu_baseline(expert0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def time_per_config(args, P, torch, dev, rank, hbm_peak, peak_kind, line):
    out = {}
    steps = max(1, min(args.steps, 10))
    want = set(args.configs.split(","))
    if "2" in want:
        time_qwen3_4b(args, P, torch, dev, rank, hbm_peak, peak_kind, line, out, steps)
    if "3" in want:
        time_qwen3_30b(args, P, torch, dev, rank, hbm_peak, peak_kind, out, steps)
    small = []
    if "4" in want:
        small.append(block2048_workload(P, torch, dev))
    if "1" in want:
        small += [small_workload(P, torch, dev, 1), small_workload(P, torch, dev, 64)]
    # small workloads: L2 flushed before every timed call
    for w in small:
        per = time_flushed(w.ops, torch, iters=max(5, steps), warmup=args.warmup)
        e = config_entry(w, per, hbm_peak, peak_kind)
        if w.name.startswith("4_"):
            e["ste_backward"] = "grad_x = grad_y (identity): no kernel, 0 bytes"
        out[w.name] = e
    del small
    torch.cuda.empty_cache()
    return out


def time_qwen3_4b(args, P, torch, dev, rank, hbm_peak, peak_kind, line, out, steps):
    """The Qwen3-4B sweep (and the re-quantisation row on its FP8 outputs)."""
    w2 = qwen3_4b_workload(P, torch, dev, rank, args.layers, max(1, args.layers_per_call), not args.per_tensor)
    ms, per, _ = time_back_to_back(w2.ops, torch, steps, args.warmup)
    out[w2.name] = config_entry(w2, per, hbm_peak, peak_kind,
                                {"ms_per_step": round(ms, 4), "elem_per_s_whole_path": w2.elems / (ms / 1e3)})
    if not args.no_next:
        w2.ops[0].run()
        line["next_rows"] = time_next_rows(args, w2, P, torch, hbm_peak, peak_kind)
    del w2
    torch.cuda.empty_cache()


def time_qwen3_30b(args, P, torch, dev, rank, hbm_peak, peak_kind, out, steps):
    """Qwen3-30B-A3B experts, MXFP8 per layer."""
    w3 = qwen3_30b_workload(P, torch, dev, rank, args.moe_layers)
    ms, per, _ = time_back_to_back(w3.ops, torch, steps, args.warmup)
    e = config_entry(w3, per, hbm_peak, peak_kind)
    for name, d in e["ops"].items():
        d["us_per_layer"] = round(d["ms"] * 1e3 / args.moe_layers, 2)
    out[w3.name] = e
    del w3
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ end to end through the public API

def e2e(args, w5, P, torch, dev, world, dist):
    """The headline path through the public Python API from pinned host
    memory: per chunk of experts an H2D copy of the BF16 inputs, every op
    (one grouped call each) and a D2H read of every result (codes and scales
    of the three formats, BF16 outputs of the three dequantisers); the
    activation once per step (H2D, fake-quant, D2H).  Copy-in, compute and
    copy-out run on three streams over two device buffer sets, so chunks
    overlap; a chunk's tensors of one kind sit in one contiguous slab on
    both sides (one copy per kind).  The same host input chunk feeds every
    chunk of the layer, and every chunk's results land in the same host
    slabs."""
    import workloads as W
    E = args.experts
    C = max(1, min(args.e2e_experts, E))
    n_chunks = -(-E // C)
    names = [n for n, _ in W.DSV3_EXPERT_SHAPES]
    shp = {n: (C,) + tuple(s) for n, s in W.DSV3_EXPERT_SHAPES}

    def slab(kind_shapes, dtype, device=None, pinned=False):
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

    tile = {n: (C, -(-s[1] // 128), -(-s[2] // 128)) for n, s in shp.items()}
    mxs = {n: (C, s[1], s[2] // 32) for n, s in shp.items()}
    pks = {n: (C, s[1], s[2] // 2) for n, s in shp.items()}
    sbs = {n: (C, s[1], s[2] // 16) for n, s in shp.items()}
    gss = {"gate_up": (C,), "down": (C,)}
    kinds = (("q", shp, torch.uint8), ("s", tile, torch.float32), ("mq", shp, torch.uint8),
             ("me", mxs, torch.uint8), ("pk", pks, torch.uint8), ("sb", sbs, torch.uint8),
             ("gs", gss, torch.float32), ("y8", shp, torch.bfloat16), ("ymx", shp, torch.bfloat16),
             ("ynv", shp, torch.bfloat16))
    host_x, hx = slab(shp, torch.bfloat16, pinned=True)
    for n in names:
        hx[n].copy_(w5.tensors["xs"][names.index(n)][:C].cpu())
    host_out = {k: slab(sh, dt, pinned=True)[0] for k, sh, dt in kinds}
    act_h = w5.tensors["act"].cpu().pin_memory()
    act_out_h = torch.empty_like(act_h).pin_memory()
    act_d = torch.empty_like(w5.tensors["act"])
    act_y = torch.empty_like(act_d)

    def device_set():
        d = {}
        d["x_flat"], d["x"] = slab(shp, torch.bfloat16, device=dev)
        for k, sh, dt in kinds:
            d[k + "_flat"], d[k] = slab(sh, dt, device=dev)
        return d

    sets = [device_set(), device_set()]
    out_bytes = sum(t.numel() * t.element_size() for t in host_out.values())
    in_bytes = host_x.numel() * 2
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "comp", "out")}
    started = {k: [False, False] for k in ("comp", "out")}
    f8 = torch.float8_e4m3fn

    def one_chunk(i):
        b = i % 2
        d = sets[b]
        with torch.cuda.stream(s_in):
            if started["comp"][b]:
                s_in.wait_event(ev["comp"][b])        # the chunk that last read this input set is done
            d["x_flat"].copy_(host_x, non_blocking=True)
            ev["in"][b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["in"][b])
            if started["out"][b]:
                s_comp.wait_event(ev["out"][b])       # this output set has been read back
            xs = [d["x"][n] for n in names]
            q = [d["q"][n].view(f8) for n in names]
            sc = [d["s"][n] for n in names]
            mq = [d["mq"][n].view(f8) for n in names]
            me = [d["me"][n] for n in names]
            pk = [d["pk"][n] for n in names]
            sb = [d["sb"][n].view(f8) for n in names]
            gs = [d["gs"]["gate_up"], d["gs"]["down"]]
            P.fp8_block_quant_grouped(xs, out=q, scale=sc)
            P.fp8_block_dequant_grouped(q, sc, out=[d["y8"][n] for n in names])
            P.mxfp8_quant_grouped(xs, out=mq, scale=me)
            P.mxfp8_dequant_grouped(mq, me, out=[d["ymx"][n] for n in names])
            P.nvfp4_quant_grouped([xs[:2], xs[2:]], out=[pk[:2], pk[2:]], sb=[sb[:2], sb[2:]], global_scale=gs)
            P.nvfp4_dequant_grouped(pk, sb, [gs[0], gs[0], gs[1]], out=[d["ynv"][n] for n in names])
            ev["comp"][b].record(s_comp)
            started["comp"][b] = True
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            for k, _, _ in kinds:
                host_out[k].copy_(d[k + "_flat"], non_blocking=True)
            ev["out"][b].record(s_out)
            started["out"][b] = True

    def activation():
        with torch.cuda.stream(s_comp):
            act_d.copy_(act_h, non_blocking=True)
            P.nvfp4_fake_quant(act_d, out=act_y)
            act_out_h.copy_(act_y, non_blocking=True)

    def run():
        activation()
        for i in range(n_chunks):
            one_chunk(i)
        cur = torch.cuda.current_stream()
        cur.wait_stream(s_in)
        cur.wait_stream(s_comp)
        cur.wait_stream(s_out)

    steps = max(1, args.steps)
    run()                                             # warm-up pass
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
        run()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    act_bytes = act_h.numel() * 2
    return {"value": w5.elems * world / (ms / 1e3), "unit": "elem/s",
            "h2d_bytes_per_step": in_bytes * n_chunks + act_bytes,
            "d2h_bytes_per_step": out_bytes * n_chunks + act_bytes,
            "ms_per_step": ms, "steps": steps,
            "note": "public Python API (one grouped call per op per chunk of %d experts), from pinned host memory "
                    "(the same host chunk feeds every chunk), every result read back: codes + scales of the "
                    "three formats, NVFP4 global scales, the BF16 outputs of the three dequantisers and of the "
                    "activation's fake-quant; copy-in, compute and copy-out on three streams with two device "
                    "buffer sets" % C}


# ------------------------------------------------------------------ reference arm

def main_reference(args, rank, world, torch, dist):
    """The CPU oracle, as it stands, on every host thread, on a bounded sample
    of the headline workload per step: 256-row slices of one expert's gate,
    up and down and of the activation."""
    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    import numpy as np
    import workloads as W
    from oracle import parallel as PO
    threads = PO.host_threads()
    rows = 256
    samples = []
    for e in range(4):
        xs = [W.bits(W.normal_bf16((rows,) + tuple(s)[1:], 0.01, seed=5000 + 10 * e + t))
              for t, (n, s) in enumerate(W.DSV3_EXPERT_SHAPES)]
        samples.append(xs)
    act = W.bits(W.normal_bf16((rows, 7168), 1.0, seed=5100))
    n = sum(x.size for x in samples[0]) + act.size

    def step(i):
        xs = samples[i % len(samples)]
        oracle_path(xs, PO, threads)
        PO.nvfp4_fake_quant(act, PO.nvfp4_group_amax([act], threads), threads)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = n / dt
    cfg = {"workload": WORKLOAD, "experts": args.experts,
           "sample_per_step": "256 rows of one expert's gate, up, down and of the activation (%d elements)" % n}
    line = {"metric": METRIC, "value": value, "unit": "elem/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "reference", "config": cfg,
            "cpu_baseline": {"value": value, "unit": "elem/s", "cores": threads, "kind": "oracle",
                             "nproc": os.cpu_count(),
                             "sample": "256-row slices of one expert's gate/up/down (FP8 block-wise and MXFP8 "
                                       "q+dq, NVFP4 q+dq with gate/up siblings) and of the activation (NVFP4 "
                                       "fake-quant), scalar C oracle on %d host threads" % threads},
            "e2e": {"value": value, "unit": "elem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
