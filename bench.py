"""Throughput of one EDiT linear compressed attention layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload px4096] [--impl ours|reference]

A step is one full layer forward (every kernel of the path) over one image
of the workload. `value` is tokens/s over all ranks (each rank runs its own
image: weak scaling, no collective on the data path), timed on the device
with CUDA events on the launching stream, L2 flushed between steps. `e2e`
is the same metric with each step's input copied from pinned host memory and
its output copied back inside the timed region; copies in, layer and copies
out run on three streams so consecutive steps overlap. `--impl reference` times the
fp64 CPU oracle on bounded crops of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time


ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_compressed_attention_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

# Stage boundaries recorded by the library's timing hook (include/edit_attn.h).
STAGES = ["kv_linear", "dwconv_s2", "kv_state", "fold_weights", "conv3x3", "groupnorm", "q_linear", "apply"]
# conv3x3 = the conv kernel alone; groupnorm = GN statistics/finalize/apply (+ the
# conv's last-wave fixup)
DOMINANT = "conv3x3"   # largest FLOP share of the layer (40%)

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the dominant kernel, from the ncu capture summarised in
# profiles/conv3x3_px4096.md; reported only while the kernel's sources are the
# ones that capture measured (hash of tc_conv.cuh + tc_gemm.cuh + common.cuh).
TRAFFIC = {"src_sha": "a0406f4948f6e4ae", "bytes_per_launch": 159911168 + 25748992}


def kernel_src_sha():
    h = hashlib.sha256()
    for f in ("tc_conv.cuh", "tc_gemm.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "linear_compressed_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def layer_flops(cfg):
    """Algorithmic FLOPs of one layer (2 per multiply-add), per step kind."""
    B, N, C, Cr = cfg["B"], cfg["H"] * cfg["W"], cfg["C"], cfg["c_red"]
    M = ((cfg["H"] + 1) // 2) * ((cfg["W"] + 1) // 2)
    d = C // cfg["heads"]
    f = {
        "conv3x3": 2.0 * B * N * Cr * 9 * C,
        "conv1x1": 2.0 * B * N * C * Cr,
        "q_linear": 2.0 * B * N * C * C,
        "kv_linear": 4.0 * B * N * C * C,
        "dwconv": 2.0 * 9 * B * M * 2 * C,
        "kv_state": 2.0 * B * M * C * (d + 1),
        "apply": 2.0 * B * N * C * (d + 1),
    }
    f["total"] = sum(f.values())
    return f


def variant_flops(cfg, qkv, proj):
    """Algorithmic FLOPs of one layer with the query / key / value processing
    qkv ('cf' | 'sc' | 'none' each) and an optional output Linear."""
    B, N, C, Cr = cfg["B"], cfg["H"] * cfg["W"], cfg["C"], cfg["c_red"]
    q, k, _ = qkv
    m = ((cfg["H"] + 1) // 2) * ((cfg["W"] + 1) // 2) if k == "sc" else N
    d = C // cfg["heads"]
    conv_fusion = 2.0 * B * N * Cr * 9 * C + 2.0 * B * N * C * Cr
    f = 2.0 * B * N * C * C + 4.0 * B * N * C * C                      # Linear_Q, Linear_K, Linear_V
    f += conv_fusion * ((q == "cf") + (k == "cf"))
    f += 2.0 * 9 * B * m * 2 * C if k == "sc" else 0.0                  # depthwise stride-2 conv
    f += 2.0 * B * m * C * (d + 1) + 2.0 * B * N * C * (d + 1)          # KV state, apply
    f += 2.0 * B * N * C * C if proj else 0.0
    return f


def min_bytes(cfg, es=2):
    B, N, C = cfg["B"], cfg["H"] * cfg["W"], cfg["C"]
    Cr = cfg["c_red"]
    weights = (9 * C * Cr + Cr * C + 3 * C * C + 18 * C) * es
    return 2 * B * N * C * es + weights


# B200 datasheet figures (dense bf16 tensor peak, HBM3e bandwidth), reported
# beside the fractions of the measured peaks.
DATASHEET = {"bf16_tflops": 2250.0, "hbm_gbs": 7700.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_id)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle
def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return 1


def oracle_layer(qkv=("cf", "sc", "sc"), proj=False):
    """The fp64 oracle's layer with the given query/key/value processing."""
    import oracle.edit_oracle as O
    if qkv == ("cf", "sc", "sc") and not proj:
        return lambda d, sub: O.edit_forward(d["x"], sub["H"], sub["W"], d, sub["heads"])
    return lambda d, sub: O.edit_variant_forward(d["x"], sub["H"], sub["W"], d, sub["heads"], *qkv, out_proj=proj)


def oracle_rate(cfg, side, reps=1, qkv=("cf", "sc", "sc"), proj=False):
    """tokens/s of the fp64 oracle on a side x side crop of the workload."""
    layer = oracle_layer(qkv, proj)
    sub = dict(cfg, B=1, H=min(side, cfg["H"]), W=min(side, cfg["W"]))
    d = make_inputs(**sub, variant_weights=qkv != ("cf", "sc", "sc") or proj)
    t0 = time.perf_counter()
    for _ in range(reps):
        layer(d, sub)
    dt = time.perf_counter() - t0
    return reps * sub["H"] * sub["W"] / dt, dt, sub


def cpu_baseline(cfg, budget_s=15.0):
    side = 16
    rate, dt, sub = oracle_rate(cfg, side)
    # grow the crop until one call takes a good part of the budget
    while dt < budget_s / 4 and side < min(cfg["H"], cfg["W"]):
        side *= 2
        rate, dt, sub = oracle_rate(cfg, side)
    reps = max(1, int(budget_s / 2 / max(dt, 1e-3)))
    rate, dt, sub = oracle_rate(cfg, side, reps)
    return {"value": rate, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle, {reps} call(s) on a {sub['H']}x{sub['W']}-token crop of the "
                      f"workload (C={cfg['C']}, {cfg['heads']} heads, same distributions), {dt:.1f} s; "
                      "its cost per token does not depend on the grid size"}


# ------------------------------------------------------------------ arms
def reduce_max(value, world, device=None):
    """Max of a per-rank float over all ranks: the whole job takes as long as
    its slowest rank (identity on one rank)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_config(cfg, rank):
    """The images rank `rank` processes: the workload's recipe with its seed
    advanced by the rank, i.e. its own share of a global batch (weak scaling;
    no data crosses ranks)."""
    return dict(cfg, seed=cfg["seed"] + rank)


def job_tokens_per_s(world, batch, tokens, steps, max_ms):
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return world * batch * tokens * steps / (max_ms / 1e3)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args, cfg):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    layer = oracle_layer(args.qkv, args.proj)
    # size each step so that warm-up + steps fit in about two minutes
    r16, _, _ = oracle_rate(cfg, 16, qkv=args.qkv, proj=args.proj)
    per_step = 60.0 / max(1, args.steps + args.warmup)
    side = 2
    while side < min(cfg["H"], cfg["W"]) and (2 * side) ** 2 / r16 <= per_step:
        side *= 2
    sub = dict(cfg, B=1, H=min(side, cfg["H"]), W=min(side, cfg["W"]))
    d = make_inputs(**sub, variant_weights=args.qkv != ("cf", "sc", "sc") or args.proj)
    for _ in range(args.warmup):
        layer(d, sub)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        layer(d, sub)
    dt = time.perf_counter() - t0
    tok = sub["H"] * sub["W"] * args.steps
    value = tok / dt
    line = {
        "impl": "reference", "metric": args.metric, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload_desc, "sample": f"{sub['H']}x{sub['W']}-token crop per step"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"fp64 numpy oracle, one {sub['H']}x{sub['W']}-token crop of the workload per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def side_measurements(dev, peaks, steps=50, warmup=5):
    """The metric's other sizes (4K and 16K tokens, and the 262K-token 8192 px
    layer), the ablation table's query/key/value processing variants (and the
    output Linear) at 65K tokens, the DiT block around the attention at 4K and
    65K tokens, and the MM-EDiT hybrid at 1024 px (4096 image + 333 prompt
    tokens): median step time with L2 flushed between steps, tokens/s and the
    fraction of each layer's roofline. The MM line adds its stage times
    (prompt projections, the two softmax passes)."""
    import torch

    from linear_compressed_attention_b200 import binding as bd

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, nstages=0):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(dev)
        evs, stage = [], []
        for s in range(steps):
            flush.zero_()
            if nstages and s == steps - 1:
                st = [torch.cuda.Event(enable_timing=True) for _ in range(nstages)]
                for e in st:
                    e.record(stream)
                bd.edit_attn_set_stage_events([e.cuda_event for e in st])
                stage = st
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if nstages and s == steps - 1:
                bd.edit_attn_set_stage_events(None)
            evs.append((e0, e1))
        torch.cuda.synchronize(dev)
        ms = statistics.median(a.elapsed_time(b) for a, b in (evs[:-1] if nstages else evs))
        return ms, stage

    res = {}
    for name in ("px1024", "px2048", "px8192"):
        cfg = dict(WORKLOADS[name])
        d = make_inputs(**cfg)
        layer = bd.EditAttention(d, cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"], cfg["dtype"], device=dev)
        x = torch.from_numpy(d["x"]).to(dev, layer.tdtype)
        out = torch.empty_like(x)
        ms, _ = timed(lambda: layer.forward(x, out))
        assert layer.status() == 0
        n = cfg["B"] * cfg["H"] * cfg["W"]
        roof = max(layer_flops(cfg)["total"] / (peaks["bf16_tflops"] * 1e12), min_bytes(cfg) / (peaks["hbm_gbs"] * 1e9))
        res[str(n)] = {"workload": name, "tokens_per_s": n / (ms / 1e3), "ms_per_step": ms,
                       "layer_roofline_frac": roof * 1e3 / ms}
        del layer, out
        if name == "px8192":
            res["row_bands_px8192"] = band_measurements(d, cfg, x, ms, flush, stream, dev)
        del x
    # the ablation table's query/key/value processing rows and the output Linear,
    # on the 65,536-token workload
    cfg = dict(WORKLOADS["px4096"], variant_weights=True)
    d = make_inputs(**cfg)
    n = cfg["B"] * cfg["H"] * cfg["W"]
    var = {}
    for qkv, proj in ((("cf", "sc", "sc"), True), (("cf", "cf", "none"), False), (("none", "sc", "sc"), False),
                      (("cf", "none", "none"), False)):
        layer = bd.EditAttention(d, cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"], cfg["dtype"], device=dev,
                                 variant=qkv, out_proj=proj)
        x = torch.from_numpy(d["x"]).to(dev, layer.tdtype)
        out = torch.empty_like(x)
        uncompressed = qkv[1] != "sc"
        ms, st = timed(lambda: layer.forward(x, out), bd.STAGE_EVENTS_EDIT if uncompressed else 0)
        assert layer.status() == 0
        extra = (2 * cfg["C"] * cfg["C"] * 2) if proj else 0
        roof = max(variant_flops(cfg, qkv, proj) / (peaks["bf16_tflops"] * 1e12),
                   (min_bytes(cfg) + extra) / (peaks["hbm_gbs"] * 1e9))
        var["-".join(qkv) + ("+out_linear" if proj else "")] = {
            "tokens_per_s": n / (ms / 1e3), "ms_per_step": ms, "gflop": variant_flops(cfg, qkv, proj) / 1e9,
            "layer_roofline_frac": roof * 1e3 / ms}
        if uncompressed and st:
            # kv_transpose_kernel (+ the VTx ones/zero rows), stage 2 of a staged step:
            # reads K'|V' (N x 2C bf16), writes KT and the value rows of VTx (N x 2C)
            # and the padding rows (heads x (NP - d) x N)
            tr_ms = st[1].elapsed_time(st[2])
            lay = layer.layout
            tr_bytes = 2 * n * 2 * cfg["C"] * 2 + cfg["heads"] * (lay["NP"] - cfg["C"] // cfg["heads"]) * lay["Mp"] * 2
            gbs = tr_bytes / (tr_ms / 1e3) / 1e9
            var["-".join(qkv)]["kv_transpose"] = {
                "ms": tr_ms, "bytes": tr_bytes, "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
                "frac": gbs / peaks["hbm_gbs"], "bound": "hbm",
                "note": "stage events of one step (no overlap with the neighbouring kernels)"}
        del layer, x, out
    res["variants_px4096"] = var
    # the DiT block around the attention (300 caption tokens, MLP 4C) at 4K and 64K tokens
    blocks = {}
    for name in ("px1024", "px4096"):
        cfg = dict(WORKLOADS[name])
        blk = dict(n_cap=300, hidden=4 * cfg["C"])
        d = make_inputs(**cfg, dit_block=blk)
        B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
        block = bd.DitBlock(d, B, H, W, blk["n_cap"], C, heads, cfg["dtype"], device=dev)
        xb = torch.from_numpy(d["x"]).to(dev, block.tdtype)
        yb = torch.from_numpy(d["y"]).to(dev, block.tdtype)
        tb = torch.from_numpy(d["t6"]).to(dev, block.tdtype)
        ob = torch.empty_like(xb)
        ms, _ = timed(lambda: block.forward(xb, yb, tb, ob))
        assert block.status() == 0
        n, nt, hid = B * H * W, B * blk["n_cap"], blk["hidden"]
        fl = (layer_flops(cfg)["total"] + 2.0 * n * C * C          # EDiT attention + its output Linear
              + 2.0 * n * C * C + 4.0 * nt * C * C + 4.0 * n * blk["n_cap"] * C + 2.0 * n * C * C  # cross-attention
              + 4.0 * n * C * hid)                                  # MLP
        by = min_bytes(cfg) + 2 * (2 * nt * C + 4 * C * C + 2 * C * hid + 6 * C)
        roof = max(fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9))
        blocks[name] = {"tokens_per_s": n / (ms / 1e3), "ms_per_step": ms, "gflop": fl / 1e9,
                        "layer_roofline_frac": roof * 1e3 / ms,
                        "workload": f"{name} grid, 300 caption tokens, MLP hidden {hid}"}
        del block, xb, yb, tb, ob
    res["dit_block"] = blocks
    cfg = dict(WORKLOADS["mm1024"])
    d = make_inputs(**cfg)
    nt = cfg["n_txt"]
    layer = bd.EditAttention(d, cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"], cfg["dtype"], n_txt=nt, mm=True,
                             device=dev)
    xi = torch.from_numpy(d["x"]).to(dev, layer.tdtype)
    xt = torch.from_numpy(d["x_txt"]).to(dev, layer.tdtype)
    oi, ot = torch.empty_like(xi), torch.empty_like(xt)
    ms, st = timed(lambda: layer.forward_mm(xi, xt, oi, ot), bd.STAGE_EVENTS_MM)
    assert layer.status() == 0
    ni, C, h = cfg["H"] * cfg["W"], cfg["C"], cfg["heads"]
    m = ((cfg["H"] + 1) // 2) * ((cfg["W"] + 1) // 2)
    sdpa_flops = 4.0 * C * (ni * nt + nt * m + nt * nt)       # QK^T and PV of the three softmax blocks
    mm_flops = layer_flops(cfg)["total"] + 2.0 * nt * C * 3 * C + sdpa_flops
    roof = max(mm_flops / (peaks["bf16_tflops"] * 1e12), min_bytes(cfg) / (peaks["hbm_gbs"] * 1e9))
    stage_ms = [st[i].elapsed_time(st[i + 1]) for i in range(len(st) - 1)] if st else []
    res["mm_edit"] = {"workload": "mm1024: MM-EDiT, 64x64 image grid (4096 tokens, M=1024) + 333 prompt tokens, "
                                  "C=1536, 24 heads x 64, bf16",
                      "tokens_per_s": (ni + nt) / (ms / 1e3), "ms_per_step": ms, "layer_roofline_frac": roof * 1e3 / ms,
                      "sdpa_gflop": sdpa_flops / 1e9,
                      "stages_ms": {"edit_part": sum(stage_ms[:8]) if len(stage_ms) > 7 else None,
                                    "prompt_projections": stage_ms[8] if len(stage_ms) > 8 else None,
                                    "image_row_softmax": stage_ms[9] if len(stage_ms) > 9 else None,
                                    "prompt_row_softmax": stage_ms[10] if len(stage_ms) > 10 else None}}
    return res


def band_measurements(d, cfg, x, full_ms, flush, stream, dev, reps=5):
    """The row-band split of one 8192 px image (seqpar: halo rows, band partials,
    records in band order, band finish) for 2 and 8 bands, run one band after
    another on this one GPU with L2 flushed before each band's kernels, as each
    rank's own GPU would start. Per band: median device time of its partials and
    of its finish. A rank of an N-GPU run would take about max(partials) +
    max(finish) plus the halo exchange and the record all-gather, which one GPU
    cannot measure; `compute_only_efficiency` = full-image layer time / (N x that
    compute time)."""
    import torch

    from linear_compressed_attention_b200 import seqpar

    H, W, C, heads = cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    x3 = x[0].reshape(H, W, C)
    out = {}
    for world in (2, 8):
        bands = [seqpar.band_bounds(H, world, r) for r in range(world)]
        layers = [seqpar.BandLayer(d, H, W, C, heads, device=dev) for _ in bands]
        exts = []
        for r0, nr in bands:
            top, bot = seqpar.halo(H, r0, nr)
            exts.append(x3[r0 - top:r0 + nr + bot].contiguous())
        records = torch.empty((world, layers[0].record_bytes), dtype=torch.uint8, device=dev)
        outs = [torch.empty((nr, W, C), dtype=torch.bfloat16, device=dev) for _, nr in bands]
        tp = [[] for _ in bands]
        tf = [[] for _ in bands]
        for rep in range(reps + 1):  # the first pass warms up
            for r, ((r0, nr), layer, ext) in enumerate(zip(bands, layers, exts)):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                layer.partials(ext, r0, nr, record=records[r])
                e1.record(stream)
                if rep:
                    tp[r].append((e0, e1))
            for r, ((r0, nr), layer, ext) in enumerate(zip(bands, layers, exts)):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                layer.finish(ext, records, r0, nr, out=outs[r])
                e1.record(stream)
                if rep:
                    tf[r].append((e0, e1))
        torch.cuda.synchronize(dev)
        assert all(layer.status() == 0 for layer in layers)
        pm = [statistics.median(a.elapsed_time(b) for a, b in t) for t in tp]
        fm = [statistics.median(a.elapsed_time(b) for a, b in t) for t in tf]
        band_ms = max(pm) + max(fm)
        out[str(world)] = {"partials_ms": pm, "finish_ms": fm, "rank_compute_ms": band_ms,
                           "compute_only_efficiency": full_ms / (world * band_ms)}
        del layers, exts, records, outs
    out["note"] = ("one GPU, bands one after another, L2 flushed before each band; halo exchange and record "
                   "all-gather not included (one GPU per call)")
    return out


def sustained_run(layer, x, out, flush, stream, dev, gpu_id, ms_hint, seconds=2.5):
    """The same step back to back for about `seconds` of device time (the
    regime of a long job under the power cap): L2 flushed between steps
    outside the per-step events, clocks sampled during the loop."""
    import torch
    n = max(100, int(seconds * 1e3 / max(ms_hint, 1e-3)))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        layer.forward(x, out)
        b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = [a.elapsed_time(b) for a, b in evs]
    return n, sum(ms), statistics.median(ms), clocks


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    from linear_compressed_attention_b200 import binding as bd

    world, rank, local = dist_setup()
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    N = H * W
    qkv, proj = args.qkv, args.proj
    is_variant = qkv != ("cf", "sc", "sc") or proj
    d = make_inputs(**rank_config(cfg, rank), variant_weights=is_variant)
    layer = bd.EditAttention(d, B, H, W, C, heads, cfg["dtype"], device=dev,
                             variant=qkv if is_variant else None, out_proj=proj)
    x = torch.from_numpy(d["x"]).to(dev, layer.tdtype)
    out = torch.empty_like(x)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    nst = bd.STAGE_EVENTS_EDIT + (1 if proj else 0)
    def new_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nst)]
        for e in evs:
            e.record(stream)      # materialise the handle
        return evs

    for _ in range(args.warmup):
        layer.forward(x, out)
    torch.cuda.synchronize(dev)
    assert layer.status() == 0, "device-side status after warm-up"

    # Stage events serialise the programmatic overlap of consecutive kernels at
    # each boundary, so only every STAGE_EVERY-th timed step records them (its
    # time counts in the total like any other step).
    STAGE_EVERY = 10
    staged = [s for s in range(args.steps) if s % STAGE_EVERY == STAGE_EVERY - 1] or [args.steps - 1]
    per_step_events = {s: new_events() for s in staged}
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    gpu_id = local
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = bd.edit_attn_kernel_launches()
    for s in range(args.steps):
        flush.zero_()                                    # L2 flush, outside the step's events
        evs = per_step_events.get(s)
        if evs is not None:
            bd.edit_attn_set_stage_events([e.cuda_event for e in evs])
        step_ev[s][0].record(stream)
        layer.forward(x, out)
        step_ev[s][1].record(stream)
        if evs is not None:
            bd.edit_attn_set_stage_events(None)
    torch.cuda.synchronize(dev)
    launches = bd.edit_attn_kernel_launches() - launches0
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    assert layer.status() == 0, "device-side status after timing"

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    # without a ConvFusion query the folding, conv and GroupNorm events are not
    # recorded: those stages merge into the query GEMM's
    names = STAGES + (["out_linear"] if proj else [])
    bounds = [0] + [i + 1 for i, n in enumerate(names)
                    if not (qkv[0] == "none" and n in ("fold_weights", "conv3x3", "groupnorm"))]
    stage_ms = {names[j - 1]: [evs[i].elapsed_time(evs[j]) for evs in per_step_events.values()]
                for i, j in zip(bounds[:-1], bounds[1:])}
    total_ms = reduce_max(sum(step_ms), world, dev)
    value = job_tokens_per_s(world, B, N, args.steps, total_ms)

    # e2e: pinned host input -> device -> layer -> pinned host output, every
    # step. Three streams pipeline consecutive steps: the copy in of step k+1
    # and the copy out of step k-1 run while the layer computes step k
    # (double-buffered device input/output and host output; events order each
    # buffer's reuse).
    xh = torch.from_numpy(d["x"]).to(layer.tdtype).pin_memory()
    ohs = [torch.empty(xh.shape, dtype=layer.tdtype).pin_memory() for _ in range(2)]
    xs, outs = [x, torch.empty_like(x)], [out, torch.empty_like(out)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_run(nsteps, e0=None, e1=None):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        if e0 is not None:
            e0.record(s_in)
        for k in range(nsteps):
            j = k % 2
            if k >= 2:
                s_in.wait_event(ev_cmp[j])        # the layer of step k-2 has read xs[j]
            with torch.cuda.stream(s_in):
                xs[j].copy_(xh, non_blocking=True)
            ev_in[j].record(s_in)
            s_cmp.wait_event(ev_in[j])
            if k >= 2:
                s_cmp.wait_event(ev_out[j])       # the copy out of step k-2 has read outs[j]
            layer.forward(xs[j], outs[j], stream=s_cmp)
            ev_cmp[j].record(s_cmp)
            s_out.wait_event(ev_cmp[j])
            with torch.cuda.stream(s_out):
                ohs[j].copy_(outs[j], non_blocking=True)
            ev_out[j].record(s_out)
        if e1 is not None:
            e1.record(s_out)                      # after the last copy out, which follows everything

    e2e_run(2)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), world, dev)
    e2e_value = job_tokens_per_s(world, B, N, e2e_steps, e2e_ms)
    nbytes = xh.numel() * xh.element_size()

    if rank == 0:
        peaks = load_peaks()
        fl = layer_flops(cfg)
        # dominant kernel: the 3x3 conv of the ConvFusion query, else the K|V GEMM
        dominant, dom_kernel, dom_flops = (
            (DOMINANT, ("tc_conv_pair_kernel" if cfg["W"] >= 128 else "tc_gemm_pair_kernel (per-tap)")
             + " conv3x3 implicit GEMM", fl["conv3x3"]) if qkv[0] == "cf" else
            ("kv_linear", "tc_linear_ring_kernel K|V Linear", fl["kv_linear"]))
        dom_ms = statistics.mean(stage_ms[dominant])
        achieved = dom_flops / (dom_ms / 1e3) / 1e12
        traffic = (TRAFFIC["bytes_per_launch"] if TRAFFIC["src_sha"] == kernel_src_sha() and not is_variant
                   and args.workload == "px4096" and not args.lib else None)
        ms_per_step = total_ms / args.steps
        vflops = variant_flops(cfg, qkv, proj)
        vbytes = min_bytes(cfg) + (2 * C * C * 2 if proj else 0)
        roof_t = max(vflops / (peaks["bf16_tflops"] * 1e12), vbytes / (peaks["hbm_gbs"] * 1e9))
        line = {
            "metric": args.metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if cfg["dtype"] == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": args.workload_desc, "global_batch": world * B, "seq_len": N,
                       "parallelism": f"independent images, {world} rank(s)",
                       "l2": "flushed between steps (256 MB write, outside the timed events); input "
                             f"{B * N * cfg['C'] * 2 / 1e6:.0f} MB", **({"lib": args.lib} if args.lib else {})},
            "roofline": {"bound": "tensor", "kernel": dom_kernel, "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                         "frac_datasheet": achieved / DATASHEET["bf16_tflops"],
                         "peak_source": f"{peaks['source']} bf16 burst", "launch_ms": dom_ms},
            "layer_roofline": {"ms": roof_t * 1e3, "frac": roof_t * 1e3 / ms_per_step,
                               "frac_datasheet": max(vflops / (DATASHEET["bf16_tflops"] * 1e12),
                                                     vbytes / (DATASHEET["hbm_gbs"] * 1e9)) * 1e3 / ms_per_step,
                               "peaks": f"frac: {peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s and HBM "
                                        f"{peaks['hbm_gbs']} GB/s; frac_datasheet: {DATASHEET['bf16_tflops']} TFLOP/s "
                                        f"dense bf16 and {DATASHEET['hbm_gbs']} GB/s",
                               "note": "max(layer FLOPs / bf16 peak, minimum bytes / HBM) over measured step time"},
            "stages_ms": {k: statistics.mean(v) for k, v in stage_ms.items()},
            "stage_sampled_steps": len(per_step_events),
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
                    "d2h_bytes_per_step": nbytes},
            "gpu_launches": launches,
        }
        # side lines on one rank only (the others would wait at the final barrier)
        if world == 1 and not args.no_side:
            n_s, tot_s, med_s, clk_s = sustained_run(layer, x, out, flush, stream, dev, gpu_id, ms_per_step)
            roof_b = max(vflops / (peaks["bf16_tflops"] * 1e12), vbytes / (peaks["hbm_gbs"] * 1e9))
            sus = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
            roof_s = max(vflops / (sus * 1e12), vbytes / (peaks["hbm_gbs"] * 1e9))
            line["sustained"] = {
                "steps": n_s, "timed_s": tot_s / 1e3, "ms_per_step": tot_s / n_s, "median_ms": med_s,
                "tokens_per_s": B * N * n_s / (tot_s / 1e3),
                "layer_roofline_frac": roof_b * 1e3 / (tot_s / n_s),
                "layer_roofline_frac_sustained_peak": roof_s * 1e3 / (tot_s / n_s),
                "clocks": clk_s,
                "note": "the timed step back to back for >= 2 s (L2 flushed between steps); the headline value "
                        "above is the short loop of --steps steps"}
        if world == 1 and args.workload == "px4096" and args.variant == "cf-sc-sc" and not args.no_side:
            line["other_sizes"] = side_measurements(dev, peaks)
        if world == 1 and not args.no_cpu_baseline and args.variant == "cf-sc-sc":
            line["cpu_baseline"] = cpu_baseline(cfg)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="px4096", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true", help="skip the side measurements (other sizes, variants, MM-EDiT)")
    ap.add_argument("--lib", default=None,
                    help="time this build of the library instead of the in-tree one (e.g. an older commit's, "
                         "for a same-box A/B); the line then records it under config.lib")
    ap.add_argument("--variant", default="cf-sc-sc",
                    help="query-key-value processing of the timed layer, each cf | sc | none (ablation table), "
                         "optionally +out_linear; default the EDiT layer cf-sc-sc")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.lib:
        if not os.path.exists(args.lib):
            raise SystemExit(f"--lib {args.lib}: no such file")
        from linear_compressed_attention_b200 import binding as bd
        bd.LIB_PATH = os.path.abspath(args.lib)
    cfg = dict(WORKLOADS[args.workload])
    if cfg.get("n_txt"):
        raise SystemExit("bench.py times the EDiT layer workloads; MM-EDiT is covered by the tests")
    args.metric = "EDiT attention-layer tokens/sec (bf16, B=1) at 4K/16K/64K tokens; % roofline"
    args.proj = args.variant.endswith("+out_linear")
    args.qkv = tuple(args.variant.replace("+out_linear", "").split("-"))
    if len(args.qkv) != 3 or any(v not in ("cf", "sc", "none") for v in args.qkv):
        raise SystemExit(f"--variant {args.variant}: expected q-k-v with each cf | sc | none")
    M = ((cfg["H"] + 1) // 2) * ((cfg["W"] + 1) // 2)
    args.workload_desc = (f"{args.workload}: EDiT layer"
                          + ("" if args.variant == "cf-sc-sc" else f" (Q/K/V processing {args.variant})")
                          + f", B={cfg['B']}, {cfg['H']}x{cfg['W']} grid "
                          f"(N={cfg['H'] * cfg['W']}, M={M}), C={cfg['C']}, c_red={cfg['c_red']}, "
                          f"{cfg['heads']} heads x {cfg['C'] // cfg['heads']}, GN {cfg['gn_groups']} groups, "
                          f"{cfg['dtype']}" + (", 5% outlier tokens x8" if cfg["outliers"] else ""))
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
