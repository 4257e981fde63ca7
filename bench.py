#!/usr/bin/env python3
"""Throughput of the layer-streamed NF4 + LoRA training step (libsoup) on B200.

Default workload: Llama-3.1-8B-shaped SFT step, batch 1 x seq 512, random-init weights
N(0, 0.02) quantised to NF4 (blocksize 64, double-quantised absmax groups of 256) and held
in page-locked host RAM, streamed one decoder layer at a time into 2 device buffers; LoRA
r=64, alpha=16 on all 7 projections; AdamW on the LoRA parameters.  One "step" = embedding,
streamed forward, lm_head + cross-entropy, streamed backward, LoRA grads, AdamW, loss read
back to the host.  Every step streams ~7 GB from host memory, far more than the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl soup|reference]

N > 1 (launched with torch.distributed.run): data-parallel replicas, each rank streams its
own copy of the base and runs its own batch; LoRA gradients are summed with one NCCL
all-reduce per step before AdamW (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "train tokens/s per step (8B-shape NF4+LoRA, streamed), % of roofline, 1 B200"
PAGES_TOK_S = 119.6  # the pages' own number: RTX 3050 Laptop 4 GB, 8B, b1, s512, streamed

WORKLOADS = {
    "llama8b-sft-b1-s512": dict(cfg=synth.L8B, B=1, S=512, loss="sft"),
    "llama8b-sft-b4-s512-zipf-masked": dict(cfg=synth.L8B_B4, B=4, S=512, loss="sft", zipf=True, mask=True),
    "llama8b-dpo-2pairs-s512": dict(cfg=synth.L8B_DPO, B=4, S=512, loss="dpo", n_pairs=2, prefix_len=256,
                                    beta=0.1),
    # same DPO step, each layer loaded once for the reference and the policy forward
    "llama8b-dpo-2pairs-s512-shared-load": dict(cfg=synth.L8B_DPO, B=4, S=512, loss="dpo", n_pairs=2,
                                                prefix_len=256, beta=0.1, dpo_shared_load=True),
    # one load per layer and each pair's 256-token prefix run once: 1536 rows through the layers
    "llama8b-dpo-2pairs-s512-shared-prefix": dict(cfg=synth.L8B_DPO, B=4, S=512, loss="dpo", n_pairs=2,
                                                  prefix_len=256, beta=0.1, dpo_shared_load=True, share_prefix=True),
    # the other preference losses on the same batch shape (KTO: 4 unpaired rows, 2 desirable)
    "llama8b-kto-4seq-s512": dict(cfg=synth.L8B_DPO, B=4, S=512, loss="kto", n_pairs=2, prefix_len=256, beta=0.1,
                                  labels=(1, 0, 1, 0)),
    "llama8b-simpo-2pairs-s512": dict(cfg=synth.L8B_DPO, B=4, S=512, loss="simpo", n_pairs=2, prefix_len=256,
                                      beta=2.0, gamma=0.5),
    "llama8b-orpo-2pairs-s512": dict(cfg=synth.L8B_DPO, B=4, S=512, loss="orpo", n_pairs=2, prefix_len=256,
                                     lambda_or=0.1),
    # the same SFT step with the layer stack in a file (stream_source = file), read through
    # page-locked staging slots
    "llama8b-sft-b1-s512-file": dict(cfg=synth.L8B, B=1, S=512, loss="sft", source="file"),
    "llama70b-sft-b1-s2048": dict(cfg=synth.L70B, B=1, S=2048, loss="sft"),
    "tiny-sft-b1-s64": dict(cfg=synth.TINY, B=1, S=64, loss="sft"),
}
DEFAULT = "llama8b-sft-b1-s512"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def measured_traffic(kernel, token_rows):
    """DRAM bytes per launch of a kernel category from an ncu capture summarised under
    profiles/, or None when the kernel's sources changed since the capture or the capture's
    launch shape (token rows) is not the workload's."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic_per_launch.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel)
    if not rec or rec.get("token_rows") != token_rows:
        return None
    h = hashlib.sha256()
    for f in rec["kernel_sources"]:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return rec["dram_bytes_per_launch"] if h.hexdigest() == rec["kernel_sources_sha256"] else None


# one kernel, two launch kinds each: the NF4 GEMM (forward x W^T and dX through the same codes
# read transposed) and the LoRA GEMMs (u, v on the main stream; dA, dB beside them)
KERNEL_GROUPS = {"gemm_nf4_fwd,gemm_nf4_dx": ("gemm_nf4_fwd", "gemm_nf4_dx"),
                 "gemm_lora,gemm_lora_grad": ("gemm_lora", "gemm_lora_grad")}


def rank_kernels(prof):
    """Names the dominant kernel of a live profile (dict category -> launches, total_ms, ...).
    The pass's own cost per launch (the empty launches of "event_overhead", bracketed like the
    others) is taken off each category first (net_ms): otherwise categories of many short
    launches look longer than they run.  Layer copies are not kernels.  Returns (kernel
    categories, groups, dominant group name, overhead ms per launch); mutates prof."""
    ov = prof.pop("event_overhead", None)
    ov_ms = ov["total_ms"] / ov["launches"] if ov and ov["launches"] else 0.0
    for v in prof.values():
        v["net_ms"] = max(v["total_ms"] - v["launches"] * ov_ms, 0.0)
    kern = {k: v for k, v in prof.items() if k != "h2d_layer_copy"}
    grouped = {k: (k,) for k in kern if not any(k in g for g in KERNEL_GROUPS.values())}
    grouped.update({name: tuple(c for c in g if c in kern) for name, g in KERNEL_GROUPS.items()})
    grouped = {k: g for k, g in grouped.items() if g}
    net = {k: sum(kern[c]["net_ms"] for c in g) for k, g in grouped.items()}
    dom = max(net, key=net.get) if net else None
    return kern, grouped, dom, ov_ms


def config_of(workload, wl, world):
    """The workload's config dict, the same in both arms."""
    return {"workload": workload, "model": wl["cfg"]["name"], "global_batch": world * wl["B"], "seq_len": wl["S"],
            "parallelism": f"dp{world}", "layer_buffers": 2, "lora_r": wl["cfg"]["lora_r"],
            "l2": "inputs larger than L2: the NF4 layer stack (GBs) is streamed from host memory every step"}


def step_flops(cfg, B, S, loss):
    """Algorithmic FLOPs of one step (no recompute counted)."""
    h, I, V, L = cfg["hidden"], cfg["intermediate"], cfg["vocab"], cfg["n_layers"]
    hq, hkv, d, r = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["lora_r"]
    T = B * S
    p_layer = h * hq * d + 2 * h * hkv * d + hq * d * h + 3 * h * I
    io = (h + hq * d) + 2 * (h + hkv * d) + (hq * d + h) + 2 * (h + I) + (I + h)
    train = L * (4 * p_layer + 6 * r * io + 6 * S * d * hq) * T + 4 * h * V * T
    if loss in ("dpo", "kto"):  # plus the LoRA-off reference forward
        train += L * (2 * p_layer + 2 * S * d * hq) * T + 2 * h * V * T
    return float(train)


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------- soup arm
def build_model(wl, device_index, seed, mode="streamed"):
    import torch
    from layer_streamed_nf4_lut_b200.model import SoupModel, lora_offset
    cfg = dict(wl["cfg"])
    B, S = wl["B"], wl["S"]
    dev = torch.device("cuda", device_index)
    source = wl.get("source", "ram") if mode == "streamed" else "ram"
    path = None
    if source == "file":
        import tempfile
        import atexit
        import shutil
        d = tempfile.mkdtemp(prefix="soup_stack_", dir=os.environ.get("SOUP_STACK_DIR"))
        atexit.register(shutil.rmtree, d, True)
        path = os.path.join(d, "stack.soup")
    gm = SoupModel(cfg, mode=mode, n_layer_buffers=2, max_tokens=B * S, device=device_index, source=source,
                   stack_path=path)
    gm.stack_path = path
    ones = torch.ones(cfg["hidden"], dtype=torch.bfloat16, device=dev)
    for i in range(cfg["n_layers"]):
        w = {}
        for j, p in enumerate(synth.PROJ_NAMES):
            w[p] = synth.normal_device(synth.proj_shape(cfg, p), seed * 100003 + 16 * i + j, 0.02, device=dev)
        gm.quantize_layer(i, w, ones, ones)
        del w
    V, h = cfg["vocab"], cfg["hidden"]
    embed = synth.normal_device((V, h), seed * 7 + 1, 0.02, device=dev).to(torch.bfloat16)
    lm = synth.normal_device((V, h), seed * 7 + 2, 0.02, device=dev).to(torch.bfloat16)
    gm.set_head(embed, ones.clone(), lm)
    params = torch.empty(gm.lora_n, dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(seed * 11 + 3)
    for layer in range(cfg["n_layers"]):
        for j, p in enumerate(synth.PROJ_NAMES):
            oa, ra, ca = lora_offset(cfg, layer, j, 0)
            ob, rb, cb = lora_offset(cfg, layer, j, 1)
            params[oa:oa + ra * ca].uniform_(-1.0 / math.sqrt(ca), 1.0 / math.sqrt(ca), generator=g)
            params[ob:ob + rb * cb].normal_(0.0, 0.01, generator=g)
    gm.set_lora(params)
    torch.cuda.synchronize(dev)
    return gm


def make_batch(wl, seed):
    cfg = dict(wl["cfg"], batch=wl["B"], seq=wl["S"])
    if wl["loss"] != "sft":
        ids = synth.preference_batch(dict(cfg, n_pairs=wl["n_pairs"], prefix_len=wl["prefix_len"]), seed)
        return ids, None
    ids = synth.token_batch(cfg, seed, zipf=wl.get("zipf", False))
    mask = synth.last_half_mask(wl["B"], wl["S"]) if wl.get("mask") else None
    return ids, mask


def run_soup(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from layer_streamed_nf4_lut_b200 import dp
    from layer_streamed_nf4_lut_b200.model import SoupModel  # noqa: F401  (fails loudly without libsoup.so)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = wl["cfg"]
    B, S, T = wl["B"], wl["S"], wl["B"] * wl["S"]
    t_setup = time.time()
    gm = build_model(wl, local_rank, seed=1234)
    ids_np, mask_np = make_batch(wl, seed=77 + rank)
    ids = torch.from_numpy(ids_np).to(dev)
    mask = torch.from_numpy(mask_np).to(dev) if mask_np is not None else None
    kw = dict(loss=wl["loss"], mask=mask, n_pairs=wl.get("n_pairs", 0), prefix_len=wl.get("prefix_len", 0),
              beta=wl.get("beta", 0.1), lr=2e-5, dpo_shared_load=wl.get("dpo_shared_load", False),
              share_prefix=wl.get("share_prefix", False),
              gamma=wl.get("gamma", 0.0), lambda_or=wl.get("lambda_or", 0.1),
              labels=np.array(wl["labels"], np.uint8) if "labels" in wl else None)
    setup_s = time.time() - t_setup

    labels_np = kw.pop("labels")
    labels_dev = torch.from_numpy(labels_np).to(dev) if labels_np is not None else None

    def one_step(ids_arg, mask_arg):
        # labels (KTO) live where the ids live
        lab = labels_dev if (isinstance(ids_arg, torch.Tensor) and ids_arg.is_cuda) else labels_np
        if world == 1:
            return gm.step(ids_arg, **dict(kw, mask=mask_arg, labels=lab), apply_optimizer=True)
        loss, _ = dp.dp_step(lambda: gm.step(ids_arg, **dict(kw, mask=mask_arg, labels=lab), apply_optimizer=False),
                             gm.lora_grads, lambda: gm.optimizer_step(2e-5))
        return loss

    h2d_gbs = gm.h2d_probe(20)
    for _ in range(args.warmup):
        loss = one_step(ids, mask)
    torch.cuda.synchronize(dev)

    if world > 1:
        dist.barrier()
    gm.reset_stats()
    torch.cuda.reset_peak_memory_stats(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            loss = one_step(ids, mask)
        e1.record(stream)
        e1.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    st = gm.stats()
    # device memory: every library allocation goes through torch's caching allocator, so the
    # peak over the timed steps covers the model (layer buffers, activations, scratch) and the
    # caller's tensors (head weights, LoRA parameters / gradients / moments, ids)
    peak_alloc = torch.cuda.max_memory_allocated(dev)
    peak_reserved = torch.cuda.max_memory_reserved(dev)
    if world > 1:
        ms = dp.max_over_ranks(ms, device=dev)
    ms_step = ms / args.steps
    tok_s = world * T * args.steps / (ms * 1e-3)
    loads_per_step = st["layer_loads"] / args.steps
    launches = st["kernel_launches"]
    file_gbs = (st["file_bytes_read"] / (st["file_read_ms"] * 1e-3) / 1e9) if st.get("file_read_ms") else None

    # Kernel times, measured after the timed steps (which carry no events: event-record nodes in
    # the graphs cost a few percent of a compute-bound step).  First an eager pass with the
    # LoRA weight-gradient side stream folded into the main stream (serialised like a profiler's
    # launch list): an event pair around every launch and layer copy gives the per-category
    # breakdown and names the dominant kernel.  Then steps run like the timed ones (graph
    # replay, side stream on) with event pairs around the dominant kernel's launches only
    # (event-record nodes of the replayed layer graphs, on the stream each launch runs on); two
    # untimed steps capture those graphs first.
    n_prof = max(1, min(args.steps, 3))
    gm.set_profiling(True)
    gm.profile(reset=True)
    for _ in range(n_prof):
        one_step(ids, mask)
    prof = gm.profile(reset=True)
    gm.set_profiling(False)
    kern, grouped, dom, ov_ms = rank_kernels(prof)
    timed = {"launches": 0}
    if dom:
        gm.set_timed_category(dom)
        for _ in range(2):
            one_step(ids, mask)
        gm.timed_category(reset=True)
        for _ in range(n_prof):
            one_step(ids, mask)
        tprof = gm.timed_profile()
        timed = gm.timed_category(reset=True)
        tov = tprof.get("event_overhead")
        timed["overhead_ms"] = tov["total_ms"] / tov["launches"] if tov and tov["launches"] else 0.0
        dom_eager = {f: sum(kern[c][f] for c in grouped[dom]) for f in ("launches", "total_ms", "flops", "bytes")}
    gm.set_timed_category(None)

    # end-to-end through the public API with host buffers: ids copied H2D inside each step,
    # loss read back to the host by each step
    ids_host = torch.from_numpy(ids_np).pin_memory()
    mask_host = torch.from_numpy(mask_np).pin_memory() if mask_np is not None else None
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step(ids_host, mask_host)
    torch.cuda.synchronize(dev)
    e2e_s = time.perf_counter() - t0
    if world > 1:
        e2e_s = dp.max_over_ranks(e2e_s, device=dev)
    e2e_tok_s = world * T * args.steps / e2e_s

    # compute-only reference (one GPU): the same step with every layer resident, no streaming;
    # tells apart the kernels' time from the streaming / overlap losses
    compute_ms = None
    if world == 1 and not args.no_compute_only:
        gm.close()
        del gm
        torch.cuda.empty_cache()
        gr = build_model(wl, local_rank, seed=1234, mode="resident")
        for _ in range(2):
            gr.step(ids, **kw, labels=labels_dev, apply_optimizer=True)
        torch.cuda.synchronize(dev)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            gr.step(ids, **kw, labels=labels_dev, apply_optimizer=True)
        c1.record(stream)
        c1.synchronize()
        compute_ms = c0.elapsed_time(c1) / args.steps
        blob_bytes = gr.blob_bytes
        gr.close()
    else:
        blob_bytes = gm.blob_bytes

    if rank != 0:
        return None
    pk = peaks()
    if wl.get("share_prefix"):  # each pair runs as one block of 2S - prefix rows
        flops = step_flops(cfg, wl["n_pairs"], 2 * S - wl["prefix_len"], wl["loss"])
    else:
        flops = step_flops(cfg, B, S, wl["loss"])
    stream_bytes = loads_per_step * blob_bytes
    t_flops = flops / (pk["bf16_sustained"] * 1e12)
    t_h2d = stream_bytes / (h2d_gbs * 1e9)
    t_roof = max(t_flops, t_h2d)
    roof_tok_s = T / t_roof
    # dominant kernel: achieved work per launch over its launches in the timed steps
    roofline = None
    if dom:
        in_timed = timed["launches"] > 0
        d = timed if in_timed else dom_eager
        per_launch_ms = d["total_ms"] / d["launches"]
        # the same launches with the event pairs' own cost (empty launches timed alike) taken off
        net_launch_ms = per_launch_ms - (timed.get("overhead_ms", 0.0) if in_timed else ov_ms)
        ridge = pk["bf16_sustained"] * 1e12 / (pk["hbm_gbs"] * 1e9)  # flop / byte
        if d["flops"] > 0 and d["flops"] / max(d["bytes"], 1.0) >= ridge:
            achieved = d["flops"] / d["launches"] / (per_launch_ms * 1e-3) / 1e12
            roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 2),
                        "peak": pk["bf16_sustained"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_sustained"], 4),
                        "peak_source": pk["source"] + " bf16 sustained", "traffic": measured_traffic(dom, T),
                        "algorithmic_bytes_per_launch": round(d["bytes"] / d["launches"]),
                        "avg_launch_ms": round(per_launch_ms, 4), "launches": d["launches"]}
        else:
            achieved = d["bytes"] / d["launches"] / (per_launch_ms * 1e-3) / 1e9
            roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4), "peak_source": pk["source"],
                        "traffic": measured_traffic(dom, T), "avg_launch_ms": round(per_launch_ms, 4), "launches": d["launches"]}
        net_ach = (d["flops"] / d["launches"] / (net_launch_ms * 1e-3) / 1e12 if roofline["unit"] == "TFLOP/s" else
                   d["bytes"] / d["launches"] / (net_launch_ms * 1e-3) / 1e9) if net_launch_ms > 0 else None
        roofline["event_overhead_ms"] = round(per_launch_ms - net_launch_ms, 4)
        roofline["achieved_net_of_event_overhead"] = round(net_ach, 2) if net_ach else None
        roofline["timing"] = ("CUDA event pair around each of its launches (event-record nodes of the replayed "
                              "layer graphs, on the launching stream) over %d steps run like the timed ones, right "
                              "after them" % n_prof if in_timed else "CUDA event pairs of the eager profiled pass")
    h2d = prof.get("h2d_layer_copy")
    profile_summary = {k: {"launches": v["launches"] // n_prof, "ms_per_step": round(v["total_ms"] / n_prof, 3),
                           "net_ms_per_step": round(v["net_ms"] / n_prof, 3),
                           "tflops": round(v["flops"] / (v["total_ms"] * 1e-3) / 1e12, 1) if v["flops"] else None,
                           "gbs": round(v["bytes"] / (v["total_ms"] * 1e-3) / 1e9, 1)}
                       for k, v in sorted(prof.items(), key=lambda kv: -kv[1]["net_ms"])}
    ids_bytes = T * 4 + (T if mask_np is not None else 0) + (B if labels_np is not None else 0)
    out = {
        "metric": METRIC, "value": round(tok_s, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": round(tok_s / PAGES_TOK_S, 2) if args.workload == DEFAULT else None,
        "dtype": "bf16", "data": "synthetic (seeded random-init weights and token ids)",
        "config": config_of(args.workload, wl, world),
        "pct_of_roofline": round(100.0 * tok_s / world / roof_tok_s, 2),
        "roofline_step": {"bound": "h2d" if t_h2d >= t_flops else "tensor", "tok_s": round(roof_tok_s, 1),
                          "frac": round(tok_s / world / roof_tok_s, 4), "h2d_gbs_measured": round(h2d_gbs, 2),
                          "stream_bytes_per_step": int(stream_bytes), "layer_loads_per_step": loads_per_step,
                          "flops_per_step": flops, "bf16_peak_tflops": pk["bf16_sustained"],
                          "achieved_h2d_gbs_in_step": round(h2d["bytes"] / (h2d["total_ms"] * 1e-3) / 1e9, 2) if h2d else None,
                          "stream_source": "file" if st.get("stream_source") == 1 else "ram",
                          "file_read_gbs_in_step": round(file_gbs, 2) if file_gbs else None},
        "compute_only_ms_per_step": round(compute_ms, 3) if compute_ms else None,
        "device_memory": {"peak_allocated_bytes": int(peak_alloc), "peak_reserved_bytes": int(peak_reserved),
                          "model_device_bytes": int(st["device_bytes"]),
                          "pinned_host_bytes": int(st["pinned_bytes"]),
                          "note": "peak of torch.cuda.max_memory_allocated over the timed steps (the library "
                                  "allocates through torch's caching allocator); the pages report 3.32 GB peak "
                                  "VRAM for the streamed 8B SFT step and 0.914x that for DPO on a 4 GB laptop GPU"},
        "roofline": roofline,
        "profile": profile_summary,
        "profile_note": "per step, over %d untimed eager steps with every launch on one stream (serialised) and "
                        "an event pair around each launch and layer copy, each launch preceded by a short busy-wait "
                        "kernel so that the pair does not time the host's submission; net_ms takes off the pair's "
                        "own cost per launch, measured on empty launches (event_overhead_us)" % n_prof,
        "event_overhead_us": round(ov_ms * 1e3, 2),
        "e2e": {"value": round(e2e_tok_s, 2), "unit": "tokens/s", "h2d_bytes_per_step": int(ids_bytes + stream_bytes),
                "h2d_input_bytes_per_step": ids_bytes, "d2h_bytes_per_step": 8},
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "final_loss": loss,
        "setup_s": round(setup_s, 1),
    }
    return out


# ---------------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(wl, seed=5):
    """Time the CPU oracle on a bounded sample of the workload: one decoder layer forward +
    backward at the workload's shape, plus (once) the head; extrapolated to a whole step."""
    from oracle import model as om
    cfg = dict(wl["cfg"])
    B, S, T = wl["B"], wl["S"], wl["B"] * wl["S"]
    rng = np.random.default_rng(seed)
    W = {}
    for p in synth.PROJ_NAMES:
        W[p] = rng.standard_normal(synth.proj_shape(cfg, p)) * 0.02
    W["attn_norm"] = np.ones(cfg["hidden"])
    W["mlp_norm"] = np.ones(cfg["hidden"])
    lo = {}
    for p in synth.PROJ_NAMES:
        o, i = synth.proj_shape(cfg, p)
        lo[p] = (rng.uniform(-1, 1, (cfg["lora_r"], i)) / math.sqrt(i), rng.standard_normal((o, cfg["lora_r"])) * 0.01)
    x = rng.standard_normal((T, cfg["hidden"]))
    dy = rng.standard_normal((T, cfg["hidden"])) * 1e-3

    def layer_once():
        t0 = time.perf_counter()
        y, cache = om.layer_forward(cfg, W, lo, x, B, S)
        om.layer_backward(cfg, W, lo, cache, dy, B, S)
        return time.perf_counter() - t0

    def head_once():
        head = dict(embed=None, lm_head=rng.standard_normal((cfg["vocab"], cfg["hidden"])) * 0.02,
                    final_norm=np.ones(cfg["hidden"]))
        ids = rng.integers(0, cfg["vocab"], (B, S))
        t0 = time.perf_counter()
        logits, hc = om.head_forward(cfg, head, x)
        loss, dl = om.sft_loss(logits, ids)
        om.head_backward(head, hc, dl)
        return time.perf_counter() - t0

    return layer_once, head_once


def threads_used():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, budget_layers=1):
    layer_once, head_once = oracle_sample(wl)
    t_layer = min(layer_once() for _ in range(budget_layers))
    t_head = head_once()
    L = wl["cfg"]["n_layers"]
    mult = 1.5 if wl["loss"] in ("dpo", "kto") else 1.0  # the reference adds a forward-only pass (~1/3 of fwd+bwd)
    t_step = L * t_layer * mult + t_head
    T = wl["B"] * wl["S"]
    return {"value": round(T / t_step, 4), "unit": "tokens/s", "cores": threads_used(), "host_cpus": os.cpu_count(),
            "kind": "oracle",
            "sample": f"one decoder layer fwd+bwd ({t_layer:.2f} s) + head fwd+bwd ({t_head:.2f} s) at the "
                      f"workload shape, float64 numpy oracle; step extrapolated as L*layer + head = {t_step:.1f} s"}


def run_reference(args, wl):
    layer_once, head_once = oracle_sample(wl)
    t_head = head_once()
    L = wl["cfg"]["n_layers"]
    mult = 1.5 if wl["loss"] in ("dpo", "kto") else 1.0
    for _ in range(args.warmup):
        layer_once()
    times = [layer_once() for _ in range(args.steps)]
    t_step = L * float(np.mean(times)) * mult + t_head
    T = wl["B"] * wl["S"]
    v = T / t_step
    # each timed step is a bounded sample (one decoder layer forward + backward at the workload
    # shape): ms_per_step is what a timed step took; the whole training step it stands for is
    # extrapolated (ms_per_step_extrapolated) and gives `value`
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(float(np.mean(times)) * 1e3, 1),
            "ms_per_step_extrapolated": round(t_step * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(args.workload, wl, 1),
            "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": threads_used(), "kind": "oracle",
                             "sample": "per step: one decoder layer fwd+bwd at the workload shape (float64 numpy "
                                       "oracle); head timed once; step = L*layer + head"},
            "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="soup", choices=["soup", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-compute-only", action="store_true", help="skip the resident (no streaming) timing")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    out = run_soup(args, wl, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
