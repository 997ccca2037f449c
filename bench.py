#!/usr/bin/env python
"""Benchmark: single-token decode attention over the mixed-format paged KV
cache (BF16/FP8 sink and window pages, 2-bit ternary older pages), on
synthetic data shaped like the workload, through libkvc's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-configs] [--no-e2e]

Prints ONE JSON line (rank 0).  A step is one decode-attention pass over the
batch's compressed cache (every layer of the stack in one launch); `value`
is its HBM throughput: the algorithmic bytes the pass must move (packed
codes + gamma, FP8 bytes + scales, BF16 pages, Q, block table, lengths,
output) divided by device time.  The cache is packed once before timing;
the pack kernels, the other cache kernels and every other workload
(`configs`) are measured in the same run and reported beside the step.
`--impl reference` times the CPU oracle on the host's cores instead.  For
N > 1 (torchrun) every rank decodes its own independent batch (weak
scaling, no collective on the data path).
"""

from __future__ import annotations

import os

os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")   # one oracle worker = one core
os.environ.setdefault("OMP_NUM_THREADS", "1")
os.environ.setdefault("MKL_NUM_THREADS", "1")

import argparse
import hashlib
import json
import math
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "decode-attention KV GB/s & % of B200 HBM peak; pack GB/s; oracle speedup"
P = 16

WORKLOAD_TEXT = {
    "tiny": "tiny decode: B=1, Hq=8, Hkv=4, D=64, L=512, sink 4, window 64 BF16, older pages ternary",
    "qwen3b": "Qwen2.5-3B-shaped layer: B=8, Hq=16, Hkv=2, D=128, L=4096, sink 4, window 256 FP8, older pages ternary, 2% outlier channels",
    "llama8b": "Llama-3-8B-shaped layer: B=32, Hq=32, Hkv=8, D=128, L=32768, sink 4, window 1024 BF16, older pages ternary, random physical page placement",
    "longctx": "long-context ragged layer: B=16, Hq=24, Hkv=4, D=256, L~U[8192,131072], sink 4, window 2048 FP8, 5% BF16 anchors, Laplace values",
    "bulk": "bulk compress + round trip: 1 GiB of bf16 KV as 32768 pages of [8 heads][16 tokens][128], N(0,1) with 1% of entries x20; ternary quantise+pack of every page, then dequantise back to bf16",
}

# the workloads measured in the `configs` block beside the step: (key,
# workload, attention layers per launch, batch, context); None keeps the
# workload's own value
CONFIG_SET = (
    ("qwen3b_36l", "qwen3b", 36, None, None),
    ("llama8b", "llama8b", 1, None, None),
    ("longctx", "longctx", 1, None, None),
    # a 32-layer stack of the Llama-3-8B-shaped layer at 4096 tokens, with
    # 1024 and 2048 (layer, sequence) entries in one launch
    ("llama8b_32l_b32_4k", "llama8b", 32, 32, 4096),
    ("llama8b_32l_b64_4k", "llama8b", 32, 64, 4096),
)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b", choices=sorted(synth.WORKLOADS) + ["bulk"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=None,
                    help="attention layers per step (default: 36 for the Qwen2.5-3B-shaped layer, "
                         "whose model has 36, else 1); all layers are decoded in one launch")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--context", type=int, default=None,
                    help="override the workload's context length (tokens)")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of replaying a captured CUDA graph")
    ap.add_argument("--decode-kernel", default=None, choices=["tc", "tcgen05"],
                    help="decode kernel: tc (default, mma.sync) or the opt-in tcgen05 kernel")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' block (bench the chosen workload alone)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the append/retier, promotion and lossless-codec timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return 6650.0, "fallback (6.65 TB/s, an earlier copy-bandwidth measurement on B200)"


# ---------------------------------------------------------------- bytes

def algorithmic_bytes(cfg, layout, B, max_pages, has_older):
    """Bytes each kernel must move for one layer of the batch, by kernel:
    a pack launch reads the bf16 pages of its pool and writes their codes
    (K and V); decode reads every page's compressed bytes once, Q, the
    block table, lengths and format tags, and writes fp32 output."""
    H, D, hq = cfg["n_kv_heads"], cfg["head_dim"], cfg["n_q_heads"]
    n_bf, n_f8, n_t = layout.pool_pages
    page_bf16 = 2 * P * H * D
    out = {
        "pack_bf16": 2 * n_bf * (2 * page_bf16),
        "pack_fp8": 2 * n_f8 * (page_bf16 + P * H * D + 4),
        "pack_ternary": 2 * n_t * (page_bf16 + P * H * D // 4 + 4 * H),
    }
    total_pages = n_bf + n_f8 + n_t
    out["decode"] = (2 * (n_bf * page_bf16 + n_f8 * (P * H * D + 4) + n_t * (P * H * D // 4 + 4 * H))
                     + B * (2 * hq * D + 4 * hq * D + 4) + 4 * total_pages
                     + (total_pages if has_older else 0))
    return out


def bulk_bytes(n, H, D, fmt="ternary"):
    """Algorithmic bytes of packing (or dequantising) n pages of H groups:
    the bf16 pages plus their codes (and gamma or the page scale)."""
    if fmt == "fp8":
        return n * (H * (2 * P * D + P * D) + 4)
    return n * H * (2 * P * D + P * D // 4 + 4)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if len(r) > 5 + i and r[5 + i].strip().lower() == "active"})
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- our arm

def max_over_ranks(value, world, dev):
    """Device time of the job: the largest of the ranks' times (every rank
    takes part in the same collective, so call it on every rank)."""
    if world <= 1:
        return value
    t = torch.tensor([float(value)], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank):
    """Each rank decodes its own independent batch (weak scaling): inputs are
    drawn with the rank as the seed."""
    return rank


# where each timed kernel's code lives: (files, kernel function, launcher);
# None = the whole files
KERNEL_SRC = {"decode": (("decode_tc.cu", "decode_common.cuh"), None, None),
              "pack_ternary": (("quant.cu",), "quant_ternary_kernel", "launch_quant_ternary"),
              "pack": (("quant.cu",), "quant_ternary_kernel", "launch_quant_ternary"),
              "dequant_ternary": (("quant.cu",), "dequant_ternary_kernel", "launch_dequant_ternary")}


def _function_text(src, name, start_at_file_head):
    """Text of the definition of `name` (to its closing brace at column 0);
    with start_at_file_head, everything before it too (the helpers it uses)."""
    i = src.find(" " + name + "(")
    if i < 0:
        return None
    j = src.find("\n}\n", i)
    if j < 0:
        return None
    start = 0 if start_at_file_head else src.rfind("\n", 0, i) + 1
    return src[start:j + 3]


def kernel_source_hash(kernel_key):
    """Hash of the code of a kernel: recorded ncu traffic stays valid only
    while that code is unchanged.  For a codec kernel that is the source
    file up to the end of the kernel (the helpers it uses come first) plus
    its launcher; for decode, its whole files."""
    spec = KERNEL_SRC.get(kernel_key)
    if spec is None:
        return None
    files, fn, launcher = spec
    text = ""
    for f in files:
        src = open(os.path.join(ROOT, "compressed_decode_attention_kvc_b200", "csrc", f)).read()
        if fn is None:
            text += src
        else:
            a = _function_text(src, fn, True)
            b = _function_text(src, launcher, False)
            if a is None or b is None:
                return None
            text += a + b
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """dram bytes per launch recorded from an ncu capture of the current
    kernel sources for this workload at its default size
    (profiles/ncu_traffic.txt), else None."""
    if workload is None:
        return None
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash(kernel_key)
    for line in open(path):
        parts = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if (parts.get("kernel") == kernel_key and parts.get("sources") == src and
                parts.get("workload") == workload and "bytes_per_launch" in parts):
            return float(parts["bytes_per_launch"])
    return None


def layers_of(args):
    """Attention layers decoded per step: the Qwen2.5-3B-shaped workload runs
    all 36 of its model's layers (one decode launch for the stack); the
    others are one layer."""
    return args.layers or (36 if args.workload == "qwen3b" else 1)


# source pages above this many bytes are drawn for one layer and packed into
# every layer's pools (each layer still has its own compressed pages and Q)
SHARED_SOURCE_BYTES = 8 << 30


class Case:
    """One decode workload on the device: synthetic bf16 K/V pages and Q,
    the planner's layout, the allocated pools (packed by `pack`), the
    workspace and output of the decode call."""

    def __init__(self, workload, dev, seed, batch=None, layers=1, context=None):
        import compressed_decode_attention_kvc_b200 as K
        from compressed_decode_attention_kvc_b200 import paged_cache as PC
        self.K, self.PC = K, PC
        over = {} if context is None else {"context": context}
        inp = synth.make_decode_inputs(workload, seed=seed, device=dev, batch=batch, **over)
        cfg = inp["cfg"]
        B, max_pages, H, _, D = inp["k_pages"].shape
        src_bytes = 2 * inp["k_pages"].numel() * 2 * layers
        self.shared_source = layers > 1 and src_bytes > SHARED_SOURCE_BYTES
        if layers > 1 and not self.shared_source:
            # further layers: their own K, V and Q, the first layer's placement
            ks, vs, qs = [inp["k_pages"]], [inp["v_pages"]], [inp["q"]]
            for l in range(1, layers):
                o = synth.make_decode_inputs(workload, seed=seed * 1000 + l, device=dev, batch=batch, **over)
                ks.append(o["k_pages"]); vs.append(o["v_pages"]); qs.append(o["q"])
                del o
            inp["k_pages"], inp["v_pages"], inp["q"] = torch.cat(ks), torch.cat(vs), torch.cat(qs)
            del ks, vs, qs
        elif self.shared_source:
            g = torch.Generator(device=dev)
            g.manual_seed(seed * 1000 + 1)
            qs = [inp["q"]] + [torch.randn(inp["q"].shape, generator=g, device=dev).to(torch.bfloat16)
                               for _ in range(1, layers)]
            inp["q"] = torch.cat(qs)
        self.workload, self.inp, self.cfg, self.layers = workload, inp, cfg, layers
        self.B, self.max_pages, self.H, self.D = B, max_pages, H, D
        self.hq = cfg["n_q_heads"]
        self.hp = K.KVC_FMT_BF16 if cfg["hp"] == "bf16" else K.KVC_FMT_FP8_E4M3
        self.older = None
        if inp["anchor"].any():
            self.older = torch.where(inp["anchor"], K.KVC_FMT_BF16, K.KVC_FMT_TERNARY2).to(torch.uint8)
        lens_h = inp["context_lens"].cpu()
        sk = None if inp["slot_key"] is None else inp["slot_key"].cpu()
        self.layout = PC.plan_paged_cache(lens_h, max_pages, cfg["sink"], cfg["window"], self.hp,
                                          older_fmt=None if self.older is None else self.older.cpu(),
                                          slot_key=sk)
        self.cache = PC.allocate_device_cache(self.layout, H, D, dev, n_layers=layers)
        src_layers = 1 if self.shared_source else layers
        self.kf = inp["k_pages"].view(src_layers * B * max_pages, H, P, D)
        self.vf = inp["v_pages"].view(src_layers * B * max_pages, H, P, D)
        if self.shared_source:
            self.cache.page_ids = [torch.cat([i.to(dev) for i in [ids] * layers])
                                   for ids in self.layout.pool_src_ids]
        self.q, self.lens = inp["q"], inp["context_lens"]
        self.ws_bytes = K.kvc_decode_workspace_size(layers * B, self.hq, H, D, max_pages)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.out = torch.empty((layers * B, self.hq, D), dtype=torch.float32, device=dev)
        self.nbytes = {k: layers * v for k, v in
                       algorithmic_bytes(cfg, self.layout, B, max_pages, self.older is not None).items()}
        self.pools = [(f, n * layers) for f, n in zip((K.KVC_FMT_BF16, K.KVC_FMT_FP8_E4M3, K.KVC_FMT_TERNARY2),
                                                        self.layout.pool_pages) if n > 0]

    PACK_NAMES = {0: "pack_bf16", 1: "pack_fp8", 2: "pack_ternary"}
    FIELDS = {0: ("k_bf16", "v_bf16", None, None), 1: ("k_fp8", "v_fp8", "k_fp8_scale", "v_fp8_scale"),
              2: ("k_tern", "v_tern", "k_gamma", "v_gamma")}

    def pack_calls(self):
        """(kernel name, call) per pool: the call packs the K and V pages of
        that pool (two launches)."""
        K, pl = self.K, self.cache.pools
        calls = []
        for f, n in self.pools:
            kn, vn, ks, vs = self.FIELDS[f]
            ids = self.cache.page_ids[f]

            def call(kn=kn, vn=vn, ks=ks, vs=vs, ids=ids, n=n, f=f):
                K.kvc_quantize_pack_pages(self.kf, ids, n, P, self.H, self.D, f, pl[kn], pl[ks] if ks else None)
                K.kvc_quantize_pack_pages(self.vf, ids, n, P, self.H, self.D, f, pl[vn], pl[vs] if vs else None)
            calls.append((self.PACK_NAMES[f], call))
        return calls

    def pack(self):
        for _, call in self.pack_calls():
            call()

    def decode(self, q=None, lens=None, out=None):
        cfg = self.cfg
        self.K.kvc_decode_attention_paged_layers(
            self.q if q is None else q, self.cache.struct, self.cache.block_table, self.older,
            self.lens if lens is None else lens, self.layers, self.B, self.hq, self.H, self.D, P,
            self.max_pages, cfg["sink"], cfg["window"], self.hp, 0.0, self.out if out is None else out,
            self.ws, self.ws_bytes)

    def check_flags(self):
        flags = self.K.kvc_decode_read_error(self.ws, self.layers * self.B, self.hq, self.H, self.D,
                                             self.max_pages)
        if flags:
            raise RuntimeError(f"{self.workload}: device error flags {flags}")

    def pages(self):
        n_bf, n_f8, n_t = (n * self.layers for n in self.layout.pool_pages)
        return {"bf16": n_bf, "fp8": n_f8, "ternary": n_t}


def graph_time(fn, reps, warmup, stream, eager=False):
    """Average device time (ms) of one call of fn: `reps` back-to-back
    replays of a CUDA graph of one call (eager calls with eager=True)
    between two events on the launching stream, after `warmup` calls."""
    g = None
    if not eager:
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
    run = g.replay if g is not None else fn
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del g
    return ms


def kernel_entry(ms, nbytes, peak, share=None, **extra):
    gbs = nbytes / (ms * 1e-3) / 1e9
    d = {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "bytes": int(nbytes),
         "share": share}
    d.update(extra)
    return d


def gpu_index():
    dev = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    return vis.split(",")[dev] if vis else dev


def run_ours(args, rank, world, dev, peak, peak_src):
    n_layers = layers_of(args)
    c = Case(args.workload, dev, rank_seed(rank), batch=args.batch, layers=n_layers, context=args.context)
    stream = torch.cuda.current_stream()
    c.pack()
    torch.cuda.synchronize()

    # the pack kernels, timed alone (the cache is packed once; a decode step
    # does not repack it)
    kernels = {}
    for name, call in c.pack_calls():
        ms = graph_time(call, min(args.steps, 10), 2, stream, args.eager)
        kernels[name] = kernel_entry(ms, c.nbytes[name], peak,
                                     note="K and V pages of the pool, two launches; not in the step")
    c.pack()                                    # the cache as the step reads it
    torch.cuda.synchronize()

    # the step: one decode-attention launch; the timed steps replay one
    # captured call (a CUDA graph), so host launch overhead is not measured
    graph = None
    if not args.eager:
        c.decode()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            c.decode()
    step = graph.replay if graph is not None else c.decode
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_index())
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    del graph
    c.check_flags()
    own_ms = total_ms / args.steps
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    step_bytes = c.nbytes["decode"]
    value = step_bytes * world * args.steps / (total_ms * 1e-3) / 1e9
    kernels["decode"] = kernel_entry(own_ms, step_bytes, peak, share=1.0,
                                     note="the step: one launch for every layer of the batch")

    full_size = args.batch is None and args.layers is None and args.context is None

    def roof(name):
        k = kernels[name]
        return {"bound": "hbm", "achieved": k["gbs"], "peak": peak, "unit": "GB/s",
                "frac": k["frac"], "traffic": ncu_traffic(name, args.workload if full_size else None),
                "kernel": name, "peak_source": peak_src, "algorithmic_bytes_per_launch": k["bytes"]}

    res = {"value": value, "ms_per_step": ms_per_step, "kernels": kernels, "roofline": roof("decode"),
           "gpu_launches": args.steps, "clocks": clk, "step_bytes": step_bytes,
           "cfg": dict(c.cfg, layers=n_layers), "pages": c.pages()}
    packs = [n for n in ("pack_ternary", "pack_fp8", "pack_bf16") if n in kernels]
    if packs:
        res["pack_roofline"] = roof(packs[0])
    if not args.no_extras and n_layers == 1:
        K = c.K
        ap = time_append_retier(args, K, c.cfg, c.cache, c.lens, c.older, c.B, c.H, c.D, c.max_pages, c.hp, peak)
        if ap is not None:
            kernels["append_retier"] = ap
        pr = time_promote(args, K, c.cfg, c.cache, c.lens, c.older, c.B, c.H, c.D, c.max_pages, c.hp, peak)
        if pr is not None:
            kernels["promote"] = pr
        ex = time_exans(args, K, c.cache, c.H, c.D, peak)
        if ex is not None:
            kernels.update(ex)
        c.pack()                                # the extras overwrite parts of the cache
        torch.cuda.synchronize()
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, c, step_bytes, world, dev)
    del c
    torch.cuda.empty_cache()
    return res


def run_e2e(args, c, step_bytes, world, dev):
    """The step through the public API with host buffers: every step copies
    its inputs (Q, context lengths, block table, anchor tags) from pinned
    host memory to the device, runs the decode call and copies the output
    back, all inside the timed region.  The compressed cache is resident on
    the device, as it is between decode steps of a server."""
    stream = torch.cuda.current_stream()
    h_q = c.q.cpu().pin_memory()
    h_l = c.lens.cpu().pin_memory()
    h_bt = c.cache.block_table.cpu().pin_memory()
    h_old = None if c.older is None else c.older.cpu().pin_memory()
    h_out = torch.empty(c.out.shape, dtype=c.out.dtype, pin_memory=True)
    q_d = torch.empty_like(c.q)
    l_d = torch.empty_like(c.lens)

    def step():
        q_d.copy_(h_q, non_blocking=True)
        l_d.copy_(h_l, non_blocking=True)
        c.cache.block_table.copy_(h_bt, non_blocking=True)
        if h_old is not None:
            c.older.copy_(h_old, non_blocking=True)
        c.decode(q=q_d, lens=l_d)
        h_out.copy_(c.out, non_blocking=True)
        stream.synchronize()
        return float(h_out[0, 0, 0])

    for _ in range(3):
        step()
    steps = max(3, min(args.steps, 50))
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    c.check_flags()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    h2d = (h_q.numel() * h_q.element_size() + h_l.numel() * 4 + h_bt.numel() * 4
           + (0 if h_old is None else h_old.numel()))
    return {"value": step_bytes * world * steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(h_out.numel() * 4),
            "ms_per_step": ms / steps, "steps": steps,
            "note": "per step: H2D of Q, lengths, block table (and anchor tags) from pinned memory, "
                    "the decode call, D2H of the fp32 output, stream synchronize"}


def run_configs(args, dev, peak, skip_key=None):
    """The other workloads, each built, packed and decoded in this run:
    decode and pack per pool as average device times over CUDA-graph
    replays.  Fractions are of the same HBM peak as the step."""
    stream = torch.cuda.current_stream()
    out = {}
    for key, wl, layers, batch, context in CONFIG_SET:
        if key == skip_key:
            continue
        c = Case(wl, dev, seed=0, batch=batch, layers=layers, context=context)
        c.pack()
        torch.cuda.synchronize()
        row = {"workload": WORKLOAD_TEXT[wl], "layers": layers, "batch": c.B,
               "context": (list(c.cfg["context"]) if isinstance(c.cfg["context"], tuple) else c.cfg["context"]),
               "entries": layers * c.B, "pages": c.pages(),
               "shared_source": c.shared_source}
        # pack rates only where every layer has its own source pages (with a
        # shared source, later layers' reads hit L2)
        for name, call in ([] if c.shared_source else c.pack_calls()):
            ms = graph_time(call, 5, 1, stream, args.eager)
            row[name] = kernel_entry(ms, c.nbytes[name], peak)
            del row[name]["share"]
        c.pack()
        torch.cuda.synchronize()
        ms = graph_time(c.decode, 20, 3, stream, args.eager)
        c.check_flags()
        row["decode"] = kernel_entry(ms, c.nbytes["decode"], peak)
        del row["decode"]["share"]
        out[key] = row
        del c
        torch.cuda.empty_cache()
    out["bulk"] = run_bulk_block(args, dev, peak)
    return out


def run_bulk_block(args, dev, peak):
    """The bulk workload's kernels, each timed alone: ternary quantise+pack
    and dequantise, FP8 page quantise and dequantise of the same 1 GiB."""
    import compressed_decode_attention_kvc_b200 as K
    stream = torch.cuda.current_stream()
    pages = synth.make_bulk_pages(seed=0, device=dev)
    n, H, _, D = pages.shape
    codes = torch.empty((n, H, P, D // 4), dtype=torch.uint8, device=dev)
    gamma = torch.empty((n, H), dtype=torch.float32, device=dev)
    f8 = torch.empty((n, H, P, D), dtype=torch.uint8, device=dev)
    sc = torch.empty((n,), dtype=torch.float32, device=dev)
    rt = torch.empty_like(pages)
    calls = {
        "pack_ternary": (lambda: K.kvc_quantize_pack_pages(pages, None, n, P, H, D, K.KVC_FMT_TERNARY2, codes, gamma),
                         bulk_bytes(n, H, D)),
        "dequant_ternary": (lambda: K.kvc_dequantize_pages(codes, gamma, None, n, P, H, D, K.KVC_FMT_TERNARY2, rt),
                            bulk_bytes(n, H, D)),
        "pack_fp8": (lambda: K.kvc_quantize_pack_pages(pages, None, n, P, H, D, K.KVC_FMT_FP8_E4M3, f8, sc),
                     bulk_bytes(n, H, D, "fp8")),
        "dequant_fp8": (lambda: K.kvc_dequantize_pages(f8, sc, None, n, P, H, D, K.KVC_FMT_FP8_E4M3, rt),
                        bulk_bytes(n, H, D, "fp8")),
    }
    row = {"workload": WORKLOAD_TEXT["bulk"], "pages": n}
    for name in ("pack_ternary", "dequant_ternary", "pack_fp8", "dequant_fp8"):
        fn, nb = calls[name]
        if name.startswith("dequant"):
            calls["pack_" + name.split("_")[1]][0]()
        ms = graph_time(fn, 10, 2, stream, args.eager)
        row[name] = kernel_entry(ms, nb, peak)
        del row[name]["share"]
    del pages, codes, gamma, f8, sc, rt
    torch.cuda.empty_cache()
    return row


def time_append_retier(args, K, cfg, cache, lens, older, B, H, D, max_pages, hp, peak):
    """The next row of the design: one decode step's cache update
    (kvc_append_retier) on this batch, timed alone and not part of the step.
    Each sequence appends token L - 1 of a length-(L - 1) cache, so the page
    leaving the window is retiered for every sequence whose L - window is a
    multiple of 16; a scratch copy of the block table is restored before
    each call, and retiered pages overwrite ternary slots 0..B-1 (timing
    only; the step above has already been measured)."""
    if cfg["window"] < 1:
        return None
    dev = lens.device
    lens_a = (lens - 1).clamp(min=0)
    bt0 = cache.block_table.clone()
    # the cache holds L tokens, so the page leaving the window at length
    # L - 1 is already ternary: give it the high-precision slot of another
    # window page (not the newest) so the retier reads a valid page
    for b, L in enumerate(lens_a.cpu().tolist()):
        x = L - cfg["window"] + 1
        if x > 0 and x % P == 0 and (x // P - 1) * P >= cfg["sink"] and L // P >= 1:
            bt0[b, x // P - 1] = cache.block_table[b, L // P - 1]
    bt = bt0.clone()
    n_t = cache.struct.n_pages[2]
    if n_t < B:
        return None
    tern_slot = torch.arange(B, dtype=torch.int32, device=dev)
    freed = torch.empty(B, dtype=torch.int32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    k_new = torch.randn((B, H, D), device=dev).to(torch.bfloat16)
    v_new = torch.randn((B, H, D), device=dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream()

    def one():
        bt.copy_(bt0)
        K.kvc_append_retier(k_new, v_new, cache.struct, bt, None, lens_a, tern_slot, freed, flags, B, H, D,
                            P, max_pages, cfg["sink"], cfg["window"], hp)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    if int(flags.item()):
        raise RuntimeError(f"append_retier device flags {int(flags.item())}")
    n_ret = int((freed >= 0).sum().item())
    # device time: replay a captured graph of reps (restore + append) pairs,
    # minus the same graph with the restore copies alone
    reps = 20
    g_full, g_copy = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_full):
        for _ in range(reps):
            one()
    with torch.cuda.graph(g_copy):
        for _ in range(reps):
            bt.copy_(bt0)
    times = []
    for g in (g_full, g_copy):
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / (5 * reps))
    del g_full, g_copy
    ms = max(times[0] - times[1], 1e-6)
    row = 2 * H * D * 2
    page = 2 * H * P * D * (2 if hp == K.KVC_FMT_BF16 else 1)
    nbytes = B * 2 * row + (0 if hp == K.KVC_FMT_BF16 else B * 2 * page) + n_ret * (page + 2 * H * (P * D // 4 + 4) + 8)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "bytes": int(nbytes),
            "share": None, "sequences_retiered": n_ret, "note": "one decode step's append + retier, not in the step"}


def time_promote(args, K, cfg, cache, lens, older, B, H, D, max_pages, hp, peak, per_seq=32):
    """The stale-to-anchor row of the design: kvc_promote_pages re-expands
    per_seq stale pages of every sequence (spread over its stale range) into
    anchors of the high-precision format, timed alone and not part of the
    step.  The anchors go to scratch pools (the struct's anchor pools are
    replaced by them); a scratch block table and tag array are restored
    before each call."""
    dev = lens.device
    L = lens.cpu().tolist()
    tags_h = None if older is None else older.cpu()
    reqs = []
    for b in range(B):
        first = -(-cfg["sink"] // P)                            # first page past the sinks
        last = max(0, (L[b] - cfg["window"]) // P)              # pages before the window's first
        cand = [j for j in range(first, last) if tags_h is None or int(tags_h[b, j]) == K.KVC_FMT_TERNARY2]
        if len(cand) >= per_seq:
            step = len(cand) // per_seq
            reqs += [(b, cand[i * step]) for i in range(per_seq)]
    if not reqs:
        return None
    n = len(reqs)
    bf = hp == K.KVC_FMT_BF16
    ak = torch.empty((n, H, P, D), dtype=torch.bfloat16 if bf else torch.uint8, device=dev)
    av = torch.empty_like(ak)
    sk = torch.empty(n, dtype=torch.float32, device=dev)
    sv = torch.empty_like(sk)
    st = K.kvc_paged_cache()
    ctypes_copy(st, cache.struct)
    if bf:
        st.k_bf16, st.v_bf16 = ak.data_ptr(), av.data_ptr()
    else:
        st.k_fp8, st.v_fp8 = ak.data_ptr(), av.data_ptr()
        st.k_fp8_scale, st.v_fp8_scale = sk.data_ptr(), sv.data_ptr()
    st.n_pages[hp] = n
    bt0 = cache.block_table.clone()
    bt = bt0.clone()
    tags0 = (torch.full((B, max_pages), K.KVC_FMT_TERNARY2, dtype=torch.uint8, device=dev) if older is None
             else older.clone())
    tags = tags0.clone()
    seq = torch.tensor([r[0] for r in reqs], dtype=torch.int32, device=dev)
    page = torch.tensor([r[1] for r in reqs], dtype=torch.int32, device=dev)
    slot = torch.arange(n, dtype=torch.int32, device=dev)
    freed = torch.empty(n, dtype=torch.int32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def restore():
        bt.copy_(bt0)
        tags.copy_(tags0)

    def one():
        restore()
        K.kvc_promote_pages(st, bt, tags, lens, seq, page, slot, n, freed, flags, B, H, D, P, max_pages,
                            cfg["sink"], cfg["window"], hp, hp)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    if int(flags.item()) or int((freed < 0).sum().item()):
        raise RuntimeError(f"promote device flags {int(flags.item())}")
    reps = 20
    g_full, g_copy = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_full):
        for _ in range(reps):
            one()
    with torch.cuda.graph(g_copy):
        for _ in range(reps):
            restore()
    times = []
    for g in (g_full, g_copy):
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / (5 * reps))
    del g_full, g_copy
    ms = max(times[0] - times[1], 1e-6)
    per_page = 2 * H * (P * D // 4 + 4) + 2 * H * P * D * (2 if bf else 1) + (0 if bf else 8)
    nbytes = n * per_page
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "bytes": int(nbytes),
            "share": None, "pages_promoted": n,
            "note": f"{n} stale pages re-expanded to {'BF16' if bf else 'FP8'} anchors, not in the step"}


def time_exans(args, K, cache, H, D, peak):
    """The lossless exponent-split codec on the step's BF16 pages (the K and
    V pages of the sinks and windows, gathered once into one source so that
    one launch codes them all): encode, then decode, each timed alone as
    graph replays (not part of the step); the decoded pages are checked
    against the source bit for bit."""
    pools = [cache.pools.get("k_bf16"), cache.pools.get("v_bf16")]
    if any(t is None or t.numel() == 0 for t in pools):
        return None
    src = torch.cat(pools)
    dev = src.device
    n = src.shape[0]
    N = H * P * D
    ws_bytes = K.kvc_exans_workspace_size(n, P, H, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dst_bytes = n * (64 + 2 * N)
    dst = torch.empty(dst_bytes, dtype=torch.uint8, device=dev)
    off = torch.empty(n + 1, dtype=torch.int64, device=dev)
    out = torch.empty_like(src)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def enc():
        K.kvc_exans_encode(src, None, n, P, H, D, ws, ws_bytes, dst, dst_bytes, off)

    def dec():
        K.kvc_exans_decode(dst, dst_bytes, off, n, None, n, P, H, D, out, flags)

    enc()
    dec()
    torch.cuda.synchronize()
    if int(flags.item()) or not torch.equal(out.view(torch.int16), src.view(torch.int16)):
        raise RuntimeError("exponent-split codec round trip failed")
    coded = int(off[-1].item())
    raw = 2 * n * N
    res = {}
    for name, fn, moved in (("exans_encode", enc, raw + coded), ("exans_decode", dec, coded + raw)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 10
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        del g
        gbs = moved / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "bytes": int(moved),
                     "share": None, "bf16_gbs": round(raw / (ms * 1e-3) / 1e9, 1),
                     "ratio": round(raw / coded, 4), "pages": n,
                     "note": "lossless exponent-split coding of the BF16 K and V pools, not in the step; "
                             "gbs counts bf16 + coded bytes, bf16_gbs the bf16 bytes alone"}
    return res


def ctypes_copy(dst, src):
    for name, _ in src._fields_:
        if name == "n_pages":
            for f in range(3):
                dst.n_pages[f] = src.n_pages[f]
        else:
            setattr(dst, name, getattr(src, name))


def run_bulk(args, rank, world, dev, peak, peak_src):
    """One step = ternary quantise+pack of every page of the 1 GiB workload,
    then dequantise all of it back to bf16 (both directions timed)."""
    import compressed_decode_attention_kvc_b200 as K
    pages = synth.make_bulk_pages(seed=rank_seed(rank), device=dev)              # [n][H][P][D] bf16
    n, H, _, D = pages.shape
    codes = torch.empty((n, H, P, D // 4), dtype=torch.uint8, device=dev)
    gamma = torch.empty((n, H), dtype=torch.float32, device=dev)
    rt = torch.empty_like(pages)
    stream = torch.cuda.current_stream()
    nb = bulk_bytes(n, H, D)
    nbytes = {"pack_ternary": nb, "dequant_ternary": nb}

    def step(ev=None):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)] if ev is not None else None
        if e: e[0].record(stream)
        K.kvc_quantize_pack_pages(pages, None, n, P, H, D, K.KVC_FMT_TERNARY2, codes, gamma)
        if e: e[1].record(stream)
        K.kvc_dequantize_pages(codes, gamma, None, n, P, H, D, K.KVC_FMT_TERNARY2, rt)
        if e:
            e[2].record(stream)
            ev.append(("pack_ternary", e[0], e[1]))
            ev.append(("dequant_ternary", e[1], e[2]))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    marks = []
    for _ in range(min(args.steps, 20)):
        step(marks)
    torch.cuda.synchronize()
    per_kernel = {}
    for name, e0, e1 in marks:
        per_kernel.setdefault(name, []).append(e0.elapsed_time(e1))
    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[torch.cuda.current_device()])
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    del graph
    step_bytes = sum(nbytes.values())
    total_ms = max_over_ranks(total_ms, world, dev)
    kernels = {}
    for name, ts in per_kernel.items():
        avg = sum(ts) / len(ts)
        gbs = nbytes[name] / (avg * 1e-3) / 1e9
        kernels[name] = {"ms": round(avg, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                         "bytes": int(nbytes[name]), "share": 0.0}
    tot = sum(k["ms"] for k in kernels.values())
    for k in kernels.values():
        k["share"] = round(k["ms"] / tot, 4)
    dom = max(kernels, key=lambda nm: kernels[nm]["ms"])

    def roof(name):
        k = kernels[name]
        return {"bound": "hbm", "achieved": k["gbs"], "peak": peak, "unit": "GB/s", "frac": k["frac"],
                "traffic": ncu_traffic(name, "bulk"), "kernel": name, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": k["bytes"]}

    res = {"value": step_bytes * world * args.steps / (total_ms * 1e-3) / 1e9,
           "ms_per_step": total_ms / args.steps, "kernels": kernels, "roofline": roof(dom),
           "pack_roofline": roof("pack_ternary"), "dequant_roofline": roof("dequant_ternary"),
           "gpu_launches": 2 * args.steps, "clocks": clk, "step_bytes": step_bytes,
           "cfg": {"batch": n, "context": P, "n_q_heads": 0, "n_kv_heads": H, "head_dim": D},
           "pages": {"bf16": 0, "fp8": 0, "ternary": n}}
    if not args.no_e2e:
        hp_src = torch.empty(pages.shape, dtype=pages.dtype, pin_memory=True)
        hp_src.copy_(pages)
        h_rt = torch.empty(pages.shape, dtype=pages.dtype, pin_memory=True)
        steps = max(2, min(args.steps, 5))

        def e2e_step():
            pages.copy_(hp_src, non_blocking=True)
            K.kvc_quantize_pack_pages(pages, None, n, P, H, D, K.KVC_FMT_TERNARY2, codes, gamma)
            K.kvc_dequantize_pages(codes, gamma, None, n, P, H, D, K.KVC_FMT_TERNARY2, rt)
            h_rt.copy_(rt, non_blocking=True)
            stream.synchronize()

        e2e_step()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        ms = max_over_ranks(ms, world, dev)
        res["e2e"] = {"value": step_bytes * world * steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
                      "h2d_bytes_per_step": int(pages.numel() * 2), "d2h_bytes_per_step": int(rt.numel() * 2),
                      "ms_per_step": ms / steps, "steps": steps}
    return res


# --------------------------------------------------------- oracle arm
#
# The CPU oracle, as it stands, on the host's cores: one worker process per
# core (spawned, so that no worker inherits the parent's CUDA context), each
# running numpy on one thread.  A worker builds the oracle's compressed cache
# of a few (sequence, KV head) pairs of the workload once, then decodes them
# over and over; only the decodes are timed, as on the GPU side.

def oracle_inputs(workload):
    """Two sequences of the workload (same shapes and value distributions
    per sequence); the oracle samples (sequence, KV head) pairs from them."""
    return synth.make_decode_inputs(workload, seed=0, device="cpu", batch=2)


def pick_pairs(cfg, inp, k, offset=0):
    B, H = inp["q"].shape[0], cfg["n_kv_heads"]
    return [((offset + i) % B, ((offset + i) // B) % H) for i in range(k)]


def oracle_pair(inp, cfg, b, g):
    """The oracle's compressed cache of sequence b, KV head g, with the
    query heads of g and the decode bytes of the pair (the GPU step's
    accounting, per (sequence, KV head))."""
    import oracle as O
    H, D, hq = cfg["n_kv_heads"], cfg["head_dim"], cfg["n_q_heads"]
    G = hq // H
    L = int(inp["context_lens"][b])
    kb = inp["k_pages"][b, :, g:g + 1].contiguous().view(torch.int16).numpy().view(np.uint16)
    vb = inp["v_pages"][b, :, g:g + 1].contiguous().view(torch.int16).numpy().view(np.uint16)
    hp = O.BF16 if cfg["hp"] == "bf16" else O.FP8_E4M3
    older = None
    if inp["anchor"].any():
        older = np.where(inp["anchor"][b:b + 1].numpy(), O.BF16, O.TERNARY).astype(np.uint8)
    cache, bt, fmt = O.build_paged_cache(kb[None], vb[None], [L], cfg["sink"], cfg["window"], hp,
                                         older_fmt=older)
    qb = inp["q"][b:b + 1, g * G:(g + 1) * G].contiguous().view(torch.int16).numpy().view(np.uint16)
    n_bf, n_f8, n_t = cache.k_bf16.shape[0], cache.k_fp8.shape[0], cache.k_tern.shape[0]
    nbytes = (2 * (n_bf * 2 * P * D + n_f8 * P * D + n_t * (P * D // 4 + 4)) + G * D * 6
              + 4 * (n_bf + n_f8 + n_t))
    return {"q": qb, "cache": cache, "bt": bt, "fmt": fmt, "L": L, "bytes": nbytes}


def oracle_decode(item):
    """One oracle decode of a prepared pair; returns its bytes."""
    import oracle as O
    O.decode_attention(item["q"], item["cache"], item["bt"], item["fmt"], [item["L"]], 1)
    return item["bytes"]


def oracle_bulk_item(n_pages=48, seed=0):
    pages = synth.make_bulk_pages(seed=seed, device="cpu", n_pages=n_pages)
    n, H, _, D = pages.shape
    return {"bits": pages.contiguous().view(torch.int16).numpy().view(np.uint16),
            "bytes": 2 * bulk_bytes(n, H, D)}


def oracle_bulk(item):
    """Oracle ternary pack + dequantise of a sample of bulk pages."""
    import oracle as O
    codes, gamma = O.quantize_pack_ternary(item["bits"])
    O.dequantize_ternary(codes, gamma)
    return item["bytes"]


def oracle_items(workload, k, offset):
    if workload == "bulk":
        return [oracle_bulk_item(seed=offset + i) for i in range(k)]
    inp = oracle_inputs(workload)
    cfg = inp["cfg"]
    return [oracle_pair(inp, cfg, b, g) for b, g in pick_pairs(cfg, inp, k, offset)]


def oracle_run(workload, item):
    return oracle_bulk(item) if workload == "bulk" else oracle_decode(item)


_ORACLE = {}


def _oracle_worker_init(workload, per_worker, counter, barrier):
    torch.set_num_threads(1)
    with counter.get_lock():
        slot = counter.value
        counter.value += 1
    _ORACLE["workload"] = workload
    _ORACLE["items"] = oracle_items(workload, per_worker, slot * per_worker)
    barrier.wait(timeout=900)


def _oracle_worker_task(i):
    items = _ORACLE["items"]
    return oracle_run(_ORACLE["workload"], items[i % len(items)])


def host_cores():
    """Cores this process may use: its CPU affinity, capped by a cgroup CPU
    quota when one is set."""
    n = len(os.sched_getaffinity(0))
    try:
        quota, period = open("/sys/fs/cgroup/cpu.max").read().split()
        if quota != "max":
            n = min(n, max(1, int(int(quota) // int(period))))
    except (OSError, ValueError):
        pass
    return n


def host_mem_available():
    """Bytes of host memory available to this process (MemAvailable, capped
    by the cgroup's limit)."""
    avail = None
    try:
        for line in open("/proc/meminfo"):
            if line.startswith("MemAvailable:"):
                avail = int(line.split()[1]) * 1024
    except OSError:
        pass
    try:
        lim = open("/sys/fs/cgroup/memory.max").read().strip()
        cur = int(open("/sys/fs/cgroup/memory.current").read().strip())
        if lim != "max":
            room = int(lim) - cur
            avail = room if avail is None else min(avail, room)
    except (OSError, ValueError):
        pass
    return avail


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# host memory one oracle worker may hold (interpreter, torch, the workload's
# two-sequence inputs while the pairs are built)
WORKER_BYTES = {"llama8b": 1 << 30, "qwen3b": 1 << 29, "longctx": 3 << 30, "tiny": 1 << 29, "bulk": 1 << 29}


class OraclePool:
    """Worker processes, one per usable core, each holding its prepared
    oracle items; `run(n)` hands out n items and returns (bytes, seconds)."""

    def __init__(self, workload, per_worker=2):
        import multiprocessing as mp
        cores = host_cores()
        mem = host_mem_available()
        cap = cores if mem is None else max(1, min(cores, int(mem * 0.6) // WORKER_BYTES[workload]))
        self.workers = cap
        self.cores_seen = cores
        ctx = mp.get_context("spawn")
        counter = ctx.Value("i", 0)
        barrier = ctx.Barrier(cap + 1)
        self.pool = ctx.Pool(cap, initializer=_oracle_worker_init,
                             initargs=(workload, per_worker, counter, barrier))
        barrier.wait(timeout=900)            # every worker has built its items

    def run(self, n):
        t0 = time.perf_counter()
        nbytes = sum(self.pool.imap_unordered(_oracle_worker_task, range(n), chunksize=1))
        return nbytes, time.perf_counter() - t0

    def close(self):
        self.pool.terminate()
        self.pool.join()


def _sample_text(workload):
    if workload == "bulk":
        return "48-page samples of the bulk workload: oracle ternary pack + dequantise"
    return (f"(sequence, KV head) pairs of the {workload} workload: oracle fp64 decode attention "
            f"over the oracle's compressed cache of the pair (cache built before timing)")


def cpu_baseline(args, budget_one=5.0, budget_all=10.0):
    """The oracle timed on one host core and on all of them."""
    workload = args.workload
    items = oracle_items(workload, 2, 0)
    oracle_run(workload, items[0])
    n1, t1 = 0, 0.0
    k = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_one or k < 2:
        n1 += oracle_run(workload, items[k % len(items)])
        k += 1
    t1 = time.perf_counter() - t0
    one = n1 / t1 / 1e9
    per_item = t1 / k
    res = {"value": one, "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{k} {_sample_text(workload)}, {t1:.1f} s on one host core",
           "one_core": {"value": one, "items": k, "seconds": round(t1, 2)},
           "cpu_model": cpu_model(), "host_cpus": os.cpu_count()}
    pool = None
    try:
        pool = OraclePool(workload)
        n = pool.workers * max(1, int(round(budget_all / per_item)))
        pool.run(pool.workers)                 # warm-up: one item per worker
        nb, dt = pool.run(n)
        res.update({"value": nb / dt / 1e9, "cores": pool.workers,
                    "sample": f"{n} {_sample_text(workload)}, {dt:.1f} s on {pool.workers} worker "
                              f"processes (one numpy thread each) over {pool.cores_seen} usable cores; "
                              f"one core alone: {one:.4g} GB/s over {k} items",
                    "all_cores": {"value": nb / dt / 1e9, "items": n, "seconds": round(dt, 2),
                                  "workers": pool.workers, "usable_cores": pool.cores_seen}})
    except Exception as e:  # keep the one-core figure if the pool cannot run
        res["all_cores"] = {"error": f"{type(e).__name__}: {e}"}
    finally:
        if pool is not None:
            pool.close()
    return res


def run_reference(args):
    """The oracle arm: each step decodes one prepared pair per worker
    process (one per usable host core), timed by the wall clock."""
    workload = args.workload
    pool = OraclePool(workload)
    try:
        for _ in range(args.warmup):
            pool.run(pool.workers)
        nbytes, dt = 0, 0.0
        for _ in range(args.steps):
            nb, t = pool.run(pool.workers)
            nbytes += nb
            dt += t
    finally:
        pool.close()
    v = nbytes / dt / 1e9
    sample = (f"each step: {pool.workers} {_sample_text(workload)}, one per worker process "
              f"(one numpy thread each, {pool.cores_seen} usable cores)")
    if workload == "bulk":
        config = bulk_config_block(args)
    else:
        cfg = dict(synth.WORKLOADS[workload])
        if args.batch:
            cfg["batch"] = args.batch
        if args.context:
            cfg["context"] = args.context
        config = config_block(args, cfg)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": pool.workers, "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model(), "host_cpus": os.cpu_count()},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def bulk_config_block(args):
    b = synth.BULK
    return {"workload": f"bulk: {WORKLOAD_TEXT['bulk']}", "n_pages": b["n_pages"],
            "n_kv_heads": b["n_kv_heads"], "head_dim": b["head_dim"], "page_size": P,
            "step": "ternary quantise+pack of all pages, then dequantise all pages to bf16",
            "l2": "inputs larger than L2 (1 GiB of bf16 pages)",
            "timing": ("CUDA events around K eager steps" if args.eager else
                       "CUDA events around K replays of one captured step (CUDA graph)")
                      + "; per-kernel times from event pairs around each launch in eager steps",
            "parallelism": f"dp{args.gpus} (independent data per GPU)"}


def config_block(args, cfg):
    ctx = cfg["context"]
    n_layers = layers_of(args)
    return {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]}"
                        + (f", {n_layers} layers per step" if n_layers > 1 else ""),
            "layers": n_layers,
            "batch": cfg["batch"], "context": list(ctx) if isinstance(ctx, tuple) else ctx,
            "n_q_heads": cfg["n_q_heads"], "n_kv_heads": cfg["n_kv_heads"], "head_dim": cfg["head_dim"],
            "page_size": P,
            "step": "one decode-attention launch (every layer of the stack) over the batch's compressed "
                    "paged cache, packed once before timing",
            "l2": "inputs larger than L2 (the compressed cache the step reads exceeds 126 MB)",
            "timing": ("CUDA events around K eager calls" if args.eager else
                       "CUDA events around K replays of one captured decode call (CUDA graph)"),
            "parallelism": f"dp{args.gpus} (independent batch per GPU)"}


def main():
    args = parse()
    if args.decode_kernel == "tcgen05":
        os.environ["KVC_DECODE_KERNEL"] = "tcgen05"
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    peak, peak_src = load_peaks()
    bulk = args.workload == "bulk"
    r = (run_bulk if bulk else run_ours)(args, rank, world, dev, peak, peak_src)
    configs = None
    if world == 1 and not args.no_configs:
        skip = None
        if not bulk and args.batch is None and args.context is None:
            n_layers = layers_of(args)
            for key, wl, layers, batch, context in CONFIG_SET:
                if wl == args.workload and layers == n_layers and batch is None and context is None:
                    skip = key
        configs = run_configs(args, dev, peak, skip_key=skip)
    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(r["value"], 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": bulk_config_block(args) if bulk else config_block(args, r["cfg"]),
            "roofline": r["roofline"], "pack_roofline": r.get("pack_roofline"),
            "kernels": r["kernels"], "pages": r["pages"], "gpu_launches": r["gpu_launches"],
            "clocks": r["clocks"], "e2e": r.get("e2e"), "configs": configs,
        }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(args)
            line["cpu_baseline"] = cb
            line["oracle_speedup"] = round(line["value"] / cb["value"], 1)
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
