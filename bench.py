#!/usr/bin/env python
"""Benchmark: compress a batch's bf16 KV into the mixed-format paged cache and
run one decode-attention pass over it (one "step"), on synthetic data shaped
like the workload, through libkvc's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

Prints ONE JSON line (rank 0).  The metric is HBM throughput: algorithmic
bytes (what the method must read and write: bf16 source pages, packed codes
+ gamma, FP8 bytes + scales, BF16 pages, Q, block table, output) divided by
device time.  `--impl reference` times the CPU oracle on a bounded sample
of the same workload instead.  For N > 1 (torchrun) every rank runs its own
independent batch (weak scaling, no collective on the data path).
"""

from __future__ import annotations

import os

os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")   # the oracle baseline runs on one core
os.environ.setdefault("OMP_NUM_THREADS", "1")

import argparse
import hashlib
import json
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
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of replaying a captured CUDA graph")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


# ---------------------------------------------------------------- bytes

def algorithmic_bytes(cfg, layout, B, max_pages, has_older):
    """Bytes each kernel of one step must move, by kernel."""
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


# where each timed kernel's code lives: (file, kernel function, launcher);
# None = the whole file
KERNEL_SRC = {"decode": ("decode_tc.cu", None, None),
              "pack_ternary": ("quant.cu", "quant_ternary_kernel", "launch_quant_ternary"),
              "pack": ("quant.cu", "quant_ternary_kernel", "launch_quant_ternary"),
              "dequant_ternary": ("quant.cu", "dequant_ternary_kernel", "launch_dequant_ternary")}


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
    its launcher; for decode, the whole file."""
    spec = KERNEL_SRC.get(kernel_key)
    if spec is None:
        return None
    f, fn, launcher = spec
    path = os.path.join(ROOT, "compressed_decode_attention_kvc_b200", "csrc", f)
    src = open(path).read()
    if fn is None:
        text = src
    else:
        a = _function_text(src, fn, True)
        b = _function_text(src, launcher, False)
        if a is None or b is None:
            return None
        text = a + b
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


def run_ours(args, rank, world, dev, peak, peak_src):
    import compressed_decode_attention_kvc_b200 as K
    from compressed_decode_attention_kvc_b200 import paged_cache as PC

    n_layers = layers_of(args)
    inp = synth.make_decode_inputs(args.workload, seed=rank_seed(rank), device=dev, batch=args.batch)
    cfg = inp["cfg"]
    B, max_pages, H, _, D = inp["k_pages"].shape
    if n_layers > 1:
        # further layers: their own K, V and Q, the first layer's placement
        ks, vs, qs = [inp["k_pages"]], [inp["v_pages"]], [inp["q"]]
        for l in range(1, n_layers):
            o = synth.make_decode_inputs(args.workload, seed=rank * 1000 + l, device=dev, batch=args.batch)
            ks.append(o["k_pages"]); vs.append(o["v_pages"]); qs.append(o["q"])
            del o
        inp["k_pages"] = torch.cat(ks)
        inp["v_pages"] = torch.cat(vs)
        inp["q"] = torch.cat(qs)              # [layers * B][Hq][D], layer-major
        del ks, vs, qs
    hq = cfg["n_q_heads"]
    hp = K.KVC_FMT_BF16 if cfg["hp"] == "bf16" else K.KVC_FMT_FP8_E4M3
    older = None
    if inp["anchor"].any():
        older = torch.where(inp["anchor"], K.KVC_FMT_BF16, K.KVC_FMT_TERNARY2).to(torch.uint8)
    lens_h = inp["context_lens"].cpu()
    sk = None if inp["slot_key"] is None else inp["slot_key"].cpu()
    layout = PC.plan_paged_cache(lens_h, max_pages, cfg["sink"], cfg["window"], hp,
                                 older_fmt=None if older is None else older.cpu(), slot_key=sk)
    cache = PC.allocate_device_cache(layout, H, D, dev, n_layers=n_layers)
    kf = inp["k_pages"].view(n_layers * B * max_pages, H, P, D)
    vf = inp["v_pages"].view(n_layers * B * max_pages, H, P, D)
    q, lens = inp["q"], inp["context_lens"]
    ws_bytes = K.kvc_decode_workspace_size(n_layers * B, hq, H, D, max_pages)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty((n_layers * B, hq, D), dtype=torch.float32, device=dev)
    nbytes = {k: n_layers * v for k, v in algorithmic_bytes(cfg, layout, B, max_pages, older is not None).items()}
    stream = torch.cuda.current_stream()

    pools = [(f, n * n_layers) for f, n in zip((K.KVC_FMT_BF16, K.KVC_FMT_FP8_E4M3, K.KVC_FMT_TERNARY2),
                                               layout.pool_pages) if n > 0]
    names = {K.KVC_FMT_BF16: "pack_bf16", K.KVC_FMT_FP8_E4M3: "pack_fp8", K.KVC_FMT_TERNARY2: "pack_ternary"}
    fields = {K.KVC_FMT_BF16: ("k_bf16", "v_bf16", None, None),
              K.KVC_FMT_FP8_E4M3: ("k_fp8", "v_fp8", "k_fp8_scale", "v_fp8_scale"),
              K.KVC_FMT_TERNARY2: ("k_tern", "v_tern", "k_gamma", "v_gamma")}
    launches_per_step = 2 * len(pools) + 1

    def step(ev=None):
        marks = []
        for f, n in pools:
            kn, vn, ks, vs = fields[f]
            pl = cache.pools
            if ev is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            K.kvc_quantize_pack_pages(kf, cache.page_ids[f], n, P, H, D, f, pl[kn], pl[ks] if ks else None)
            K.kvc_quantize_pack_pages(vf, cache.page_ids[f], n, P, H, D, f, pl[vn], pl[vs] if vs else None)
            if ev is not None:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(stream)
                marks.append((names[f], e0, e1))
        if ev is not None:
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        K.kvc_decode_attention_paged_layers(q, cache.struct, cache.block_table, older, lens, n_layers, B,
                                            hq, H, D, P, max_pages, cfg["sink"], cfg["window"], hp, 0.0,
                                            out, ws, ws_bytes)
        if ev is not None:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
            marks.append(("decode", e0, e1))
            ev.extend(marks)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # per-kernel device times: eager steps with an event pair around each launch
    marks = []
    for _ in range(min(args.steps, 20)):
        step(marks)
    torch.cuda.synchronize()
    per_kernel = {}
    for name, e0, e1 in marks:
        per_kernel.setdefault(name, []).append(e0.elapsed_time(e1))
    # the timed steps replay one captured step (a CUDA graph), so host-side
    # launch overhead is not in the measurement
    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(args.warmup):
            graph.replay()
        stream = torch.cuda.current_stream()
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
    flags = K.kvc_decode_read_error(ws, n_layers * B, hq, H, D, max_pages)
    if flags:
        raise RuntimeError(f"device error flags {flags}")

    step_bytes = sum(nbytes.values())
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = step_bytes * world * args.steps / (total_ms * 1e-3) / 1e9

    kernels = {}
    for name, ts in per_kernel.items():
        avg = sum(ts) / len(ts)
        gbs = nbytes[name] / (avg * 1e-3) / 1e9
        kernels[name] = {"ms": round(avg, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                         "bytes": int(nbytes[name]), "share": 0.0}
    tot = sum(k["ms"] for k in kernels.values())
    for k in kernels.values():
        k["share"] = round(k["ms"] / tot, 4)
    dom = max(kernels, key=lambda n: kernels[n]["ms"])

    def roof(name):
        k = kernels[name]
        traffic = ncu_traffic(name, args.workload if args.batch is None and args.layers is None else None)
        return {"bound": "hbm", "achieved": k["gbs"], "peak": peak, "unit": "GB/s",
                "frac": k["frac"], "traffic": traffic, "kernel": name, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": k["bytes"]}

    res = {
        "value": value, "ms_per_step": ms_per_step, "kernels": kernels, "roofline": roof(dom),
        "decode_roofline": roof("decode"), "gpu_launches": launches_per_step * args.steps,
        "clocks": clk, "step_bytes": step_bytes, "cfg": dict(cfg, layers=n_layers),
        "pages": {"bf16": layout.pool_pages[0], "fp8": layout.pool_pages[1], "ternary": layout.pool_pages[2]},
    }

    ap = None if n_layers > 1 else time_append_retier(args, K, cfg, cache, lens, older, B, H, D, max_pages,
                                                       hp, peak)
    if ap is not None:
        res["kernels"]["append_retier"] = ap
    pr = None if n_layers > 1 else time_promote(args, K, cfg, cache, lens, older, B, H, D, max_pages, hp,
                                                 peak)
    if pr is not None:
        res["kernels"]["promote"] = pr
    ex = None if n_layers > 1 else time_exans(args, K, cache, H, D, peak)
    if ex is not None:
        res["kernels"].update(ex)
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, K, PC, inp, cfg, layout, cache, kf, vf, older, ws, ws_bytes, out,
                             step_bytes, world, dev, hp, n_layers)
    return res


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


def run_e2e(args, K, PC, inp, cfg, layout, cache, kf, vf, older, ws, ws_bytes, out, step_bytes,
            world, dev, hp, n_layers=1):
    """Same step through the public API with host buffers: planner on the
    host, H2D of the bf16 pages / Q / lengths / block table from pinned
    memory, pack + decode, D2H of the output, all inside the timed region."""
    B, max_pages, H, _, D = inp["k_pages"].shape
    B //= n_layers                                   # the inputs stack the layers
    hq = cfg["n_q_heads"]
    hk = torch.empty(kf.shape, dtype=kf.dtype, pin_memory=True)
    hv = torch.empty(vf.shape, dtype=vf.dtype, pin_memory=True)
    hk.copy_(kf)
    hv.copy_(vf)
    hq_t = inp["q"].cpu().pin_memory()
    hl = inp["context_lens"].cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h_older = None if older is None else older.cpu()
    sk = None if inp["slot_key"] is None else inp["slot_key"].cpu()
    q_d = torch.empty_like(inp["q"])
    l_d = torch.empty_like(inp["context_lens"])
    stream = torch.cuda.current_stream()

    def step():
        lay = PC.plan_paged_cache(hl, max_pages, cfg["sink"], cfg["window"], hp, older_fmt=h_older, slot_key=sk)
        kf.copy_(hk, non_blocking=True)
        vf.copy_(hv, non_blocking=True)
        q_d.copy_(hq_t, non_blocking=True)
        l_d.copy_(hl, non_blocking=True)
        cache.block_table.copy_(lay.block_table.pin_memory(), non_blocking=True)
        for f in range(3):
            if lay.pool_pages[f]:
                ids = lay.pool_src_ids[f]
                if n_layers > 1:
                    ids = torch.cat([ids + l * B * max_pages for l in range(n_layers)])
                cache.page_ids[f].copy_(ids.pin_memory(), non_blocking=True)
        PC.compress_into(cache, kf, vf)
        K.kvc_decode_attention_paged_layers(q_d, cache.struct, cache.block_table, older, l_d, n_layers, B,
                                            hq, H, D, P, max_pages, cfg["sink"], cfg["window"], hp, 0.0,
                                            out, ws, ws_bytes)
        hout.copy_(out, non_blocking=True)
        stream.synchronize()
        return float(hout[0, 0, 0])

    for _ in range(2):
        step()
    steps = max(2, min(args.steps, 10))
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    ms = max_over_ranks(ms, world, dev)
    h2d = (hk.numel() * 2 + hv.numel() * 2 + hq_t.numel() * 2 + hl.numel() * 4
           + layout.block_table.numel() * 4 + n_layers * sum(len(x) for x in layout.pool_src_ids) * 4)
    return {"value": step_bytes * world * steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(hout.numel() * 4),
            "ms_per_step": ms / steps, "steps": steps}


# ------------------------------------------------------- bulk workload

def bulk_bytes(n, H, D):
    """Algorithmic bytes of packing (or dequantising) n pages of H groups."""
    return n * H * (2 * P * D + P * D // 4 + 4)


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


def oracle_bulk_sample(n_pages=48, seed=0):
    """Oracle work on a sample of bulk pages: pack + dequantise; returns bytes."""
    import oracle as O
    pages = synth.make_bulk_pages(seed=seed, device="cpu", n_pages=n_pages)
    bits = pages.contiguous().view(torch.int16).numpy().view(np.uint16)
    codes, gamma = O.quantize_pack_ternary(bits)
    O.dequantize_ternary(codes, gamma)
    n, H, _, D = pages.shape
    return 2 * bulk_bytes(n, H, D)


# --------------------------------------------------------- oracle arm

def oracle_sample_step(inp, cfg, pairs):
    """Oracle work on a bounded sample: compress every page of the sampled
    (sequence, KV head) pairs and decode those pairs.  Returns algorithmic
    bytes of the sample (same accounting as the GPU step)."""
    import oracle as O
    H, D = cfg["n_kv_heads"], cfg["head_dim"]
    hq = cfg["n_q_heads"]
    G = hq // H
    nbytes = 0
    for b, g in pairs:
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
        O.decode_attention(qb, cache, bt, fmt, [L], 1)
        n_bf, n_f8, n_t = cache.k_bf16.shape[0], cache.k_fp8.shape[0], cache.k_tern.shape[0]
        grp = 2 * P * D
        nbytes += 2 * n_bf * 2 * grp + 2 * n_f8 * (grp + P * D) + 2 * n_t * (grp + P * D // 4 + 4)
        nbytes += 2 * (n_bf * grp + n_f8 * P * D + n_t * (P * D // 4 + 4)) + G * D * 6 + 4 * (n_bf + n_f8 + n_t)
    return nbytes


def oracle_inputs(workload):
    """Two sequences of the workload (same shapes and value distributions
    per sequence); the oracle arms sample (sequence, KV head) pairs from
    them."""
    return synth.make_decode_inputs(workload, seed=0, device="cpu", batch=2)


def pick_pairs(cfg, inp, k, offset=0):
    B, H = inp["q"].shape[0], cfg["n_kv_heads"]
    return [((offset + i) % B, (offset + i) % H) for i in range(k)]


def cpu_baseline(args, budget_s=12.0):
    if args.workload == "bulk":
        nbytes, k = 0, 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < budget_s:
            nbytes += oracle_bulk_sample(seed=k)
            k += 1
        dt = time.perf_counter() - t0
        return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                "sample": f"{k} x 48 pages of the bulk workload: oracle ternary pack + dequantise, "
                          f"{dt:.1f} s on one host core"}
    inp = oracle_inputs(args.workload)
    cfg = inp["cfg"]
    pairs_done, nbytes = 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        nbytes += oracle_sample_step(inp, cfg, pick_pairs(cfg, inp, 1, pairs_done))
        pairs_done += 1
    dt = time.perf_counter() - t0
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{pairs_done} (sequence, KV head) pairs of the {args.workload} workload: oracle "
                      f"pack of all their pages + fp64 decode attention, {dt:.1f} s on one host core"}


def run_reference(args):
    if args.workload == "bulk":
        for i in range(args.warmup):
            oracle_bulk_sample(seed=i)
        t0 = time.perf_counter()
        nbytes = sum(oracle_bulk_sample(seed=args.warmup + i) for i in range(args.steps))
        dt = time.perf_counter() - t0
        v = nbytes / dt / 1e9
        sample = "each step: 48 pages of the bulk workload - oracle ternary pack + dequantise, on one host core"
        return {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": bulk_config_block(args),
                "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    inp = oracle_inputs(args.workload)
    cfg = inp["cfg"]
    for i in range(args.warmup):
        oracle_sample_step(inp, cfg, pick_pairs(cfg, inp, 1, i))
    t0 = time.perf_counter()
    nbytes = 0
    for i in range(args.steps):
        nbytes += oracle_sample_step(inp, cfg, pick_pairs(cfg, inp, 1, args.warmup + i))
    dt = time.perf_counter() - t0
    v = nbytes / dt / 1e9
    sample = (f"each step: one (sequence, KV head) pair of the {args.workload} workload - oracle pack "
              f"of all its pages + fp64 decode attention, on one host core")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            # the workload our arm runs; the sample drawn from it is in cpu_baseline
            "config": config_block(args, dict(cfg, batch=args.batch or synth.WORKLOADS[args.workload]["batch"])),
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
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


def layers_of(args):
    """Attention layers decoded per step: the Qwen2.5-3B-shaped workload runs
    all 36 of its model's layers (one pack launch per format, one decode
    launch for the stack); the others are one layer."""
    return args.layers or (36 if args.workload == "qwen3b" else 1)


def config_block(args, cfg):
    ctx = cfg["context"]
    n_layers = layers_of(args)
    return {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]}"
                        + (f", {n_layers} layers per step" if n_layers > 1 else ""),
            "layers": n_layers,
            "batch": cfg["batch"], "context": list(ctx) if isinstance(ctx, tuple) else ctx,
            "n_q_heads": cfg["n_q_heads"], "n_kv_heads": cfg["n_kv_heads"], "head_dim": cfg["head_dim"],
            "page_size": P, "step": "pack every page of the batch into its format (bf16 copy / fp8 / "
                                    "ternary) + one decode-attention pass over the compressed cache",
            "l2": "inputs larger than L2 (bf16 source pages of the batch exceed 126 MB)",
            "timing": ("CUDA events around K eager steps" if args.eager else
                       "CUDA events around K replays of one captured step (CUDA graph)")
                      + "; per-kernel times from event pairs around each launch in eager steps",
            "parallelism": f"dp{args.gpus} (independent batch per GPU)"}


def main():
    args = parse()
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
    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(r["value"], 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": bulk_config_block(args) if bulk else config_block(args, r["cfg"]),
            "roofline": r["roofline"], "decode_roofline": r.get("decode_roofline"),
            "kernels": r["kernels"], "pages": r["pages"], "gpu_launches": r["gpu_launches"],
            "clocks": r["clocks"], "e2e": r.get("e2e"),
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
