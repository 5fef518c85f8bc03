"""Benchmark of the WUSH-KV runtime hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over the Qwen3-8B-shaped decode layer
(batch 16, 32 query / 8 KV heads, head_dim 128, context 32768, percentile-affine
2-bit K/V): append of the step's new token per sequence (key transform, quantize,
pack), query map by T_k^{-T}, split-K GQA decode attention over the packed cache.
`value` is the step's algorithmic HBM bytes / device time (GB/s); the quantize-
append throughput is measured beside it on a 2048-token chunk (QuEST 2-bit, the
bit-width sweep's shape).  With N > 1 (torchrun) every rank runs the same workload
on its own GPU (independent replicas, no collective on the data path); the time is
the max over ranks and `value` sums all ranks' bytes.

--impl reference times the fp64 CPU oracle (the only other implementation of the
method here) on a bounded sample of the same workload on the host cores.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import gen  # noqa: E402
from synth.configs import QWEN8B_DECODE, QWEN8B_LONG, QWEN8B_SWEEP, QWEN32B_STACK, quest  # noqa: E402

METRIC = "2-bit KV decode-attn HBM GB/s (% of peak) & quant-append tokens/s, 1×B200"
TAU = 1.0 / math.sqrt(128)
L2_FLUSH_BYTES = 512 << 20


# ncu summary of the decode kernel at this workload; its DRAM traffic is reported only
# while the kernel sources still hash to the value recorded beside it.
DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_tc_qwen8b_affine2.md")
DECODE_SOURCES = ("decode_tc.cu", "sm100.cuh", "wushkv_common.cuh", "wushkv_quant.cuh", "tmap.cu", "tmap.h")
APPEND_LAUNCHES, QUERY_LAUNCHES, DECODE_LAUNCHES = 1, 1, 2     # kernels per C-ABI call


def decode_source_hash():
    import hashlib
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "decode_attention_quant_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_decode_traffic():
    """DRAM read+write bytes per decode-kernel launch from the committed ncu summary,
    or None when there is none or the kernel changed since it was captured."""
    if not os.path.exists(DECODE_PROFILE):
        return None
    fields = {}
    with open(DECODE_PROFILE) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    try:
        if fields.get("kernel_source_sha256") != decode_source_hash():
            return None
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _f16_tensor_peak():
    """Dense fp16 tensor peak in TFLOP/s: the measured bf16 burst GEMM rate (fp16 and bf16
    run at the same dense rate), else the fallback bf16 figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured bf16 burst (fp16 runs at the bf16 rate)"
    return 1590.0, "fallback bf16 burst (fp16 runs at the bf16 rate)"


def chunk_flops(batch, n_q, num_q_heads, ctx):
    """Algorithmic FLOPs of one chunk-attention call: for every (query row, cached
    position) pair, a 128-long score dot product and a 128-long value accumulation, two
    FLOPs per multiply-add (the causal mask's savings on the last n_q positions ignored)."""
    return 4 * 128 * batch * n_q * num_q_heads * ctx


# --------------------------------------------------------------------- byte counts
def group_bytes(qspec):
    return 16 * qspec.bits + 2 * qspec.meta_per_group


def decode_bytes(w, ctx_per_seq):
    """Cache read (codes + meta of K and V) plus q' in and out written."""
    cache = sum(ctx_per_seq) * w.num_kv_heads * 2 * group_bytes(w.quant)
    return cache + w.batch * w.num_q_heads * 128 * (4 + 4)


def append_bytes(w, n_tokens):
    """bf16 K and V read, codes + meta written, T_k read once per KV head."""
    return (w.batch * n_tokens * w.num_kv_heads * (2 * 256 + 2 * group_bytes(w.quant))
            + w.num_kv_heads * 128 * 128 * 4)


def query_bytes(w):
    return w.batch * w.num_q_heads * 128 * (2 + 4) + w.num_kv_heads * 128 * 128 * 4


# ------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [s.strip() for s in line.split(",")]))

    def mark(self):
        return time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t_from=0.0, t_to=float("inf"), window=""):
        rows = [r for t, r in self.rows if t_from <= t <= t_to and len(r) > 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "window": window}
        num = lambda v: v.replace(".", "").isdigit()  # noqa: E731
        sm = [float(r[1]) for r in rows if num(r[1])]
        mx = [float(r[2]) for r in rows if num(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() in ("active", "1")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "window": window}


# ------------------------------------------------------------------- distributed
def dist_setup(n_gpus, backend=None):
    if n_gpus <= 1 and "WORLD_SIZE" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(n_gpus)))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our kernels
def build_history(dq, w, cache, tk, device):
    """Untimed appends of positions 0 .. history-1 (chunks of 4096 tokens)."""
    chunk = 4096
    t = 0
    while t < w.history:
        n = min(chunk, w.history - t)
        k = gen.keys(w, 0, w.batch, t, n, device=device)
        v = gen.values(w, 0, w.batch, t, n, device=device)
        sp = torch.full((w.batch,), t, dtype=torch.int32, device=device)
        dq.quantize_append(cache, k, v, sp, tk)
        t += n
    torch.cuda.synchronize()


def run_ours(args, rank, world, local):
    import decode_attention_quant_b200 as dq
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = QWEN8B_DECODE
    qs = w.quant
    tk_np, tinv_np = gen.transforms(w)
    tk = torch.from_numpy(tk_np).to(device)
    tinv = torch.from_numpy(tinv_np).to(device)
    cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha, qs.rank_lo,
                           qs.rank_hi, device=device)
    build_history(dq, w, cache, tk, device)
    pos = w.history                                        # the step's token goes to position ctx-1
    k_new = gen.keys(w, 0, w.batch, pos, 1, device=device, salt=1)
    v_new = gen.values(w, 0, w.batch, pos, 1, device=device, salt=1)
    q = gen.queries(w, device=device).contiguous()
    start = torch.full((w.batch,), pos, dtype=torch.int32, device=device)
    ctx = torch.full((w.batch,), w.ctx, dtype=torch.int32, device=device)
    q_t = torch.empty(q.shape, dtype=torch.float32, device=device)
    out = torch.empty_like(q_t)
    ws = torch.empty(dq.decode_workspace_bytes(cache, w.num_q_heads), dtype=torch.uint8, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    # The query map does not depend on the append, so it runs on a side stream forked from
    # the step's stream and joined back before the decode: the two small launches overlap.
    side = torch.cuda.Stream(device)

    def one_step(s, ev_i=None):
        side.wait_stream(s)                              # after the previous step's decode
        if ev_i is not None:
            ev_i[2].record(side)
        dq.transform_query(q, tinv, w.num_kv_heads, out=q_t, stream=side)
        if ev_i is not None:
            ev_i[3].record(side)
            ev_i[0].record(s)
        dq.quantize_append(cache, k_new, v_new, start, tk, status, stream=s)
        if ev_i is not None:
            ev_i[1].record(s)
        s.wait_stream(side)
        if ev_i is not None:
            ev_i[4].record(s)
        dq.decode_attention(cache, q_t, ctx, TAU, out=out, workspace=ws, status=status, stream=s)
        if ev_i is not None:
            ev_i[5].record(s)

    def step():
        one_step(torch.cuda.current_stream(device))

    launches_per_step = APPEND_LAUNCHES + QUERY_LAUNCHES + DECODE_LAUNCHES
    clk = ClockSampler(local).__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # untimed soak so that the clock sampler (100 ms period) sees the GPU under this load
    soak_from = time.time()
    while time.time() - soak_from < 1.0:
        for _ in range(20):
            step()
        torch.cuda.synchronize()

    # external: when captured into a graph, the records stay timestamped event nodes
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)] for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True, external=True)
    t1 = torch.cuda.Event(enable_timing=True, external=True)

    def steps(s, per_launch):
        for i in range(args.steps):
            one_step(s, ev[i] if per_launch else None)

    def timed_steps(s):
        t0.record(s)
        steps(s, False)
        t1.record(s)

    # The K timed steps are captured once into a CUDA graph (the library's calls allocate
    # and synchronise nothing) and replayed once, so the host's per-call Python overhead
    # cannot leave the device idle between launches; eager launches if capture fails.  A
    # second graph of the same steps with an event around every launch gives the per-call
    # times (decode roofline, step breakdown) without adding event records to the timed one.
    graph = graph_ev = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                timed_steps(torch.cuda.current_stream())
            graph_ev = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_ev):
                steps(torch.cuda.current_stream(), True)
        except Exception as exc:  # noqa: BLE001 - report and time the eager loop instead
            print(f"graph capture failed ({exc}); timing eager launches", file=sys.stderr)
            graph = graph_ev = None
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed_steps")           # lets a profiler select these launches
    if graph is not None:
        graph.replay()
    else:
        timed_steps(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    timed_to = time.time()
    clk.__exit__(None, None, None)
    ms_total = max_over_ranks(t0.elapsed_time(t1), world)
    if graph_ev is not None:                            # per-call times, outside the timed region
        graph_ev.replay()
    else:
        steps(stream, True)
    torch.cuda.synchronize()
    barrier(world)
    ms_step = ms_total / args.steps
    dec_ms = statistics.mean(ev[i][4].elapsed_time(ev[i][5]) for i in range(args.steps))
    breakdown = {name: round(statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)), 5)
                 for j, name in ((0, "append_ms"), (2, "query_map_ms"), (4, "decode_ms"))}
    breakdown["overlap"] = "query map on a side stream, concurrent with the append"
    step_bytes = decode_bytes(w, [w.ctx] * w.batch) + append_bytes(w, 1) + query_bytes(w)
    value = world * step_bytes / (ms_step * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    dec_alg = decode_bytes(w, [w.ctx] * w.batch)
    achieved = dec_alg / (dec_ms * 1e-3) / 1e9

    # end to end through the C ABI with host buffers: new K/V and q in, output out
    h_k = k_new.cpu().pin_memory()
    h_v = v_new.cpu().pin_memory()
    h_q = q.cpu().pin_memory()
    h_out = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    d_k, d_v, d_q = torch.empty_like(k_new), torch.empty_like(v_new), torch.empty_like(q)

    def e2e_step():
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            d_q.copy_(h_q, non_blocking=True)
            dq.transform_query(d_q, tinv, w.num_kv_heads, out=q_t, stream=side)
        d_k.copy_(h_k, non_blocking=True)
        d_v.copy_(h_v, non_blocking=True)
        dq.quantize_append(cache, d_k, d_v, start, tk, status, stream=stream)
        stream.wait_stream(side)
        dq.decode_attention(cache, q_t, ctx, TAU, out=out, workspace=ws, status=status, stream=stream)
        h_out.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    h2d = (k_new.numel() + v_new.numel() + q.numel()) * 2
    d2h = out.numel() * 4

    # sub-benchmarks (all by default; --only picks some, e.g. for a profiler run)
    want = (lambda name: True) if not args.only else (lambda name: name in args.only.split(","))
    skipped = {"skipped": "not selected by --only"}
    # decode over the same rows in a paged cache (256-token pages in shuffled order)
    paged = bench_paged_decode(dq, cache, q_t, ctx, out, args, world) if want("paged") else skipped
    # quantize-append throughput: 2048-token chunk per sequence, QuEST 2-bit
    app = bench_append(dq, device, args, world) if want("append") else skipped
    # causal 16-query chunk attention over the packed cache
    chunk = bench_chunk(dq, device, args, world) if want("chunk") else skipped
    # decode-step append with RoPE fused in front of the transform
    rope_app = bench_rope_append(dq, device, args, world) if want("rope") else skipped
    # decode-step append with structured key transforms
    struct_app = bench_structured_append(dq, device, args, world) if want("structured") else skipped
    # every workload's decode call and the sweep's chunk appends at 3 and 4 bits
    dec_all = bench_decode_workloads(dq, device, args, world) if want("workloads") else skipped
    app_all = ([app] + [bench_append(dq, device, args, world, bits=b) for b in (3, 4)]) if want("append") else skipped
    # the 64-layer Qwen3-32B-shaped stack, one CUDA graph per step
    stack = bench_stack(dq, device, args, world) if want("stack") else skipped
    st = int(status.item())
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8 codes / fp16 meta / fp32 accumulate", "data": "synthetic",
        "config": {"workload": f"{w.name}: 1-token append + query map + split-K decode per step",
                   "batch": w.batch, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
                   "head_dim": 128, "ctx": w.ctx, "quantizer": "percentile-affine 2-bit ranks 2/125",
                   "l2": "inputs larger than L2 (packed cache 302 MB > 126 MB L2)", "parallelism": f"replicas x{world}",
                   "launch": ("one CUDA graph of the timed steps" if graph is not None else "eager launches")
                   + "; per step the query map runs on a side stream beside the append"},
        "step_bytes": step_bytes,
        "step_breakdown": breakdown,
        "roofline": {"bound": "hbm", "kernel": "decode call (split-K decode_tc_kernel + combine)",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": profiled_decode_traffic(),
                     "alg_bytes_per_launch": dec_alg, "launch_ms": round(dec_ms, 5)},
        "append": app,
        "paged_decode": paged,
        "chunk_attention": chunk,
        "append_rope": rope_app,
        "append_structured": struct_app,
        "decode_workloads": dec_all,
        "append_workloads": app_all,
        "stack": stack,
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(soak_from, timed_to, "1 s untimed soak of the same step + the timed steps"),
        "device_status": st,
    }
    return res


def bench_paged_decode(dq, cache, q_t, ctx, out, args, world, page_size=256):
    """The step's decode call over a paged copy of the cache: same rows, pages shuffled."""
    pps = cache.capacity // page_size
    num_pages = cache.batch * pps
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(0)).to(torch.int32)
    bt = perm.view(cache.batch, pps)
    pools = {}
    for name, t in cache.tensors().items():
        # page bt[b, p] holds rows p * page_size .. of sequence b (all KV heads)
        src = t.view(cache.batch, cache.num_kv_heads, pps, page_size, t.shape[-1]).permute(0, 2, 1, 3, 4)
        pool = torch.empty((num_pages, cache.num_kv_heads, page_size, t.shape[-1]), dtype=t.dtype, device=t.device)
        pool[bt.view(-1).long().to(t.device)] = src.reshape(num_pages, cache.num_kv_heads, page_size, t.shape[-1])
        pools[name] = pool
    pc = dq.PackedCache(cache.batch, cache.num_kv_heads, cache.capacity, cache.kind, cache.bits, cache.clip_alpha,
                        cache.rank_lo, cache.rank_hi, tensors=pools, page_size=page_size, num_pages=num_pages,
                        block_table=bt)
    ws = torch.empty(dq.decode_workspace_bytes(pc, q_t.shape[1]), dtype=torch.uint8, device=q_t.device)
    o2 = torch.empty_like(out)
    stream = torch.cuda.current_stream(q_t.device)
    for _ in range(max(3, args.warmup)):
        dq.decode_attention(pc, q_t, ctx, TAU, out=o2, workspace=ws)
    torch.cuda.synchronize()
    # K back-to-back calls between two events: the device queue stays ahead of the host's
    # per-call work (tensor-map encoding, argument marshalling); the cache is > L2
    reps = max(5, args.steps)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        dq.decode_attention(pc, q_t, ctx, TAU, out=o2, workspace=ws)
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / reps, world)
    same = bool(torch.equal(o2, out))
    by = decode_bytes(QWEN8B_DECODE, [cache.capacity] * cache.batch)
    del pools, pc
    return {"page_size": page_size, "ms": round(ms, 5), "GB/s": round(world * by / (ms * 1e-3) / 1e9, 1),
            "frac_of_peak": round(by / (ms * 1e-3) / 1e9 / _peaks()[0], 4), "output_equals_contiguous": same,
            "l2": "inputs larger than L2"}


def bench_chunk(dq, device, args, world):
    """Causal chunk attention (16 queries per sequence over the packed cache) on two
    shapes: a Qwen3-32B-shaped layer at context 8192 (cache above L2) and the last
    chunk of a 2048-token Qwen3-8B-shaped sequence, QuEST 2-bit, L2 flushed before
    each rep.  Bytes: the cache up to ctx read once, queries in and outputs out."""
    n_q = 16
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    peak, _ = _peaks()
    res = []
    for name, batch, hq, hkv, ctx in (("qwen3_32b_layer_b32_ctx8192_chunk16_quest2", 32, 64, 8, 8192),
                                      ("qwen3_8b_b16_ctx2048_chunk16_quest2", 16, 32, 8, 2048)):
        qs = quest(2)
        c = gen.random_cache(batch, hkv, ctx, qs.kind, qs.bits, seed=ctx, device=device)
        cache = dq.PackedCache(batch, hkv, ctx, qs.kind, qs.bits, qs.clip_alpha, tensors=c)
        q = torch.randn(batch, n_q, hq, 128, generator=torch.Generator(device=device).manual_seed(1),
                        device=device)
        ctx_t = torch.full((batch,), ctx, dtype=torch.int32, device=device)
        out = torch.empty_like(q)
        ws = torch.empty(dq.chunk_workspace_bytes(cache, hq, n_q), dtype=torch.uint8, device=device)
        for _ in range(max(3, args.warmup)):
            dq.chunk_attention(cache, q, ctx_t, TAU, out=out, workspace=ws)
        torch.cuda.synchronize()
        times = []
        for _ in range(max(5, args.steps)):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            torch.cuda.nvtx.range_push(f"chunk_attention_{name}")   # lets a profiler select these launches
            a.record(stream)
            dq.chunk_attention(cache, q, ctx_t, TAU, out=out, workspace=ws)
            b.record(stream)
            torch.cuda.nvtx.range_pop()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = max_over_ranks(statistics.median(times), world)
        by = batch * hkv * ctx * 2 * group_bytes(qs) + 2 * q.numel() * 4
        gbs = by / (ms * 1e-3) / 1e9
        fl = chunk_flops(batch, n_q, hq, ctx)
        tpeak, tkind = _f16_tensor_peak()
        tops = fl / (ms * 1e-3) / 1e12
        res.append({"workload": name, "n_q": n_q, "ms": round(ms, 5), "GB/s": round(world * gbs, 1),
                    "frac_of_peak": round(gbs / peak, 4), "alg_bytes": by,
                    "roofline": {"bound": "tensor", "achieved": round(tops, 1), "peak": round(tpeak, 1),
                                 "unit": "TFLOP/s", "frac": round(tops / tpeak, 4), "peak_kind": tkind,
                                 "flops_per_call": fl, "hbm_floor_ms": round(by / (peak * 1e9) * 1e3, 5),
                                 "tensor_floor_ms": round(fl / (tpeak * 1e12) * 1e3, 5),
                                 "mma_flops_per_call": 2 * fl,
                                 "note": "both contractions run as two fp16 MMAs (hi + lo parts of q' and "
                                         "of p * scale), so the MMAs execute twice the algorithmic FLOPs"},
                    "launches_per_call": 2,
                    "queries_per_s": round(world * batch * n_q * hq / (ms * 1e-3), 1),
                    "l2": "flushed (512 MB write) before each rep"})
        del c, cache, q, out, ws
    return res


def device_time_per_call(fn, reps, args, world):
    """Device time (ms) per call of `fn`: `reps` calls captured back to back in one CUDA
    graph and replayed between two events, so that the host's per-call work (argument
    checks, marshalling) cannot leave the device idle between short launches."""
    for _ in range(max(3, args.warmup)):
        fn()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            fn()
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    del graph
    return max_over_ranks(a.elapsed_time(b) / reps, world)


def bench_rope_append(dq, device, args, world):
    """Decode-step append (one token for each of 16 sequences x 8 KV heads, Qwen3-8B
    shapes, affine 2-bit) with RoPE fused in front of the transform, against the same
    append given post-RoPE keys: back-to-back calls between two events (inputs L2-warm)."""
    w = QWEN8B_DECODE
    qs = w.quant
    cap = 4096
    cache = dq.PackedCache(w.batch, w.num_kv_heads, cap, qs.kind, qs.bits, qs.clip_alpha, device=device)
    tk = torch.from_numpy(gen.transforms(w)[0]).to(device)
    table = gen.rope_table(cap, w.rope_theta).to(device)
    sp = torch.arange(w.batch, dtype=torch.int32, device=device) * 200
    k_pre = gen.keys(w, 0, w.batch, sp.tolist(), 1, rope=False, device=device)
    k_post = gen.keys(w, 0, w.batch, sp.tolist(), 1, device=device)
    v = gen.values(w, 0, w.batch, sp.tolist(), 1, device=device)
    reps = max(50, 10 * args.steps)
    fused = device_time_per_call(lambda: dq.quantize_append_rope(cache, k_pre, v, sp, table, tk), reps, args, world)
    plain = device_time_per_call(lambda: dq.quantize_append(cache, k_post, v, sp, tk), reps, args, world)
    return {"workload": f"{w.name}: 1 token x 16 sequences x 8 KV heads", "fused_rope_us": round(fused * 1e3, 2),
            "post_rope_input_us": round(plain * 1e3, 2), "calls": reps,
            "timing": "device time of the calls captured back to back in one CUDA graph",
            "l2": "inputs L2-warm (back-to-back calls)"}


def bench_structured_append(dq, device, args, world):
    """Decode-step append (one token for each of 16 sequences x 8 KV heads, affine 2-bit)
    with a dense, a block-diagonal (b = 32) and a Hadamard-diagonal key transform:
    back-to-back calls between two events (inputs L2-warm).  A failure is reported in
    the returned object, so that the main measurement line still prints."""
    try:
        w = QWEN8B_DECODE
        qs = w.quant
        cap = 4096
        cache = dq.PackedCache(w.batch, w.num_kv_heads, cap, qs.kind, qs.bits, qs.clip_alpha, device=device)
        sp = torch.arange(w.batch, dtype=torch.int32, device=device) * 200
        k = gen.keys(w, 0, w.batch, sp.tolist(), 1, device=device)
        v = gen.values(w, 0, w.batch, sp.tolist(), 1, device=device)
        dense = torch.from_numpy(gen.transforms(w)[0]).to(device)
        g = torch.Generator().manual_seed(5)
        blocks = (torch.randn(w.num_kv_heads, 4, 32, 32, generator=g) / 32 ** 0.5).to(device)
        scales = (torch.rand(w.num_kv_heads, 128, generator=g) * 3.75 + 0.25).to(device)
        reps = max(50, 10 * args.steps)
        t_dense = device_time_per_call(lambda: dq.quantize_append(cache, k, v, sp, dense), reps, args, world)
        t_block = device_time_per_call(
            lambda: dq.quantize_append_structured(cache, k, v, sp, dq.TRANSFORM_BLOCK_DIAG, blocks, block=32),
            reps, args, world)
        t_had = device_time_per_call(
            lambda: dq.quantize_append_structured(cache, k, v, sp, dq.TRANSFORM_HADAMARD_DIAG, scales),
            reps, args, world)
        return {"workload": f"{w.name}: 1 token x 16 sequences x 8 KV heads", "dense_us": round(t_dense * 1e3, 2),
                "block_diag_32_us": round(t_block * 1e3, 2), "hadamard_diag_us": round(t_had * 1e3, 2),
                "calls": reps, "timing": "device time of the calls captured back to back in one CUDA graph",
                "l2": "inputs L2-warm (back-to-back calls)"}
    except Exception as e:  # noqa: BLE001 - reported in the output line
        return {"error": f"{type(e).__name__}: {e}"}


def bench_decode_workloads(dq, device, args, world):
    """One decode call on each workload shape (random packed caches of the full context,
    all larger than L2): K back-to-back calls between two events.  Bytes: the cache's
    codes and meta of K and V up to ctx, plus q' in and the output out."""
    peak, _ = _peaks()
    res = []
    for w in (QWEN8B_DECODE, QWEN8B_SWEEP(2), QWEN8B_SWEEP(3), QWEN8B_SWEEP(4), QWEN8B_LONG, QWEN32B_STACK):
        try:
            qs = w.quant
            c = gen.random_cache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, seed=w.seed, device=device)
            cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha, qs.rank_lo,
                                   qs.rank_hi, tensors=c)
            q = torch.randn(w.batch, w.num_q_heads, 128, generator=torch.Generator(device=device).manual_seed(2),
                            device=device)
            ctx = torch.full((w.batch,), w.ctx, dtype=torch.int32, device=device)
            out = torch.empty_like(q)
            ws = torch.empty(dq.decode_workspace_bytes(cache, w.num_q_heads), dtype=torch.uint8, device=device)
            stream = torch.cuda.current_stream(device)
            for _ in range(max(3, args.warmup)):
                dq.decode_attention(cache, q, ctx, TAU, out=out, workspace=ws)
            torch.cuda.synchronize()
            reps = max(5, args.steps)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                dq.decode_attention(cache, q, ctx, TAU, out=out, workspace=ws)
            b.record(stream)
            torch.cuda.synchronize()
            ms = max_over_ranks(a.elapsed_time(b) / reps, world)
            by = decode_bytes(w, [w.ctx] * w.batch)
            gbs = by / (ms * 1e-3) / 1e9
            res.append({"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads, "ctx": w.ctx,
                        "bits": qs.bits, "quantizer": "quest" if qs.kind == 0 else "affine", "ms": round(ms, 5),
                        "GB/s": round(world * gbs, 1), "frac_of_peak": round(gbs / peak, 4), "alg_bytes": by,
                        "tokens_per_s": round(world * w.batch * w.ctx / (ms * 1e-3), 1),
                        "splits": int(dq.decode_workspace_bytes(cache, w.num_q_heads)
                                      // (w.batch * w.num_q_heads * 132 * 4)),
                        "l2": "cache larger than L2, back-to-back calls"})
            del c, cache, q, out, ws
        except Exception as e:  # noqa: BLE001 - reported in the output line
            res.append({"workload": w.name, "error": f"{type(e).__name__}: {e}"})
    return res


def bench_stack(dq, device, args, world):
    """The Qwen3-32B-shaped 64-layer stack: per layer the append of a 16-token chunk per
    sequence (QuEST 2-bit, own T_k), the query map and decode attention at context 8192,
    all 64 layers captured in one CUDA graph; K replays between two events.  The caches'
    history is random packed data (the kernels' time does not depend on the values)."""
    try:
        w = QWEN32B_STACK
        qs = w.quant
        n = w.append_tokens
        start = torch.full((w.batch,), w.history, dtype=torch.int32, device=device)
        ctx = torch.full((w.batch,), w.ctx, dtype=torch.int32, device=device)
        status = torch.zeros(1, dtype=torch.int32, device=device)
        layers = []
        for layer in range(w.layers):
            tk, tinv = gen.transforms(w, layer)
            c = gen.random_cache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, seed=w.seed + layer, device=device)
            cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha, tensors=c)
            q = gen.queries(w, layer, device=device).contiguous()
            layers.append((cache, gen.keys(w, 0, w.batch, w.history, n, layer=layer, device=device, salt=1),
                           gen.values(w, 0, w.batch, w.history, n, layer=layer, device=device, salt=1),
                           torch.from_numpy(tk).to(device), torch.from_numpy(tinv).to(device), q,
                           torch.empty(q.shape, dtype=torch.float32, device=device),
                           torch.empty(q.shape, dtype=torch.float32, device=device),
                           torch.empty(dq.decode_workspace_bytes(cache, w.num_q_heads), dtype=torch.uint8,
                                       device=device)))

        # one stream: the 16-token appends run the persistent tensor-core kernel on every SM,
        # so a query map beside them only slows the step (measured 6.33 against 6.07 ms)
        def step():
            for cache, k, v, tk, tinv, q, q_t, out, ws in layers:
                dq.quantize_append(cache, k, v, start, tk, status)
                dq.transform_query(q, tinv, w.num_kv_heads, out=q_t)
                dq.decode_attention(cache, q_t, ctx, TAU, out=out, workspace=ws, status=status)

        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream(device)
        reps = max(3, min(args.steps, 10))
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(a.elapsed_time(b) / reps, world)
        del graph
        dec = w.layers * decode_bytes(w, [w.ctx] * w.batch)
        by = dec + w.layers * (append_bytes(w, n) + query_bytes(w))
        peak, _ = _peaks()
        return {"workload": f"{w.name}: per layer 16-token append + query map + decode, 64 layers",
                "ms_per_step": round(ms, 4), "step_bytes": by, "decode_bytes": dec,
                "GB/s": round(world * by / (ms * 1e-3) / 1e9, 1), "frac_of_peak": round(by / (ms * 1e-3) / 1e9 / peak, 4),
                "launches_per_step": w.layers * (APPEND_LAUNCHES + QUERY_LAUNCHES + DECODE_LAUNCHES),
                "ms_at_70pct_of_peak": round(by / (0.7 * peak * 1e9) * 1e3, 4), "replays": reps,
                "device_status": int(status.item()), "launch": "one CUDA graph per step",
                "l2": "caches larger than L2 (142.6 MB per layer)"}
    except Exception as e:  # noqa: BLE001 - reported in the output line
        return {"error": f"{type(e).__name__}: {e}"}


def bench_append(dq, device, args, world, bits=2):
    w = QWEN8B_SWEEP(bits)
    qs = w.quant
    tk = torch.from_numpy(gen.transforms(w)[0]).to(device)
    n = w.append_tokens
    cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha, device=device)
    k = gen.keys(w, 0, w.batch, w.history, n, device=device)
    v = gen.values(w, 0, w.batch, w.history, n, device=device)
    sp = torch.full((w.batch,), w.history, dtype=torch.int32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    for _ in range(max(3, args.warmup)):
        dq.quantize_append(cache, k, v, sp, tk)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    # each rep: an L2 flush, then the chunk between two events (the flush keeps the device
    # busy while the host prepares the call, so no host time falls between the events)
    times = []
    for _ in range(max(5, args.steps)):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("append_chunk")      # lets a profiler select these launches
        a.record(stream)
        dq.quantize_append(cache, k, v, sp, tk)
        b.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    ms = max_over_ranks(statistics.median(times), world)
    by = append_bytes(w, n)
    peak, _ = _peaks()
    gbs = by / (ms * 1e-3) / 1e9
    return {"workload": f"{w.name}: 2048-token chunk x 16 sequences x 8 KV heads", "tokens_per_s":
            round(world * w.batch * n / (ms * 1e-3), 1), "ms": round(ms, 5), "GB/s": round(world * gbs, 1),
            "frac_of_peak": round(gbs / peak, 4), "alg_bytes": by, "l2": "flushed (512 MB write) before each rep"}


# ------------------------------------------------------------------- oracle arm
def oracle_sample(w, pairs, seed=0):
    """Inputs for the oracle on `pairs` (sequence, KV head) pairs of the workload: a
    random packed cache of the full context, the step's new token, queries."""
    c = gen.random_cache(1, pairs, w.ctx, w.quant.kind, w.quant.bits, seed=seed)
    c = {k: v.numpy() for k, v in c.items()}
    for k in ("k_meta", "v_meta"):
        c[k] = c[k].view(np.uint16)
    tk, tinv = gen.transforms(w)
    g = w.group
    k_new = gen.keys(w, 0, 1, w.ctx - 1, 1).float().numpy()[:, :, :1].repeat(pairs, axis=2).astype(np.float64)
    v_new = gen.values(w, 0, 1, w.ctx - 1, 1).float().numpy()[:, :, :1].repeat(pairs, axis=2).astype(np.float64)
    q = np.tile(gen.queries(w).float().numpy()[:1, :g].astype(np.float64), (1, pairs, 1))
    return c, k_new, v_new, q, np.stack([tk[0]] * pairs), np.stack([tinv[0]] * pairs)


def time_oracle(w, pairs, seconds_cap=30.0):
    """One bounded oracle pass: append of 1 token, query map, decode for `pairs` pairs."""
    sys.path.insert(0, ROOT)
    import oracle.wushkv_oracle as orc
    c, k_new, v_new, q, tk, tinv = oracle_sample(w, pairs)
    qs = w.quant
    t0 = time.perf_counter()
    orc.quantize_append(c, k_new, v_new, [w.ctx - 1], qs.kind, qs.bits, qs.clip_alpha, qs.rank_lo, qs.rank_hi,
                        tk=tk.astype(np.float64))
    qt = orc.transform_query(q, tinv.astype(np.float64), pairs)
    orc.decode_attention(c, qt, [w.ctx], TAU, qs.kind, qs.bits, pairs)
    dt = time.perf_counter() - t0
    # the same byte accounting as the GPU step, for the sampled pairs
    frac = pairs / (w.batch * w.num_kv_heads)
    by = frac * (decode_bytes(w, [w.ctx] * w.batch) + append_bytes(w, 1) + query_bytes(w))
    return dt, by


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def cpu_baseline(w, pairs=64):
    dt, by = time_oracle(w, pairs)
    return {"value": round(by / dt / 1e9, 4), "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{pairs} of {w.batch * w.num_kv_heads} (sequence, KV head) pairs at ctx {w.ctx}: "
                      f"1-token append + query map + decode, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = QWEN8B_DECODE
    pairs = 1
    for _ in range(args.warmup):
        time_oracle(w, pairs)
    tot_t = tot_b = 0.0
    for _ in range(args.steps):
        dt, by = time_oracle(w, pairs)
        tot_t += dt
        tot_b += by
    val = tot_b / tot_t / 1e9
    ms = tot_t / args.steps * 1e3
    cb = {"value": round(val, 4), "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
          "sample": f"each step: {pairs} of {w.batch * w.num_kv_heads} (sequence, KV head) pairs at ctx {w.ctx}"}
    return {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name}: 1-token append + query map + split-K decode per step (sampled)",
                       "batch": w.batch, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
                       "ctx": w.ctx},
            "cpu_baseline": cb, "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of a captured graph")
    ap.add_argument("--only", default="", help="comma list of sub-benchmarks to run besides the main step "
                    "(paged, append, chunk, rope, structured, workloads, stack); default: all")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            res = run_ours(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(QWEN8B_DECODE)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
