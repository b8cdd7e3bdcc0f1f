"""Benchmark: decode KV-read bandwidth (and causal prefill TFLOPS) of the GQA library on B200.

Default workload (``decode_8k``): B=8, h_q=32, d_h=128, T=8192, swept over h_kv in {32, 8, 1}
(MHA / GQA / MQA). One step = for each variant, one ``kv_append`` of the new token's K/V at
position 8191 followed by one ``gqa_decode`` over the 8192 cached keys. ``value`` is the KV bytes
the decodes must read (2 * B * h_kv * T * d_h * 2 per variant) divided by the device time of the
whole step, in GB/s. L2 is flushed (a 256 MiB write, then a 256 MiB read) between steps, outside
the timed events.

A ``paged`` object repeats the decode_8k step over a paged cache (16-token pages in a shuffled
pool: ``kv_append_paged`` + ``gqa_decode_paged``), timed the same way; a ``window`` object runs
decode_8k and prefill_4k with a 1024-key sliding window (work counted inside the window only); a
``backward`` object times gqa_prefill_backward on prefill_4k; an ``mla`` object times gqa_mla_decode
over a latent cache; a ``ragged`` object times gqa_decode on ragged_decode (64 sequences with
seeded lengths on [1024, 32768]); a ``chunked`` object times the chunked prefill (512 new queries
over 32768 keys) and its kv_append.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload.
Run with no flags for N=1; under torchrun every rank runs an independent replica (the path needs
no exchange between GPUs) and rank 0 prints one JSON line with the max-over-ranks time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GQA decode KV-read GB/s vs HBM peak; causal prefill TFLOPS vs bf16 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def decode_kv_bytes(B, h_kv, lengths, d_h, s=2):
    """Algorithmic KV bytes one decode reads: 2 * h_kv * len * d_h * s per sequence."""
    return sum(2 * h_kv * int(n) * d_h * s for n in lengths)


def prefill_flops(B, h_q, d_h, S_q, q_start, kv_len, window=0):
    """Algorithmic causal prefill FLOPs: 4 * d_h per visible (query, key) pair per head (with a
    sliding window of W, row at position p sees keys max(0, p - W + 1) .. p)."""
    pairs = 0
    for i in range(S_q):
        p = q_start + i
        hi = min(kv_len, p + 1)
        lo = max(0, p - window + 1) if window else 0
        pairs += max(0, hi - lo)
    return 4 * d_h * B * h_q * pairs


def _code_only(text):
    """Source with // and /* */ comments and trailing blanks removed, so that a comment edit does
    not count as a kernel change (string literals in these files hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_digest(paths):
    """Digest of the kernel sources' code (comments ignored) at the time the counters were taken."""
    h = hashlib.sha256()
    for p in sorted(paths):
        h.update(_code_only(open(os.path.join(ROOT, p), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(summary_name, digest):
    """DRAM bytes per launch recorded in profiles/<summary_name> for the kernel source `digest`,
    or None when absent or taken on a different version of the kernel."""
    p = os.path.join(ROOT, "profiles", summary_name)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"kernel_source_digest:\s*([0-9a-f]+)", text)
    if not m or m.group(1) != digest:
        return None
    out = {}
    for key, val in re.findall(r"traffic_bytes_per_launch\[([^\]]+)\]:\s*([0-9]+)", text):
        out[key] = int(val)
    for key, val in re.findall(r"algorithmic_bytes\[([^\]]+)\]:\s*([0-9]+)", text):
        out["algorithmic:" + key] = int(val)
    return out or None


DECODE_SOURCES = ["kv_cache_attention_gqa_b200/csrc/decode.cu", "kv_cache_attention_gqa_b200/csrc/common.cuh"]
PREFILL_SOURCES = ["kv_cache_attention_gqa_b200/csrc/prefill_sm100.cu", "kv_cache_attention_gqa_b200/csrc/common.cuh",
                   "kv_cache_attention_gqa_b200/csrc/tcgen05.cuh"]


def scaled_traffic(summary_name, sources, key, algorithmic_bytes):
    """DRAM bytes per launch from an ncu summary taken on a (possibly smaller) case of the same
    kernel, scaled to `algorithmic_bytes` by the captured case's traffic / algorithmic ratio; None
    when absent or captured on a different version of the kernel."""
    rec = recorded_traffic(summary_name, source_digest(sources))
    if not rec or key not in rec or ("algorithmic:" + key) not in rec:
        return None
    return round(rec[key] * algorithmic_bytes / rec["algorithmic:" + key])


class L2Flush:
    """Evict L2 between timed steps: write a 256 MiB buffer (twice the 126 MB L2), then read a
    second one, so the dirty lines of the write are written back here and not during the next
    timed kernel. Both run outside the timed events."""

    def __init__(self, dev):
        import torch

        self.a = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.b = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self, i):
        self.a.fill_(i & 0xFF)
        self.b.sum()


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, p in rows:
            for nm, v in zip(names, p[5:9]):
                if v.lower() in ("active", "1"):
                    reasons.add(nm)
        busy = [r[0] for r in rows if r[0] > 0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


def decode_config(world, launch="cuda_graph"):
    """The `config` object of the decode_8k line (shared by both arms)."""
    return {"workload": "decode_8k: B=8, h_q=32, d_h=128, T=8192, h_kv in {32,8,1}; per step and variant one "
                        "kv_append (1 token at position 8191) + one gqa_decode over 8192 keys",
            "B": 8, "h_q": 32, "d_h": 128, "T": 8192, "h_kv": [32, 8, 1],
            "l2": "flushed between steps (256 MiB write then 256 MiB read, outside the timed events)",
            "launch": launch, "parallelism": f"replicas x{world} (no exchange)"}


def max_over_ranks(x, dist, device):
    """The largest value of `x` over all ranks (the job's time is its slowest replica's)."""
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(unit_per_step, steps, world, total_ms):
    """Whole-job rate: the units all ranks processed divided by the (max-over-ranks) time."""
    return unit_per_step * steps * world / (total_ms / 1e3)


# ---------------------------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------------------------

def build_variants(args, rank, dev, page_size=0, window=0):
    """decode_8k inputs per h_kv: contiguous caches, or (page_size > 0) K/V pools of that page
    size with a shuffled block table, plus the new token's K/V appended at position T-1."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    variants = []
    for h_kv in args.h_kv:
        shape = workloads.DECODE_8K[h_kv]
        bt = None
        if page_size:
            q, k, v, bt, kv_len = workloads.paged_decode_inputs(shape, page_size, seed=args.seed + rank,
                                                                device=dev)
        else:
            q, k, v, kv_len = workloads.decode_inputs(shape, seed=args.seed + rank, device=dev)
        # the new token: its K/V row is appended at position T-1, then the query attends
        g = torch.Generator(device=dev)
        g.manual_seed(10_000 + args.seed + rank + h_kv)
        k_new = torch.randn(shape.B, h_kv, 1, shape.d_h, generator=g, device=dev).to(torch.bfloat16)
        v_new = torch.randn(shape.B, h_kv, 1, shape.d_h, generator=g, device=dev).to(torch.bfloat16)
        pos = (kv_len - 1).contiguous()
        out = torch.empty_like(q)
        ws = torch.zeros(gqa.decode_workspace_size(shape.B, shape.h_q, h_kv, shape.T_max, shape.d_h),
                         dtype=torch.uint8, device=dev)
        n_read = min(window, shape.T_max) if window else shape.T_max  # keys each query reads
        variants.append(dict(h_kv=h_kv, shape=shape, q=q, k=k, v=v, kv_len=kv_len, k_new=k_new,
                             v_new=v_new, pos=pos, out=out, ws=ws, bt=bt, window=window,
                             bytes=decode_kv_bytes(shape.B, h_kv, [n_read] * shape.B, shape.d_h)))
    return variants


def decode_step(variants):
    """One decode step per variant: kv_append of the new token, then gqa_decode (paged variants
    use kv_append_paged / gqa_decode_paged). `record[i]` = (start, end) events around decode i."""
    import kv_cache_attention_gqa_b200 as gqa

    def step(record=None):
        for i, var in enumerate(variants):
            if var["bt"] is None:
                gqa.kv_append(var["k"], var["v"], var["k_new"], var["v_new"], var["pos"])
            else:
                gqa.kv_append_paged(var["k"], var["v"], var["k_new"], var["v_new"], var["pos"], var["bt"])
            if record is not None:
                record[i][0].record()
            if var["bt"] is None:
                gqa.decode(var["q"], var["k"], var["v"], kv_len=var["kv_len"], out=var["out"], ws=var["ws"],
                           window=var["window"])
            else:
                gqa.decode_paged(var["q"], var["k"], var["v"], var["bt"], kv_len=var["kv_len"],
                                 out=var["out"], ws=var["ws"], window=var["window"])
            if record is not None:
                record[i][1].record()
    return step


def time_decode(args, variants, flush, stream, local, dist, dev):
    """Warm up, capture the step in a CUDA graph, then time `args.steps` replays, each after an L2
    flush outside the events. Returns the max-over-ranks total, per-step per-variant decode times
    (ms), the launch mode, clocks and wall time.

    Two graphs of the same step are timed, one after the other. The step graph holds only the
    library's launches (appends, decodes, merges): each decode is a programmatic dependent of the
    append before it, so its launch and prologue overlap the append, and the step's events sit
    outside the graph; this gives the step time. The instrumented graph adds an event node before
    and after each decode (which serialises the decode behind the append again); its replays give
    each decode's own duration for the per-variant rates and the roofline object."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa

    step = decode_step(variants)
    for _ in range(args.warmup):
        flush(1)
        step()
    torch.cuda.synchronize()
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    E = lambda **kw: torch.cuda.Event(enable_timing=True, **kw)  # noqa: E731
    inner = [(E(external=True), E(external=True)) for _ in variants]
    graph = graph_ev = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            graph_ev = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_ev):
                step(inner)
            graph.replay()
            graph_ev.replay()
            torch.cuda.synchronize()
            inner[0][0].elapsed_time(inner[0][1])
        except Exception as exc:  # pragma: no cover - depends on the driver/runtime
            print(f"graph capture unavailable ({exc}); timing eager launches", file=sys.stderr)
            graph = graph_ev = None
            torch.cuda.synchronize()
    mode = "cuda_graph" if graph is not None else "eager"

    def replay(g, rec):
        if g is not None:
            g.replay()
        else:
            step(rec)

    step_ev = [(E(), E()) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    t0 = time.perf_counter()
    for s in range(args.steps):
        flush(s)  # evict the caches from L2 (outside the step's events)
        step_ev[s][0].record(stream)
        replay(graph, None)
        step_ev[s][1].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    # the instrumented replays: one decode's duration per variant and step
    dec_ms = []
    for s in range(args.steps):
        flush(s)
        replay(graph_ev, inner)
        torch.cuda.synchronize()
        dec_ms.append([a.elapsed_time(b) for a, b in inner])
    clocks = sampler.stop()
    if dist is not None:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    del graph, graph_ev
    return {"total_ms": total_ms, "dec_ms": dec_ms, "mode": mode, "clocks": clocks, "wall": wall}


def per_variant_rates(variants, dec_ms, hbm_peak):
    out = {}
    for i, var in enumerate(variants):
        ms = statistics.mean(row[i] for row in dec_ms)
        out[f"h_kv={var['h_kv']}"] = {"decode_us": round(ms * 1e3, 2), "kv_bytes": var["bytes"],
                                      "GB_s": round(var["bytes"] / (ms / 1e3) / 1e9, 1),
                                      "frac_of_hbm_peak": round(var["bytes"] / (ms / 1e3) / 1e9 / hbm_peak, 4)}
    return out


def run_paged(args, rank, dev, stream, local, hbm_peak, peak_kind):
    """decode_8k over a paged cache (16-token pages, shuffled pool): same metric, on one rank."""
    page = args.page_size
    variants = build_variants(args, rank, dev, page_size=page)
    t = time_decode(args, variants, L2Flush(dev), stream, local, None, dev)
    step_bytes = sum(var["bytes"] for var in variants)
    dec_total_ms = sum(sum(row) for row in t["dec_ms"]) / args.steps
    achieved = step_bytes / (dec_total_ms / 1e3) / 1e9
    return {"workload": f"decode_8k over a paged cache: {page}-token pages in a shuffled pool (3 spare "
                        "pages), block table per sequence; per step and variant one kv_append_paged + "
                        "one gqa_decode_paged",
            "page_size": page, "launch": t["mode"],
            "value": round(step_bytes * args.steps / (t["total_ms"] / 1e3) / 1e9, 1), "unit": "GB/s",
            "decode_GB_s": round(achieved, 1), "frac_of_hbm_peak": round(achieved / hbm_peak, 4),
            "peak_kind": f"hbm_gbs of {peak_kind}",
            "per_variant": per_variant_rates(variants, t["dec_ms"], hbm_peak),
            "clocks": t["clocks"]}


def run_backward(args, dev, stream, tf_peak, peak_kind):
    """Backward pass of prefill_4k (B=1, h_q=32, h_kv=8, S=T=4096, d_h=128, causal): dQ, dK, dV from
    the forward's O and lse. Algorithmic work: five GEMMs per visible (query, key) pair (S, dP, dV,
    dK, dQ), 10 * d_h FLOPs, i.e. 2.5 times the forward's."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    shape = workloads.PREFILL_4K
    q, k, v = workloads.prefill_inputs(shape, seed=args.seed, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(20_000 + args.seed)
    d_o = torch.randn(q.shape, generator=g, device=dev).to(torch.bfloat16)
    o, lse = gqa.prefill(q, k, v, return_lse=True)
    ws = torch.empty(2 * 32 * 4096 * 4 + 1024, dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    for _ in range(max(3, args.warmup)):
        gqa.prefill_backward(q, k, v, o, d_o, lse, ws=ws)
    torch.cuda.synchronize()
    n = max(5, args.steps)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush(i)
        evs[i][0].record(stream)
        gqa.prefill_backward(q, k, v, o, d_o, lse, ws=ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error in the backward line")
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    flops = prefill_flops(1, 32, 128, 4096, 0, 4096) * 5 // 2
    tflops = flops / (ms / 1e3) / 1e12
    return {"workload": "prefill_4k backward: dQ, dK, dV (B=1, h_q=32, h_kv=8, S_q=T=4096, d_h=128, causal)",
            "value": round(tflops, 1), "unit": "TFLOP/s", "ms": round(ms, 4),
            "launches": "rowterm + one grid of dK/dV and dQ CTAs (two kernels), eager, L2 flushed between runs",
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(tflops / tf_peak, 4), "peak_kind": f"bf16_tflops of {peak_kind}",
                         "algorithmic_flops_per_launch": flops}}


def graph_timed(fn, flush, steps, warmup):
    """Mean device time (ms) of `fn` captured once in a CUDA graph and replayed `steps` times, each
    replay after an L2 flush outside the events (eager launches if capture fails)."""
    import torch

    for _ in range(warmup):
        flush(1)
        fn()
    torch.cuda.synchronize()
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        graph.replay()
        torch.cuda.synchronize()
    except Exception:  # pragma: no cover - depends on the driver/runtime
        graph = None
        torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush(i)
        evs[i][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    mode = "cuda_graph" if graph is not None else "eager"
    del graph
    return statistics.mean(a.elapsed_time(b) for a, b in evs), mode


def run_mla(args, dev, hbm_peak, tf_peak, peak_kind):
    """MLA decode over a latent cache [第 09 章 §09.3]: B=8, T=8192, rows of 576 (latent 512 +
    rotary 64), 16 and 128 query heads. Algorithmic bytes: the cache rows once per call
    (B * T * 576 * 2); FLOPs: 2 * B * h_q * T * (576 + 512)."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    flush = L2Flush(dev)
    out = {}
    for h_q in (16, 128):
        shape = workloads.MLA_DECODE[h_q]
        q, cache, kl = workloads.mla_decode_inputs(shape, seed=args.seed, device=dev, nan_tail=False)
        o = torch.empty((shape.B, h_q, shape.d_v), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(gqa._lib._lib.gqa_mla_decode_workspace_size(shape.B, h_q, shape.T_max, shape.d_v, 0, 0),
                         dtype=torch.uint8, device=dev)
        fn = lambda: gqa.mla_decode(q, cache, kv_len=kl, scale=shape.scale, out=o, ws=ws)  # noqa: E731
        ms, mode = graph_timed(fn, flush, max(5, args.steps), max(3, args.warmup))
        if gqa.get_device_error() != 0:
            raise RuntimeError("device error in the MLA line")
        nbytes = shape.B * shape.T_max * shape.d_qk * 2
        flops = 2 * shape.B * h_q * shape.T_max * (shape.d_qk + shape.d_v)
        out[f"h_q={h_q}"] = {"decode_us": round(ms * 1e3, 2), "cache_bytes": nbytes,
                             "GB_s": round(nbytes / (ms / 1e3) / 1e9, 1),
                             "frac_of_hbm_peak": round(nbytes / (ms / 1e3) / 1e9 / hbm_peak, 4),
                             "TFLOP_s": round(flops / (ms / 1e3) / 1e12, 1), "launch": mode}
        del q, cache, o, ws
    return {"workload": "MLA decode over a latent cache: B=8, T=8192, rows of 576 (latent 512 + rotary 64), "
                        "h_q in {16, 128}, one gqa_mla_decode per variant",
            "peak_kind": f"hbm_gbs / bf16_tflops of {peak_kind}", "hbm_peak": hbm_peak, "tensor_peak": tf_peak,
            "per_variant": out, "gpu_launches_per_call": 2}


def run_ragged(args, dev, hbm_peak, peak_kind):
    """ragged_decode: B=64, h_q=64, h_kv=8, d_h=128, cached lengths uniform on [1024, 32768]
    (seeded), cache allocated at 32768 with NaN past each length. One gqa_decode per call; the
    algorithmic bytes are the visible K/V rows only (2 * h_kv * d_h * 2 bytes per key)."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    import dataclasses

    shape = workloads.RAGGED_DECODE
    if args.ragged_b != shape.B:  # profiling aid: fewer sequences of the same length distribution
        shape = dataclasses.replace(shape, B=args.ragged_b)
    q, k, v, kv_len = workloads.decode_inputs(shape, seed=args.seed, device=dev)
    out = torch.empty_like(q)
    ws = torch.zeros(gqa.decode_workspace_size(shape.B, shape.h_q, shape.h_kv, shape.T_max, shape.d_h),
                     dtype=torch.uint8, device=dev)
    fn = lambda: gqa.decode(q, k, v, kv_len=kv_len, out=out, ws=ws)  # noqa: E731
    ms, mode = graph_timed(fn, L2Flush(dev), max(5, args.steps), max(3, args.warmup))
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error in the ragged decode line")
    lens = kv_len.cpu().tolist()
    nbytes = decode_kv_bytes(shape.B, shape.h_kv, lens, shape.d_h)
    gbs = nbytes / (ms / 1e3) / 1e9
    finite = bool(torch.isfinite(out.float()).all())  # the NaN past every length never reaches O
    del q, k, v, out, ws
    return {"workload": f"ragged_decode: B={shape.B}, h_q=64, h_kv=8, d_h=128, lengths uniform on [1024, 32768] "
                        f"(seed {args.seed}, sum {sum(lens)}), cache allocated at 32768 with NaN past each length; "
                        "one gqa_decode per call, L2 flushed between calls",
            "launch": mode, "value": round(gbs, 1), "unit": "GB/s", "us": round(ms * 1e3, 2),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4), "peak_kind": f"hbm_gbs of {peak_kind}",
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": scaled_traffic("decode_ragged_decode_b16.md", DECODE_SOURCES, "ragged_b16", nbytes),
                         "traffic_note": "ncu DRAM read + write of 16 sequences of the same length distribution, "
                                         "scaled by algorithmic bytes"},
            "output_finite": finite, "gpu_launches_per_call": 2}


def run_chunked(args, dev, tf_peak, peak_kind):
    """chunked prefill: 32256 cached positions plus 512 new queries at positions 32256..32767
    (B=1, h_q=32, h_kv=8, d_h=128). kv_append writes the new K/V rows first; the attention and the
    append are timed separately."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    shape = workloads.CHUNKED_PREFILL
    k, v, k_new, v_new, q = workloads.chunked_prefill_inputs(shape, seed=args.seed, device=dev)
    pos = torch.full((shape.B,), shape.q_start, dtype=torch.int32, device=dev)
    kl = torch.full((shape.B,), shape.kv_len, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    flush = L2Flush(dev)
    app = lambda: gqa.kv_append(k, v, k_new, v_new, pos)  # noqa: E731
    att = lambda: gqa.prefill(q, k, v, q_start=pos, kv_len=kl, out=out)  # noqa: E731
    app_ms, _ = graph_timed(app, flush, max(5, args.steps), max(3, args.warmup))
    ms, mode = graph_timed(att, flush, max(5, args.steps), max(3, args.warmup))
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error in the chunked prefill line")
    flops = prefill_flops(shape.B, shape.h_q, shape.d_h, shape.S_q, shape.q_start, shape.kv_len)
    tflops = flops / (ms / 1e3) / 1e12
    app_bytes = 2 * 2 * k_new.nbytes  # K and V rows read once and written once
    del k, v, k_new, v_new, q, out
    return {"workload": "chunked prefill: B=1, h_q=32, h_kv=8, d_h=128, 32256 cached + 512 new queries at "
                        "positions 32256..32767, T=32768, causal by absolute position; L2 flushed between calls",
            "launch": mode, "value": round(tflops, 1), "unit": "TFLOP/s", "ms": round(ms, 4),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(tflops / tf_peak, 4), "peak_kind": f"bf16_tflops of {peak_kind}",
                         "algorithmic_flops_per_launch": flops,
                         "traffic": scaled_traffic("prefill_chunked_prefill.md", PREFILL_SOURCES, "chunked",
                                                   138412032),
                         "traffic_note": "ncu DRAM read + write of one launch (K/V + Q: 138,412,032 B)"},
            "kv_append": {"us": round(app_ms * 1e3, 2), "bytes": app_bytes,
                          "GB_s": round(app_bytes / (app_ms / 1e3) / 1e9, 1)}}


def run_prefill_small(args, dev, tf_peak, peak_kind):
    """prefill_small: B=1, h_q=4, h_kv=2 (r=2), S_q=T=256, d_h=64, causal, N(0,1) -- the d_h=64
    tcgen05 instantiation. 33.7 MFLOP of work is a few microseconds of one launch on 8 CTAs: the
    line is launch- and latency-bound, so its TFLOPS is reported, not held to the tensor peak."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    shape = workloads.PREFILL_SMALL
    q, k, v = workloads.prefill_inputs(shape, seed=args.seed, device=dev)
    out = torch.empty_like(q)
    fn = lambda: gqa.prefill(q, k, v, out=out)  # noqa: E731
    ms, mode = graph_timed(fn, L2Flush(dev), max(20, args.steps), max(3, args.warmup))
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error in the prefill_small line")
    flops = prefill_flops(shape.B, shape.h_q, shape.d_h, shape.S_q, 0, shape.T_max)
    tflops = flops / (ms / 1e3) / 1e12
    return {"workload": "prefill_small: B=1, h_q=4, h_kv=2, S_q=T=256, d_h=64, causal; one gqa_prefill per call, "
                        "L2 flushed between calls",
            "launch": mode, "value": round(tflops, 2), "unit": "TFLOP/s", "us": round(ms * 1e3, 2),
            "bound": "launch/latency (8 tiles of 128 rows on 148 SMs)",
            "frac_of_bf16_peak": round(tflops / tf_peak, 5), "peak_kind": f"bf16_tflops of {peak_kind}",
            "algorithmic_flops_per_launch": flops, "gpu_launches_per_call": 1}


def run_window(args, rank, dev, stream, local, hbm_peak, tf_peak, peak_kind):
    """Sliding window of 1024 keys [第三章 §3.7]: decode_8k (each query reads its 1024 most recent
    keys) and prefill_4k; the work counted is only what lies inside the windows."""
    W = args.window
    variants = build_variants(args, rank, dev, window=W)
    t = time_decode(args, variants, L2Flush(dev), stream, local, None, dev)
    step_bytes = sum(var["bytes"] for var in variants)
    dec_total_ms = sum(sum(row) for row in t["dec_ms"]) / args.steps
    achieved = step_bytes / (dec_total_ms / 1e3) / 1e9
    per_variant = per_variant_rates(variants, t["dec_ms"], hbm_peak)
    del variants
    return {"window": W,
            "decode": {"workload": f"decode_8k with a {W}-key sliding window: per step and variant one "
                                   "kv_append + one gqa_decode reading the window's keys", "launch": t["mode"],
                       "value": round(step_bytes * args.steps / (t["total_ms"] / 1e3) / 1e9, 1), "unit": "GB/s",
                       "decode_GB_s": round(achieved, 1), "frac_of_hbm_peak": round(achieved / hbm_peak, 4),
                       "peak_kind": f"hbm_gbs of {peak_kind}", "per_variant": per_variant,
                       "gpu_launches": args.steps * 3 * len(args.h_kv)},
            "prefill": run_prefill(args, dev, stream, tf_peak, peak_kind, window=W)}


def run_ours(args, rank, world, dist):
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hbm_peak, tf_peak, tf_sust, peak_kind = load_peaks()
    if args.prefill_only:  # profiling aid: the prefill_4k line alone
        return {"prefill": run_prefill(args, dev, stream, tf_peak, peak_kind)}
    if args.paged_only:  # profiling aid: the paged decode_8k line alone
        return {"paged": run_paged(args, rank, dev, stream, local, hbm_peak, peak_kind)}
    if args.mla_only:  # profiling aid: the MLA line alone
        return {"mla": run_mla(args, dev, hbm_peak, tf_peak, peak_kind)}
    if args.backward_only:  # profiling aid: the backward line alone
        return {"backward": run_backward(args, dev, stream, tf_peak, peak_kind)}
    if args.window_only:  # profiling aid: the sliding-window lines alone
        return {"window": run_window(args, rank, dev, stream, local, hbm_peak, tf_peak, peak_kind)}
    if args.ragged_only:  # profiling aid: the ragged decode line alone
        return {"ragged": run_ragged(args, dev, hbm_peak, peak_kind)}
    if args.chunked_only:  # profiling aid: the chunked prefill line alone
        return {"chunked": run_chunked(args, dev, tf_peak, peak_kind)}
    if args.small_only:  # profiling aid: the prefill_small line alone
        return {"prefill_small": run_prefill_small(args, dev, tf_peak, peak_kind)}

    variants = build_variants(args, rank, dev)
    flush = L2Flush(dev)
    t = time_decode(args, variants, flush, stream, local, dist, dev)
    total_ms, dec_ms, mode, clocks, wall = t["total_ms"], t["dec_ms"], t["mode"], t["clocks"], t["wall"]

    step_bytes = sum(var["bytes"] for var in variants)
    value = job_throughput(step_bytes, args.steps, world, total_ms) / 1e9
    per_variant = per_variant_rates(variants, dec_ms, hbm_peak)
    dec_total_ms = sum(sum(row) for row in dec_ms) / args.steps
    achieved = step_bytes / (dec_total_ms / 1e3) / 1e9
    digest = source_digest(DECODE_SOURCES)
    traffic = recorded_traffic("decode_splitkv_decode_8k.md", digest)
    traffic_per_launch = None
    if traffic and all(f"h_kv={v['h_kv']}" in traffic for v in variants):
        traffic_per_launch = round(sum(traffic[f"h_kv={v['h_kv']}"] for v in variants) / len(variants))
    roofline = {"bound": "hbm", "kernel": "decode_bf16_kernel + merge_kernel (events bracket both launches of one gqa_decode, "
                          "in the instrumented replays of the step)",
                "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "peak_kind": f"hbm_gbs of {peak_kind}",
                "traffic": traffic_per_launch,
                "algorithmic_bytes_per_launch": round(step_bytes / len(variants)),
                "kernel_source_digest": digest}

    e2e = run_e2e(args, variants, dev, stream, dist, world) if not args.skip_e2e else None
    prefill = run_prefill(args, dev, stream, tf_peak, peak_kind) if not args.skip_prefill else None
    n_variants = len(variants)
    del variants
    paged = None
    if not args.skip_paged:
        paged = run_paged(args, rank, dev, stream, local, hbm_peak, peak_kind)
        paged["gpu_launches"] = args.steps * 3 * len(args.h_kv)
    backward = run_backward(args, dev, stream, tf_peak, peak_kind) if not args.skip_backward else None
    mla = run_mla(args, dev, hbm_peak, tf_peak, peak_kind) if not args.skip_mla else None
    window = None
    if not args.skip_window:
        window = run_window(args, rank, dev, stream, local, hbm_peak, tf_peak, peak_kind)
    ragged = run_ragged(args, dev, hbm_peak, peak_kind) if not args.skip_ragged else None
    chunked = run_chunked(args, dev, tf_peak, peak_kind) if not args.skip_chunked else None
    small = run_prefill_small(args, dev, tf_peak, peak_kind) if not args.skip_small else None

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 (no dataset)",
        "config": decode_config(world, mode),
        "roofline": roofline,
        "per_variant": per_variant,
        "gpu_launches": args.steps * 3 * n_variants,  # kv_append, decode, merge per variant
        "clocks": clocks,
        "e2e": e2e,
        "wall_s_timed_region": round(wall, 3),
    }
    if prefill is not None:
        result["prefill"] = prefill
    if paged is not None:
        result["paged"] = paged
    if window is not None:
        result["window"] = window
    if backward is not None:
        result["backward"] = backward
    if mla is not None:
        result["mla"] = mla
    if ragged is not None:
        result["ragged"] = ragged
    if chunked is not None:
        result["chunked"] = chunked
    if small is not None:
        result["prefill_small"] = small
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
    return result


def run_e2e(args, variants, dev, stream, dist, world):
    """The same step through the public API with host buffers. Per step: one copy of every
    variant's q and new K/V rows from a pinned host staging buffer, then per variant append +
    decode (outputs into one device buffer), then one copy of all outputs back to the host."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa

    align = 256  # each tensor's slice starts on a 256-byte boundary (TMA needs 16)

    def layout(tensors):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.nbytes + align - 1) // align * align
        return offs, n

    ins = [t for var in variants for t in (var["q"], var["k_new"], var["v_new"])]
    outs = [var["out"] for var in variants]
    in_offs, in_n = layout(ins)
    out_offs, out_n = layout(outs)
    host_in = torch.empty(in_n, dtype=torch.uint8).pin_memory()
    host_out = torch.empty(out_n, dtype=torch.uint8).pin_memory()
    dev_in = torch.empty(in_n, dtype=torch.uint8, device=dev)
    dev_out = torch.empty(out_n, dtype=torch.uint8, device=dev)

    def view(buf, off, like):
        return buf[off:off + like.nbytes].view(like.dtype).view(like.shape)

    for t, off in zip(ins, in_offs):
        view(host_in, off, t).copy_(t.cpu())
    dv_in = [view(dev_in, off, t) for t, off in zip(ins, in_offs)]
    dv_out = [view(dev_out, off, t) for t, off in zip(outs, out_offs)]
    h2d = sum(t.nbytes for t in ins)
    d2h = sum(t.nbytes for t in outs)

    def step():
        dev_in.copy_(host_in, non_blocking=True)
        for i, var in enumerate(variants):
            qd, knd, vnd = dv_in[3 * i:3 * i + 3]
            gqa.kv_append(var["k"], var["v"], knd, vnd, var["pos"])
            gqa.decode(qd, var["k"], var["v"], kv_len=var["kv_len"], out=dv_out[i], ws=var["ws"])
        host_out.copy_(dev_out, non_blocking=True)

    flush = L2Flush(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    step_bytes = sum(var["bytes"] for var in variants)

    def timed(run):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for s in range(args.steps):
            flush(s)
            evs[s][0].record(stream)
            run()
            evs[s][1].record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), dist, dev)

    # The step as a serving loop runs it: the same public calls and both copies captured once in a
    # CUDA graph and replayed every step (the copies read and write the pinned host buffers on every
    # replay). The eager launches are timed as well and reported beside it.
    graph = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            graph.replay()
            torch.cuda.synchronize()
        except Exception:  # pragma: no cover - depends on the driver/runtime
            graph = None
            torch.cuda.synchronize()
    used_graph = graph is not None
    total_eager = timed(step)
    total = timed(graph.replay) if used_graph else total_eager
    # the host copies of the outputs equal the graph-timed step's device outputs (same inputs,
    # same plan: the decode is deterministic)
    same = all(torch.equal(view(host_out, off, o), o.cpu()) for o, off in zip(outs, out_offs))
    del graph
    return {"value": round(job_throughput(step_bytes, args.steps, world, total) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(total / args.steps, 4), "copies_per_step": 2,
            "launch": "cuda_graph (public calls and copies captured once)" if used_graph else "eager",
            "eager": {"value": round(job_throughput(step_bytes, args.steps, world, total_eager) / 1e9, 1),
                      "unit": "GB/s", "ms_per_step": round(total_eager / args.steps, 4)},
            "outputs_match_device_step": same}


def run_prefill(args, dev, stream, tf_peak, peak_kind, window=0):
    """Secondary line: causal prefill prefill_4k (B=1, h_q=32, h_kv=8, T=4096, d_h=128), TFLOPS
    (optionally with a sliding window: only the pairs inside the window count as work)."""
    import torch

    import kv_cache_attention_gqa_b200 as gqa
    import workloads

    shape = workloads.PREFILL_4K
    q, k, v = workloads.prefill_inputs(shape, seed=args.seed, device=dev)
    out = torch.empty_like(q)
    try:
        gqa.prefill(q, k, v, out=out, window=window)
    except gqa.GQAError as e:
        return {"unavailable": str(e)}
    flush = L2Flush(dev)
    for _ in range(max(3, args.warmup)):
        gqa.prefill(q, k, v, out=out, window=window)
    torch.cuda.synchronize()
    n = max(5, args.steps)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush(i)
        evs[i][0].record(stream)
        gqa.prefill(q, k, v, out=out, window=window)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if gqa.get_device_error() != 0:
        raise RuntimeError("device error in the prefill line")
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    flops = prefill_flops(1, 32, 128, 4096, 0, 4096, window)
    tflops = flops / (ms / 1e3) / 1e12
    wtxt = f", sliding window {window}" if window else ""
    return {"workload": f"prefill_4k: B=1, h_q=32, h_kv=8, S_q=T=4096, d_h=128, causal{wtxt}",
            "value": round(tflops, 1), "unit": "TFLOP/s", "ms": round(ms, 4),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(tflops / tf_peak, 4), "peak_kind": f"bf16_tflops of {peak_kind}",
                         "algorithmic_flops_per_launch": flops}}


# ---------------------------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------------------------

def _oracle_sample_inputs(seed=0):
    import workloads

    out = []
    for h_kv in (32, 8, 1):
        shape = workloads.DECODE_8K[h_kv]
        small = workloads.DecodeShape(B=1, h_q=shape.h_q, h_kv=h_kv, T_max=shape.T_max, d_h=shape.d_h)
        q, k, v, kv_len = workloads.decode_inputs(small, seed=seed)
        out.append((h_kv, workloads.to_f64(q), workloads.to_f64(k), workloads.to_f64(v), kv_len.numpy()))
    return out


def _threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _time_until(fn, budget_s, max_reps=1000):
    """Run `fn` until about `budget_s` seconds have passed; returns (repetitions, seconds)."""
    reps, t = 0, 0.0
    while (t < budget_s or reps == 0) and reps < max_reps:
        t0 = time.perf_counter()
        fn()
        t += time.perf_counter() - t0
        reps += 1
    return reps, t


def cpu_baseline_per_config(args, budget_s=3.0):
    """The fp64 oracle on a bounded sample of each of the other workloads, at the same seed and
    shapes as the GPU lines: prefill_small whole; prefill_4k one query head (4096 x 4096 pairs);
    chunked prefill one query head (512 queries over 32768 keys); ragged_decode one sequence (the
    first of the seeded lengths, all 64 query heads). Each sample repeats for about `budget_s`."""
    import numpy as np

    import oracle
    import workloads

    f64 = workloads.to_f64
    out = {}
    # C1 prefill_small, whole
    sh = workloads.PREFILL_SMALL
    q, k, v = (f64(t) for t in workloads.prefill_inputs(sh, seed=args.seed))
    reps, t = _time_until(lambda: oracle.attention_ref(q, k, v), budget_s)
    fl = prefill_flops(sh.B, sh.h_q, sh.d_h, sh.S_q, 0, sh.T_max)
    out["prefill_small"] = {"GFLOP_s": round(fl * reps / t / 1e9, 3), "s_per_call": round(t / reps, 5),
                            "sample": "the whole workload (4 heads, 256 rows)", "reps": reps}
    # C3 prefill_4k, one query head
    sh = workloads.PREFILL_4K
    q, k, v = workloads.prefill_inputs(sh, seed=args.seed)
    q0, k0, v0 = f64(q[0, 0]), f64(k[0, 0]), f64(v[0, 0])
    pos = np.arange(sh.S_q)
    reps, t = _time_until(lambda: oracle.head_attention(q0, k0, v0, pos, sh.kv_len, sh.d_h ** -0.5), budget_s)
    fl = prefill_flops(1, 1, sh.d_h, sh.S_q, 0, sh.kv_len)
    out["prefill_4k"] = {"GFLOP_s": round(fl * reps / t / 1e9, 3), "s_per_head": round(t / reps, 4),
                         "sample": "query head 0 of 32 (4096 x 4096 causal pairs)", "reps": reps}
    # C5 chunked prefill, one query head
    sh = workloads.CHUNKED_PREFILL
    k, v, k_new, v_new, q = workloads.chunked_prefill_inputs(sh, seed=args.seed)
    k[:, :, sh.q_start:] = k_new
    v[:, :, sh.q_start:] = v_new
    q0, k0, v0 = f64(q[0, 0]), f64(k[0, 0]), f64(v[0, 0])
    pos = sh.q_start + np.arange(sh.S_q)
    reps, t = _time_until(lambda: oracle.head_attention(q0, k0, v0, pos, sh.kv_len, sh.d_h ** -0.5), budget_s)
    fl = prefill_flops(1, 1, sh.d_h, sh.S_q, sh.q_start, sh.kv_len)
    out["chunked_prefill"] = {"GFLOP_s": round(fl * reps / t / 1e9, 3), "s_per_head": round(t / reps, 4),
                              "sample": "query head 0 of 32 (512 queries over 32768 keys)", "reps": reps}
    # C4 ragged decode, one sequence
    sh = workloads.RAGGED_DECODE
    n0 = int(workloads.ragged_lengths(args.seed, sh.B, sh.len_lo, sh.len_hi)[0])
    one = workloads.DecodeShape(B=1, h_q=sh.h_q, h_kv=sh.h_kv, T_max=n0, d_h=sh.d_h)
    q, k, v, kl = workloads.decode_inputs(one, seed=args.seed)
    q, k, v, kl = f64(q), f64(k), f64(v), kl.numpy()
    reps, t = _time_until(lambda: oracle.decode_ref(q, k, v, kv_len=kl), budget_s)
    nb = decode_kv_bytes(1, sh.h_kv, [n0], sh.d_h)
    out["ragged_decode"] = {"GB_s": round(nb * reps / t / 1e9, 4), "s_per_sequence": round(t / reps, 4),
                            "sample": f"one sequence of length {n0} (the first seeded length), 64 query heads",
                            "reps": reps}
    return out


def cpu_baseline(args, budget_s=10.0):
    """fp64 oracle on a bounded sample of decode_8k: sequence 0 of each h_kv variant, repeated
    until about `budget_s` seconds of CPU work; plus the other workloads' samples."""
    import oracle

    samples = _oracle_sample_inputs(args.seed)
    nbytes, t_total, reps = 0, 0.0, 0
    while t_total < budget_s and reps < 1000:
        for h_kv, q, k, v, kv_len in samples:
            t0 = time.perf_counter()
            oracle.decode_ref(q, k, v, kv_len=kv_len)
            t_total += time.perf_counter() - t0
            nbytes += decode_kv_bytes(1, h_kv, kv_len, 128)
        reps += 1
    res = {"value": round(nbytes / t_total / 1e9, 4), "unit": "GB/s", "cores": _threads(), "kind": "oracle",
           "sample": f"decode_8k, sequence 0 of each h_kv variant (all 32 query heads, 8192 keys), "
                     f"{reps} repetitions, {t_total:.1f} s of fp64 NumPy"}
    if not args.skip_oracle_configs:
        res["per_config"] = cpu_baseline_per_config(args)
    return res


def run_reference(args, rank):
    """The reference arm: the oracle, as it stands, on the host cores; one step = the decode of one
    sequence of each h_kv variant (a bounded sample of decode_8k)."""
    import oracle

    samples = _oracle_sample_inputs(args.seed)
    step_bytes = sum(decode_kv_bytes(1, h_kv, kv_len, 128) for h_kv, _, _, _, kv_len in samples)
    for _ in range(args.warmup):
        for h_kv, q, k, v, kv_len in samples:
            oracle.decode_ref(q, k, v, kv_len=kv_len)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for h_kv, q, k, v, kv_len in samples:
            oracle.decode_ref(q, k, v, kv_len=kv_len)
    dt = time.perf_counter() - t0
    value = step_bytes * args.steps / dt / 1e9
    sample = "decode_8k, sequence 0 of each h_kv variant (32 query heads, 8192 keys) per step, fp64 NumPy"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded N(0,1) bf16 upcast to fp64",
            "config": decode_config(1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--skip-prefill", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-oracle-configs", action="store_true",
                    help="time the oracle on decode_8k only (not on the other workloads' samples)")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of a CUDA graph")
    ap.add_argument("--prefill-only", action="store_true", help="only the prefill_4k line (profiling aid)")
    ap.add_argument("--skip-paged", action="store_true")
    ap.add_argument("--paged-only", action="store_true", help="only the paged decode_8k line (profiling aid)")
    ap.add_argument("--page-size", dest="page_size", type=int, default=16,
                    help="page size of the paged decode_8k line (a multiple of 16)")
    ap.add_argument("--skip-window", action="store_true")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--skip-mla", action="store_true")
    ap.add_argument("--mla-only", action="store_true", help="only the MLA line (profiling aid)")
    ap.add_argument("--backward-only", action="store_true", help="only the backward line (profiling aid)")
    ap.add_argument("--window-only", action="store_true", help="only the sliding-window lines (profiling aid)")
    ap.add_argument("--window", type=int, default=1024, help="sliding window of the window lines")
    ap.add_argument("--skip-ragged", action="store_true")
    ap.add_argument("--ragged-only", action="store_true", help="only the ragged decode line (profiling aid)")
    ap.add_argument("--ragged-b", dest="ragged_b", type=int, default=64,
                    help="sequences of the ragged decode line (profiling aid; the workload has 64)")
    ap.add_argument("--skip-chunked", action="store_true")
    ap.add_argument("--chunked-only", action="store_true", help="only the chunked prefill line (profiling aid)")
    ap.add_argument("--skip-small", action="store_true")
    ap.add_argument("--small-only", action="store_true", help="only the prefill_small line (profiling aid)")
    ap.add_argument("--h-kv", dest="h_kv", type=int, nargs="+", default=[32, 8, 1],
                    help="decode_8k variants to run (default: all three); fewer only for profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank)), flush=True)
        return

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        res = run_ours(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
