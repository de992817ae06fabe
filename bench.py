"""Benchmark of the packed-KV hot path: one step = one full block-by-block decode.

A step appends every block of K/V of every layer into the packed cache
(quantize + bit-pack) and runs each block's packed-KV attention, in decode
order (block-major: for s in blocks, for l in layers). Inputs are seeded
synthetic K/V/Q shaped like the workload, resident in HBM before timing.

Prints ONE JSON line on rank 0. `value` = query tokens x layers decoded per
second (B * N * L per step) over the whole step, max over ranks; per-kernel
numbers (quantize+pack GB/s, attention tokens/s, roofline fractions) are in
the `quant_pack` / `attention` / `roofline` keys.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload var_d30] [--bits 3]
                  [--also infinity_2b|none]   # further workloads, each its own sub-record
  python bench.py --impl reference ...   # the CPU oracle, bounded sample

Each workload also times the same decode through vq_append_attention_block
(`fused`: append and attention in one launch where that is faster).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import WORKLOADS, default_softmax_scale, make_kv, make_q  # noqa: E402

METRIC = "KV quant+pack GB/s; packed-KV attention tokens/s; % of HBM/tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# DRAM bytes per layer of each kernel family, from one ncu capture of layer 0
# (profiles/dram_traffic.json); valid only while the kernels' sources are the
# ones that capture ran.
KERNEL_SOURCES = {
    "attention": ("attention.cuh", "attention_pipe.cuh", "quant_pack.cuh", "tc_ptx.cuh", "vq_device.cuh",
                  "vq_internal.h", "vq_api.cu"),
    "quant_pack": ("quant_pack.cuh", "tc_ptx.cuh", "vq_device.cuh", "vq_internal.h", "vq_api.cu"),
}


def kernel_sources_sha256(family):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[family]:
        with open(os.path.join(ROOT, "bit_kv_cache_25_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload, family, layers):
    """(DRAM bytes per step, note): the captured bytes of one layer times the
    layer count (every layer has the same shapes), or (None, why not)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None, "no capture"
    e = json.load(open(p)).get(workload, {}).get(family)
    if not e:
        return None, "no capture of this workload"
    if e.get("sources_sha256") != kernel_sources_sha256(family):
        return None, "kernel sources changed since the capture"
    return e["bytes_per_layer"] * layers, f"ncu capture of layer 0 ({e['launches_per_layer']} launches) x {layers} layers"


# ------------------------------------------------------------------ algorithmic work
def word_rows(n, bits):
    c = 32 // bits
    return (n + c - 1) // c


def quant_bytes(w, bits, s):
    """Algorithmic HBM bytes of one append (K and V) of block s of one layer."""
    esize = 4 if w.kv_dtype == "f32" else 2
    B, H, D, n = w.batch, w.heads, w.head_dim, w.block_tokens[s]
    per = esize * B * H * n * D + 4 * B * H * word_rows(n, bits) * D + 8 * B * H * D
    return 2 * per


def attn_work(w, bits, s):
    """(flops, bytes) of the attention of block s of one layer (fp32 output)."""
    B, H, D, n = w.batch, w.heads, w.head_dim, w.block_tokens[s]
    P = w.prefix(s) + n
    flops = 4 * B * H * n * P * D
    words = sum(word_rows(w.block_tokens[k], bits) for k in range(s + 1))
    byts = 2 * B * H * n * D + 4 * B * H * n * D + 8 * B * H * D * words + 16 * B * H * D * (s + 1)
    return flops, byts


def workload_config(w, bits):
    """The `config` of both arms' JSON lines: the workload and what the timed
    region reads (inputs larger than L2, so no flush between steps)."""
    esize = 4 if w.kv_dtype == "f32" else 2
    inputs = w.layers * w.batch * w.heads * w.tokens * w.head_dim * (2 * esize + 2)
    return {"workload": w.name, "bits": bits, "layers": w.layers, "heads": w.heads, "head_dim": w.head_dim,
            "batch": w.batch, "blocks": w.num_blocks, "tokens": w.tokens, "kv_dtype": w.kv_dtype,
            "per_rank": "one full decode per step",
            "l2": f"inputs {inputs / 1e9:.1f} GB > L2 (126 MB), no flush",
            "token_unit": "B*N*L query tokens x layers per step (append + attention)"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if world != n_gpus and rank == 0:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE {world}", file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over all ranks (device timings are reduced with MAX)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank_step: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: every rank decodes its own batch (replicas), so the
    job processes world x tokens per step in the slowest rank's step time."""
    return world * tokens_per_rank_step / (ms_per_step_max / 1e3)


# ------------------------------------------------------------------ CPU oracle sample
def oracle_unit(w, bits, layer_kv, q, b, h, sigma):
    """One (b, h) unit of one layer through the oracle: append every block of
    K and V, then every block's attention. Returns seconds."""
    import numpy as np

    import oracle.vq_oracle as vo
    k, v = layer_kv
    t0 = time.perf_counter()
    kh = k[b:b + 1, h:h + 1].float().numpy()
    vh = v[b:b + 1, h:h + 1].float().numpy()
    qh = q[b:b + 1, h:h + 1].float().numpy()
    pk, sk, zk = vo.cache_append(kh, w.block_tokens, bits)
    pv, sv, zv = vo.cache_append(vh, w.block_tokens, bits)
    for s, n in enumerate(w.block_tokens):
        khat = vo.dequantize_cache(pk, sk, zk, w.block_tokens, 1, 1, w.head_dim, bits, s)
        vhat = vo.dequantize_cache(pv, sv, zv, w.block_tokens, 1, 1, w.head_dim, bits, s)
        p0 = w.prefix(s)
        out = vo.attention_f64(qh[:, :, p0:p0 + n], khat, vhat, sigma)
        assert np.isfinite(out).all()
    return time.perf_counter() - t0


def host_cores():
    """CPU cores this process may run on (the host's core count)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_sample(w, bits, budget_s=15.0, max_units=4096):
    """Time the oracle on (b, h) units of layer 0 until ~budget_s; return
    (tokens_per_s scaled to the whole step, units, seconds)."""
    k, v = _small_kv(w)
    q = _small_q(w)
    sigma = default_softmax_scale(w)
    total, units = 0.0, 0
    while units < max_units and (total < budget_s or units == 0):
        b = units % k.shape[0]
        h = (units // k.shape[0]) % w.heads
        total += oracle_unit(w, bits, (k, v), q, b, h, sigma)
        units += 1
    per_unit = total / units
    # one step = B*H*L units; value = B*N*L tokens per step time
    tokens_per_s = w.batch * w.tokens * w.layers / (per_unit * w.batch * w.heads * w.layers)
    return tokens_per_s, units, total


def _small_kv(w):
    """Layer-0 K/V of a batch of at most two (same distribution) for the CPU sample."""
    import dataclasses
    return make_kv(dataclasses.replace(w, batch=min(2, w.batch)), 0, device="cpu")


def _small_q(w):
    import dataclasses
    return make_q(dataclasses.replace(w, batch=min(2, w.batch)), 0, device="cpu")


# ------------------------------------------------------------------ the reference arm (oracle)
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    bits = args.bits or w.bits[0]
    import dataclasses
    wk = dataclasses.replace(w, batch=min(w.batch, 2))
    k, v = make_kv(wk, 0, device="cpu")
    q = make_q(wk, 0, device="cpu")
    sigma = default_softmax_scale(w)
    times = []
    u = 0
    for i in range(args.warmup + args.steps):
        dt = 0.0
        for _ in range(args.ref_units):
            b, h = u % wk.batch, (u // wk.batch) % w.heads
            dt += oracle_unit(w, bits, (k, v), q, b, h, sigma)
            u += 1
        if i >= args.warmup:
            times.append(dt)
    per_unit = sum(times) / len(times) / args.ref_units
    value = w.tokens / (per_unit * w.heads)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_unit * args.ref_units * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, bits),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                         "blas_threads": blas_threads(), "quantize_threads": 1,
                         "sample": f"each step: {args.ref_units} (batch, head) units of layer 0 through the oracle (append of all "
                                   "blocks of K and V + every block's float64 attention), scaled by B*H*L units; the "
                                   "quantize steps run single-threaded numpy, the attention matmuls on the BLAS threads"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ our arm
def roofline_entry(kernel, bound, achieved, peak, unit, algorithmic, traffic, tnote, peak_note, extra=None):
    r = {"kernel": kernel, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
         "frac": achieved / peak, "traffic": traffic, "algorithmic": algorithmic,
         "traffic_unit": "DRAM bytes read + written per step (all launches of the kernel family in one decode)",
         "traffic_source": tnote, "peak_source": peak_note}
    if extra:
        r.update(extra)
    return r


def measure(args, vq, w, bits, world, seed, dev):
    """One workload: inputs resident in HBM, the whole decode captured as a CUDA
    graph and timed over args.steps replays (barrier + synchronize on both
    sides, max over ranks), then each kernel family of each block replayed
    alone for the per-kernel numbers. Returns the JSON fields of this workload."""
    L, S, B, H, D, N = w.layers, w.num_blocks, w.batch, w.heads, w.head_dim, w.tokens
    sigma = default_softmax_scale(w)
    desc = vq.CacheDesc(B, H, D, bits, w.block_tokens)
    ks, vs, qs, caches = [], [], [], []
    for layer in range(L):
        k, v = make_kv(w, layer, seed=seed, device=dev)
        ks.append(k)
        vs.append(v)
        qs.append(make_q(w, layer, seed=seed, device=dev))
        caches.append(vq.LayerCache(desc, device=dev))
    nmax = max(w.block_tokens)
    out = torch.empty((B, H, nmax, D), dtype=torch.float32, device=dev)
    outs = [out[:, :, :n] for n in w.block_tokens]

    def enqueue_fused(blocks, layers):
        for s in blocks:
            p0, n = w.prefix(s), w.block_tokens[s]
            for layer in layers:
                vq.vq_append_attention_block(desc, caches[layer], s, ks[layer][:, :, p0:p0 + n],
                                             vs[layer][:, :, p0:p0 + n], qs[layer][:, :, p0:p0 + n], sigma, outs[s])

    def enqueue(blocks, layers, do_quant=True, do_attn=True):
        for s in blocks:
            p0, n = w.prefix(s), w.block_tokens[s]
            for layer in layers:
                if do_quant:
                    vq.vq_cache_append(desc, caches[layer], s, ks[layer][:, :, p0:p0 + n],
                                       vs[layer][:, :, p0:p0 + n])
                if do_attn:
                    vq.vq_attention_block(desc, caches[layer], s, qs[layer][:, :, p0:p0 + n], sigma, outs[s])

    # The whole step, and each kernel family per block, captured once as CUDA
    # graphs: replays launch without host gaps, so CUDA events around a replay
    # time the kernels themselves.
    all_blocks, all_layers = range(S), range(L)
    enqueue(all_blocks, all_layers)           # eager warm-up: configures kernel attributes
    enqueue_fused(all_blocks, all_layers)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(cap):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            enqueue(all_blocks, all_layers)
        graphs["step"] = g
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            enqueue_fused(all_blocks, all_layers)
        graphs["fused"] = g
        for s in all_blocks:
            for kind in ("quant", "attn"):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    enqueue([s], all_layers, do_quant=(kind == "quant"), do_attn=(kind == "attn"))
                graphs[(kind, s)] = g
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def timed(g, reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    for _ in range(args.warmup):
        graphs["step"].replay()
    torch.cuda.synchronize()
    assert vq.vq_poll_device_error() == 0

    q_bytes = sum(quant_bytes(w, bits, s) for s in range(S)) * L
    a_flops = sum(attn_work(w, bits, s)[0] for s in range(S)) * L
    a_bytes = sum(attn_work(w, bits, s)[1] for s in range(S)) * L
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for _ in range(args.steps):
            graphs["step"].replay()
        stop.record(stream)
        torch.cuda.synchronize()
        # the same decode through the fused append+attention entry point
        fused_ms = timed(graphs["fused"], args.steps)
        # per-kernel, per-block times (same replays, each family alone)
        by_block = []
        t_quant = t_attn = 0.0
        for s in range(S):
            tq = timed(graphs[("quant", s)], args.steps)
            ta = timed(graphs[("attn", s)], args.steps)
            t_quant += tq
            t_attn += ta
            qb = quant_bytes(w, bits, s) * L
            af, ab = attn_work(w, bits, s)
            by_block.append({"block": s, "n": w.block_tokens[s], "quant_ms": round(tq, 4),
                             "quant_gbs": round(qb / (tq / 1e3) / 1e9, 1), "attn_ms": round(ta, 4),
                             "attn_gbs": round(ab * L / (ta / 1e3) / 1e9, 1),
                             "attn_tflops": round(af * L / (ta / 1e3) / 1e12, 2)})
    barrier(world)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    assert vq.vq_poll_device_error() == 0
    ms_step = elapsed_ms / args.steps
    tokens_step = B * N * L
    peaks, peak_src = load_peaks()
    hbm, tc_burst, tc_sus = peaks["hbm_gbs"], peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    peak_note = f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})"
    q_ms, a_ms = t_quant, t_attn
    q_gbs = q_bytes / (q_ms / 1e3) / 1e9
    a_gbs = a_bytes / (a_ms / 1e3) / 1e9
    a_tflops = a_flops / (a_ms / 1e3) / 1e12
    # the attention's bound: the larger of its HBM time and its tensor time at the burst peak
    a_bound = "hbm" if a_bytes / (hbm * 1e9) >= a_flops / (tc_burst * 1e12) else "tensor"
    if a_bound == "hbm":
        a_frac = {"frac": a_gbs / hbm}
    else:
        a_frac = {"frac": a_tflops / tc_burst, "frac_vs_sustained": a_tflops / tc_sus}
    rooflines = {}
    traffic, tnote = measured_traffic(w.name, "attention", L)
    if a_bound == "hbm":
        rooflines["attention"] = roofline_entry("attention", "hbm", a_gbs, hbm, "GB/s", a_bytes, traffic, tnote,
                                                peak_note)
    else:
        rooflines["attention"] = roofline_entry(
            "attention", "tensor", a_tflops, tc_burst, "TFLOP/s", a_flops, traffic, tnote,
            peak_note + "; bf16 burst peak", {"peak_sustained": tc_sus, "frac_vs_sustained": a_tflops / tc_sus})
    traffic, tnote = measured_traffic(w.name, "quant_pack", L)
    rooflines["quant_pack"] = roofline_entry("quant_pack", "hbm", q_gbs, hbm, "GB/s", q_bytes, traffic, tnote,
                                             peak_note)
    dominant = "attention" if a_ms >= q_ms else "quant_pack"
    res = {
        "workload": w.name, "bits": bits, "ms_per_step": ms_step,
        "value": weak_scaling_value(tokens_step, world, ms_step), "unit": "tokens/s",
        "config": workload_config(w, bits),
        "quant_pack": {"ms_per_step": q_ms, "gbs": q_gbs, "frac_hbm": q_gbs / hbm, "bytes_per_step": q_bytes},
        "attention": {"ms_per_step": a_ms, "tokens_per_s": tokens_step / (a_ms / 1e3), "gbs": a_gbs,
                      "tflops": a_tflops, "bound": a_bound, "frac_roofline": a_frac["frac"],
                      **({"frac_vs_sustained": a_frac["frac_vs_sustained"]} if "frac_vs_sustained" in a_frac else {}),
                      "flops_per_step": a_flops, "bytes_per_step": a_bytes},
        "roofline": rooflines[dominant],
        "roofline_other": rooflines["quant_pack" if dominant == "attention" else "attention"],
        "fused": {"ms_per_step": fused_ms, "value": weak_scaling_value(tokens_step, world, fused_ms),
                  "unit": "tokens/s", "launches_per_step": L * sum(1 if n <= 256 else 2 for n in w.block_tokens),
                  "note": "the same decode through vq_append_attention_block (append and attention in one launch "
                          "where that is faster: CUDA-core blocks with at most 4 (batch, head) per SM; two "
                          "launches otherwise), replayed alone after the timed steps"},
        "clocks": clk.summary(),
        "gpu_launches": 2 * L * S * args.steps,
        "by_block": by_block,
    }
    if args.e2e and w.name == args.workload:
        res["e2e"] = run_e2e(args, vq, w, bits, desc, caches, outs, dev, world)
    del graphs, ks, vs, qs, caches, out, outs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    from bit_kv_cache_25_b200 import vq

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    import dataclasses
    names = [args.workload] + [x for x in args.also.split(",") if x and x != "none" and x != args.workload]
    results = []
    for name in names:
        w = WORKLOADS[name]
        if args.layers:
            w = dataclasses.replace(w, layers=args.layers)   # smaller case for profiler captures
        bits = (args.bits or w.bits[0]) if name == args.workload else w.bits[0]
        results.append(measure(args, vq, w, bits, world, 1000003 * rank, dev))
    head = results[0]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": head["config"],
        "quant_pack": head["quant_pack"], "attention": head["attention"], "roofline": head["roofline"],
        "roofline_other": head["roofline_other"], "fused": head["fused"], "clocks": head["clocks"],
        "gpu_launches": sum(r["gpu_launches"] for r in results),
        "timing": "step = one CUDA-graph replay of the whole decode; per-kernel times from graphs of each kernel "
                  "family per block, replayed alone",
        "by_block": head["by_block"],
    }
    if "e2e" in head:
        line["e2e"] = head["e2e"]
    for r in results[1:]:
        line[r["workload"]] = {k: r[k] for k in ("bits", "ms_per_step", "value", "unit", "config", "quant_pack",
                                                 "attention", "roofline", "roofline_other", "fused", "clocks",
                                                 "gpu_launches", "by_block")}
    if rank == 0 and not args.no_cpu:
        w = WORKLOADS[args.workload]
        bits = args.bits or w.bits[0]
        tps, units, secs = cpu_sample(w, bits, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                                "blas_threads": blas_threads(), "quantize_threads": 1,
                                "sample": f"{units} (batch, head) units of layer 0 of {w.name} through the oracle "
                                          f"(append of all blocks + float64 attention of every block), {secs:.1f} s, "
                                          f"scaled by B*H*L units per step; the quantize steps run single-threaded "
                                          f"numpy, the attention matmuls on the BLAS threads"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_e2e(args, vq, w, bits, desc, caches, outs, dev, world):
    """Same decode through the public API with host inputs: every step copies each
    layer's K, V, Q from pinned host memory, runs its appends and attentions, and
    copies its outputs back. The host holds one layer of inputs, reused for
    every layer. Three streams overlap the work of neighbouring layers: the
    inputs of layer l+1 go up and the outputs of layer l-1 come down while
    layer l computes (two device buffers of each, ordered by events)."""
    L, S = w.layers, w.num_blocks
    k0, v0 = make_kv(w, 0, seed=7, device="cpu")
    q0 = make_q(w, 0, seed=7, device="cpu")
    hk, hv, hq = k0.pin_memory(), v0.pin_memory(), q0.pin_memory()
    dk = [torch.empty_like(hk, device=dev) for _ in range(2)]
    dv = [torch.empty_like(hv, device=dev) for _ in range(2)]
    dq = [torch.empty_like(hq, device=dev) for _ in range(2)]
    B, H, D, N = w.batch, w.heads, w.head_dim, w.tokens
    dout = [torch.empty((B, H, N, D), dtype=torch.float32, device=dev) for _ in range(2)]
    hout = torch.empty((B, H, N, D), dtype=torch.float32).pin_memory()
    sigma = default_softmax_scale(w)
    stream = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def step():
        for layer in range(L):
            b = layer % 2
            up.wait_event(computed[b])           # buffer b's previous layer has been used
            with torch.cuda.stream(up):
                dk[b].copy_(hk, non_blocking=True)
                dv[b].copy_(hv, non_blocking=True)
                dq[b].copy_(hq, non_blocking=True)
                in_ready[b].record(up)
            stream.wait_event(in_ready[b])
            stream.wait_event(out_done[b])       # dout[b] has been copied out
            for s in range(S):
                p0, n = w.prefix(s), w.block_tokens[s]
                vq.vq_cache_append(desc, caches[layer], s, dk[b][:, :, p0:p0 + n], dv[b][:, :, p0:p0 + n],
                                   stream=stream)
                vq.vq_attention_block(desc, caches[layer], s, dq[b][:, :, p0:p0 + n], sigma,
                                      dout[b][:, :, p0:p0 + n], stream=stream)
            computed[b].record(stream)
            down.wait_event(computed[b])
            with torch.cuda.stream(down):
                hout.copy_(dout[b], non_blocking=True)
                out_done[b].record(down)
        # the step ends when its last outputs are on the host
        stream.wait_event(out_done[(L - 1) % 2])

    steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(1):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)  # no copy of the timed steps starts before the clock does
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    h2d = L * sum(t.numel() * t.element_size() for t in (hk, hv, hq))
    d2h = L * hout.numel() * hout.element_size()
    return {"value": world * B * N * L / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "overlap": "inputs of layer l+1 and outputs of layer l-1 copied while layer l computes"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="var_d30", choices=sorted(WORKLOADS))
    ap.add_argument("--bits", type=int, default=0)
    ap.add_argument("--also", default="infinity_2b",
                    help="comma-separated workloads measured after the headline one ('none' to skip)")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-units", type=int, default=8)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling only)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
