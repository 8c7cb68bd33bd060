"""KV compress throughput of the JoLT / FlashJoLT library on a LLaMA-3.1-8B-shaped 64K cache.

One step = jolt_compress (FlashJoLT) of the whole cache (K and V, 32 layers x 8 KV heads x
65536 tokens x 128 features, bf16, 8 GiB) at the 2x budget, then again at the 3x budget.
`value` is input GB/s over the timed steps (inputs resident in HBM and larger than L2; the
L2 is also flushed between steps), `e2e` is the same metric through the public API with
the caches copied in from pinned host memory and the blobs read back every step.  The
Mistral-7B-shaped cache (1024 tokens) is timed beside it as an extra key, with the JoLT
(exact) arm.  For N > 1 every rank compresses its own cache (weak scaling; the units of
different caches are independent, so no collective is involved).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--method randomized|exact]
  python bench.py --impl reference ...   # the float64 CPU oracle on a bounded sample
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV compress throughput (input GB/s) at 2x/3x budget"
RATIOS = (2.0, 3.0)
L2_BYTES = 126 * 1024 * 1024
# DRAM bytes (read + write) per launch of the dominant kernel from an ncu capture of the
# current kernel, keyed by workload; a workload without an entry reports null.  The table
# kernel on the LLaMA-3.1-8B/64K cache: 11,376,815,104 read + 210,655,744 written (one-pass
# metrics, full size; the one-pass input is the 8.6 GB cache, U and P', about 11.6 GB)
KERNEL_TRAFFIC_BYTES = {("llama31_8b_64k", "table_kernel"): 11376815104 + 210655744}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="jolt", choices=["jolt", "reference"])
    ap.add_argument("--method", default="randomized", choices=["randomized", "exact"])
    ap.add_argument("--workload", default="llama31_8b_64k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the exact-arm and decompress side figures")
    ap.add_argument("--profile-case", default=None, choices=["mistral7b_4layers", "mistral7b", "llama31_8b_64k", "llama31_8b_4layers_T8192"],
                    help="run two compress + decompress calls of one case (for ncu captures) and exit")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per workload of the other shapes (LLaMA-2-13B, LLaMA-3.1-8B/64K) and "
                         "per context length of the Mistral-shaped sweep, JoLT and FlashJoLT, then exit")
    return ap.parse_args()


def profile_case(args):
    """Two FlashJoLT (or JoLT) compress + decompress calls of one case, for ncu captures:
    mistral7b_4layers (16 MiB of K and V), the full Mistral-shaped cache (128 MiB, about 1 GiB
    of workspace with FlashJoLT), the LLaMA-3.1-8B/64K cache (8 GiB; for launch lists only) or
    one layer group of it at 8192 tokens (128 MiB), with the same kernels as the timed run."""
    import torch
    from kv_cache_compression_group_b200 import synth, jolt as J
    if args.profile_case in ("mistral7b", "llama31_8b_64k"):
        w = synth.WORKLOADS[args.profile_case]
    elif args.profile_case == "llama31_8b_4layers_T8192":
        # the LLaMA-3.1-8B generator and candidate sets (token ranks up to 960) on one layer
        # group of 8192 tokens: the long-context kernels at a size a full ncu capture can take
        w = synth.small_workload("llama31_8b_64k", n_layers=4, T=8192)
    else:
        w = synth.small_workload("mistral7b", n_layers=4)
    K, V = synth.make_cache(w, 0)
    Kd, Vd = K.cuda(), V.cuda()
    opts = J.default_options(w.T, w.D, args.method)
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
    for _ in range(2):
        blob = comp.compress(Kd, Vd, w.bf16_bytes() // 2, 0)
        Kh, Vh = comp.decompress(blob)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile_case, "method": args.method,
                      "total_bytes": J.read_header(blob)[1]}))


def sweep(args):
    """Compress and decompress throughput of the other workload shapes: LLaMA-2-13B and
    LLaMA-3.1-8B/64K (FlashJoLT, 2x / 3x), and the Mistral-shaped generator at T = 512 ..
    32768 (FlashJoLT; JoLT up to T = 2048, 2x).  Each case: the first call runs directly, the second is
    captured as a CUDA graph, then three replays are timed with CUDA events (inputs resident
    in HBM; the 126 MB L2 holds a small part of the larger caches)."""
    import torch
    from kv_cache_compression_group_b200 import synth, jolt as J
    cases = [("llama2_13b", "randomized", (2.0, 3.0)), ("llama31_8b_64k", "randomized", (2.0, 3.0))]
    for T in (512, 1024, 2048, 8192, 32768):
        for meth in (("exact", "randomized") if T <= 2048 else ("randomized",)):
            cases.append((f"sweep_T{T}", meth, (2.0,)))
    cache = {}
    for name, meth, ratios in cases:
        w = synth.sweep_workload(int(name[7:])) if name.startswith("sweep_T") else synth.WORKLOADS[name]
        if name not in cache:
            cache.clear()
            K, V = synth.make_cache(w, 0)
            cache[name] = (K.cuda(), V.cuda())
            del K, V
        Kd, Vd = cache[name]
        opts = J.default_options(w.T, w.D, meth)
        comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, Kd.dtype, opts)
        for ratio in ratios:
            budget = int(w.bf16_bytes() / ratio)
            blob = torch.empty(min(budget, comp.blob_max), dtype=torch.uint8, device="cuda")
            for _ in range(3):
                comp.compress(Kd, Vd, budget, 0, blob=blob)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(3):
                comp.compress(Kd, Vd, budget, 0, blob=blob)
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / 3
            _, total, _ = J.read_header(blob)
            Ko, Vo = comp.decompress(blob)
            torch.cuda.synchronize()
            a.record()
            Ko, Vo = comp.decompress(blob, K_out=Ko, V_out=Vo)
            b.record()
            torch.cuda.synchronize()
            dms = a.elapsed_time(b)
            ek, ev = J.relative_errors(Kd, Vd, Ko, Vo, w.layers_per_group)
            del Ko, Vo
            print(json.dumps({"sweep": name, "method": meth, "ratio": ratio, "shape": [w.n_layers, w.n_heads, w.T, w.D],
                              "input_bytes": w.input_bytes(), "compress_ms": ms, "compress_gbs": w.input_bytes() / ms / 1e6,
                              "latency_per_layer_group_ms": ms / w.n_groups, "decompress_ms": dms,
                              "decompress_out_gbs": w.input_bytes() / dms / 1e6, "total_bytes": total,
                              "rel_err_K": ek, "rel_err_V": ev, "token_ranks": list(opts.token_ranks)}), flush=True)
        del comp
        torch.cuda.empty_cache()


def workload_config(w, method, opts):
    return {
        "workload": f"{w.name}: K and V [{w.n_layers}, {w.n_heads}, {w.T}, {w.D}] {w.dtype}, "
                    f"layer groups of {w.layers_per_group}, {'FlashJoLT' if method == 'randomized' else 'JoLT'} "
                    f"compress at {'/'.join(f'{r:g}x' for r in RATIOS)} budgets",
        "n_layers": w.n_layers, "n_kv_heads": w.n_heads, "n_tokens": w.T, "head_dim": w.D,
        "layers_per_group": w.layers_per_group, "method": method,
        "token_ranks": list(opts.token_ranks), "feature_ranks": list(opts.feature_ranks),
        "bits": list(opts.bits), "oversample": opts.oversample, "power_iters": opts.power_iters,
        "budgets_bytes": [int(w.bf16_bytes() / r) for r in RATIOS],
        "generator": f"{w.n_components} rank-one terms, s_i = exp(-i/{w.decay:g}), noise {w.noise}, "
                     f"key scales lognormal(0, {w.key_sigma})",
        "l2": "flushed between steps (write of a 256 MiB buffer)",
    }


# ------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except FileNotFoundError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm = [float(r[1]) for r in self.rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            if len(r) < 9:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# roofline model of the library's stages (algorithmic work per launch)
# ------------------------------------------------------------------------------------------
def table_alu_ops(w, opts, n_units):
    """Quantiser arithmetic of the distortion table: per element and (r_T, r_D) candidate,
    1 residual subtraction + 2 block min/max + 1 offset from lo, then per bit-width b > 0:
    scale-and-round (1 FMA with the shift constant), 1 subtraction back to the integer,
    1 FMA for the error and 1 FMA to accumulate its square; b = 0 is 1 FMA."""
    per = 4 + sum(4 if b > 0 else 1 for b in opts.bits)
    elems = n_units * w.layers_per_group * w.n_heads * w.T * w.D
    return elems * len(opts.token_ranks) * len(opts.feature_ranks) * per, per


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


# ------------------------------------------------------------------------------------------
SAMPLE_TOKENS = 1024


def oracle_sample_input(w, seed):
    """The bounded sample the float64 oracle is timed on: the keys of layer group 0 of the
    workload, restricted to its first SAMPLE_TOKENS tokens ([L_g, H, 1024, D]; for the
    1024-token Mistral shape that is the whole unit)."""
    from kv_cache_compression_group_b200 import synth
    K = synth.make_cache(w, seed, kv=0, layers=range(0, w.layers_per_group))
    return K[:, :, :min(w.T, SAMPLE_TOKENS)].contiguous()


def oracle_sample(w, opts_j, seed, ratio, K):
    """The float64 oracle as it stands on the sample unit K: factors, distortion table with
    the workload's candidate sets, allocation at the unit's share of the budget, encoding."""
    import oracle as O
    from kv_cache_compression_group_b200 import synth
    X = synth.to_f64(K)
    Lg, H, T, D = X.shape
    oo = O.Options(opts_j.token_ranks, opts_j.feature_ranks, opts_j.bits, opts_j.method,
                   opts_j.oversample, opts_j.power_iters)
    t0 = time.perf_counter()
    f = O.unit_factors(X, 0, 0, oo, seed)
    tab = O.distortion_table(X, f.U_s, f.W_s, f.C_s, f.sigma, oo).reshape(1, -1)
    B = O.bytes_table(T, D, Lg * H, oo).reshape(1, -1)
    budget = int(X.size * 2 / ratio) - O.header_bytes(1)
    al = O.allocate(tab, B, budget)
    if al.status == "ok":
        O.encode_unit(X, f, oo, int(al.choice[0]), float(tab[0, al.choice[0]]))
    dt = time.perf_counter() - t0
    return dt, X.size * 2


def sample_text(w, K, extra=""):
    Lg, H, T, D = K.shape
    return (f"one unit: keys of layer group 0 of {w.name}, first {T} of {w.T} tokens ([{Lg}, {H}, {T}, {D}] bf16, "
            f"{K.numel() * 2 / 2**20:.0f} MiB), the workload's candidate sets{extra}")


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        n = 1
    return n, len(os.sched_getaffinity(0))


# ------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The oracle on the host cores: each step is the sample unit at 2x or 3x (alternating)."""
    from kv_cache_compression_group_b200 import synth, jolt as J
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    opts = J.default_options(w.T, w.D, args.method)
    K = oracle_sample_input(w, 0)
    times, nbytes = [], 0
    for i in range(args.warmup + args.steps):
        dt, nb = oracle_sample(w, opts, 0, RATIOS[i % 2], K)
        if i >= args.warmup:
            times.append(dt)
            nbytes += nb
    tot = sum(times)
    value = nbytes / tot / 1e9
    threads, cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / len(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.method, opts),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "host_cores": cores, "kind": "oracle",
                         "sample": sample_text(w, K, ", budgets alternating 2x / 3x, one unit per step")},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------
def fp32_peak(J, dev, stream):
    """FP32-pipe rate measured in this process: FMAs per second of the library's probe kernel,
    scalar (FFMA) and packed (FFMA2), best of three launches each after a warm-up.  Each FMA
    counts as one operation, as in the algorithmic operation counts."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sink = torch.empty(sms * 8 * 256, dtype=torch.float32, device=dev)
    out = {}
    for packed in (False, True):
        J.fp32_rate_probe(packed, 2000, sink)
        best = 0.0
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ops = J.fp32_rate_probe(packed, 20000, sink)
            b.record(stream)
            torch.cuda.synchronize()
            best = max(best, ops / (a.elapsed_time(b) / 1e3) / 1e12)
        out["ffma2_tops" if packed else "ffma_tops"] = best
    out["peak_tops"] = max(out["ffma_tops"], out["ffma2_tops"])
    out["note"] = "measured in this run: FMAs per second of a probe kernel, 8 CTAs of 256 threads per SM"
    return out


def stage_rooflines(w, opts, n_units, prof, n_calls, per_call_ms, peaks, peak_src, alu, chosen):
    """Algorithmic work of each library stage (per compress call) against its own bound, for
    the stages that take more than 5 % of a compress.  Work counts what the method computes,
    not what the implementation adds (the bf16 hi + lo halves of fp32 operands, recomputed
    operators, the compensated residual sums of the encoder): achieved = algorithmic work /
    measured stage time.  `chosen`: the unit records of the blobs of one step (one list per
    budget), for the stages whose work depends on the allocation."""
    S = w.layers_per_group * w.n_heads
    N = S * w.T * w.D                       # elements per unit
    M = S * w.D
    T = w.T
    k = max(opts.token_ranks) + opts.oversample
    q = opts.power_iters
    rT, nD = max(opts.token_ranks), len(opts.feature_ranks)
    hbm = float(peaks["hbm_gbs"])
    tens = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    work = {
        # products with the cache: Y = X Omega, then (Z = X^T Q, Y = X Q_z) per power iteration,
        # then Z = X^T Q for the Rayleigh-Ritz Gram: 2 T M k each
        "sketch_product": ("tensor", (2 + 2 * q) * 2.0 * T * M * k * n_units, "FLOP"),
        # Cholesky-QR Grams: (q + 2) passes on T x k, q on M x k; m k^2 each (symmetric)
        "qr_gram": ("tensor", ((q + 2) * T + q * M) * float(k) * k * n_units, "FLOP"),
        # Q = Y L^{-T}: m k^2 per pass (triangular)
        "qr_trsm": ("tensor", ((q + 2) * T + q * M) * float(k) * k * n_units, "FLOP"),
        "ritz_vectors": ("tensor", 2.0 * T * k * rT * n_units, "FLOP"),
        "table_kernel": ("alu", table_alu_ops(w, opts, n_units)[0], "op"),
        # the reconstruction U_s[:, :r_T] P' of every slice whose unit stores a residual (b > 0),
        # at the ranks the allocation chose, averaged over the step's budgets
        "encode": ("tensor", sum(2.0 * w.T * S * w.D * r["r_T"] for recs in chosen for r in recs if r["bits"] > 0)
                   / max(1, len(chosen)), "FLOP"),
        "feature_factor": ("hbm", 2.0 * N * n_units, "B"),
        # Z = X W (2 N r_D) and U^T Z (2 r_T T S r_D) at the largest ranks
        "core": ("tensor", (2.0 * N * max(opts.feature_ranks) + 2.0 * rT * T * S * max(opts.feature_ranks)) * n_units,
                 "FLOP"),
    }
    lines = []
    for name, (ms, launches, _) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
        ms_call = ms / n_calls
        if ms_call < 0.05 * per_call_ms:
            continue
        line = {"kernel": name, "ms_per_launch": ms_call, "share_of_compress": ms_call / per_call_ms}
        if name in work:
            bound, amount, unit = work[name]
            t = ms_call / 1e3
            if bound == "tensor":
                ach, peak, u = amount / t / 1e12, tens, "TFLOP/s"
                src = f"{peak_src} bf16 dense, sustained"
            elif bound == "hbm":
                ach, peak, u = amount / t / 1e9, hbm, "GB/s"
                src = f"{peak_src} HBM copy"
            else:
                ach, peak, u = amount / t / 1e12, alu["peak_tops"], "Top/s"
                src = "measured FP32-pipe probe (best of scalar FFMA and packed FFMA2)"
            line.update({"bound": bound, "achieved": ach, "peak": peak, "unit": u, "frac": ach / peak,
                         "work_per_launch": amount, "work_unit": unit, "peak_source": src})
        else:
            line["bound"] = "latency"
        lines.append(line)
    return lines


def attend_extras(J, comp, blob, w, dev, stream):
    """Decode-side attention over the stored factors of the 2x blob: one decode step of 4
    query heads per KV head against every cached token, layer by layer (all layers timed
    together with CUDA events after a warm-up pass).  Bytes are those the kernels must read
    for a layer: both token factors, the codes and the scales of the layer's slices."""
    import torch
    nq = 4 * w.n_heads
    att = J.Attention(comp, blob, nq)
    q = torch.randn((nq, w.D), dtype=torch.float32, device=dev, generator=torch.Generator(dev).manual_seed(1))
    outs = torch.empty_like(q)
    for layer in range(w.n_layers):
        att.attend(layer, q, out=outs)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for layer in range(w.n_layers):
        att.attend(layer, q, out=outs)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / w.n_layers
    _, _, recs = J.read_header(blob)
    nbytes = 0.0
    for g in range(w.n_groups):
        rk, rv = recs[2 * g], recs[2 * g + 1]
        for r in (rk, rv):
            nbytes += 2.0 * w.T * r["r_T"]                                   # token factor
            nbytes += w.n_heads * w.T * (w.D // 16) * (2 * r["bits"] + 4) if r["bits"] else 0.0
    nbytes /= w.n_groups
    return {"query_heads": nq, "ms_per_layer": ms, "bytes_per_layer": nbytes, "gbs": nbytes / ms / 1e6,
            "note": "host sync per call to read the blob header is inside the timed region"}


def mistral_extras(J, synth, dev, stream, flush):
    """The Mistral-7B-shaped cache (1024 tokens): FlashJoLT compress at 2x and 3x (graph
    replays, events around each call, L2 flushed before), and JoLT (exact) at 2x."""
    import torch
    w = synth.WORKLOADS["mistral7b"]
    K, V = synth.make_cache(w, 0)
    Kd, Vd = K.to(dev), V.to(dev)
    out = {"workload": f"mistral7b: K and V [{w.n_layers}, {w.n_heads}, {w.T}, {w.D}] bf16, layer groups of 4"}
    for meth in ("randomized", "exact"):
        o2 = J.default_options(w.T, w.D, meth)
        c2 = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, o2, dev)
        res = {}
        for ratio in ((2.0, 3.0) if meth == "randomized" else (2.0,)):
            budget = int(w.bf16_bytes() / ratio)
            blob = torch.empty(min(budget, c2.blob_max), dtype=torch.uint8, device=dev)
            for _ in range(3):   # direct run, graph capture, one replay
                c2.compress(Kd, Vd, budget, 0, blob=blob)
            ts = []
            for _ in range(5):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                c2.compress(Kd, Vd, budget, 0, blob=blob)
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            ms = sorted(ts)[len(ts) // 2]
            Ko, Vo = c2.decompress(blob)
            ek, ev = J.relative_errors(Kd, Vd, Ko, Vo, w.layers_per_group)
            res[f"{ratio:g}x"] = {"compress_ms": ms, "gbs": w.input_bytes() / ms / 1e6, "rel_err_K": ek, "rel_err_V": ev}
        out["FlashJoLT" if meth == "randomized" else "JoLT"] = res
        del c2
    out["flashjolt_speedup_over_jolt_2x"] = out["JoLT"]["2x"]["compress_ms"] / out["FlashJoLT"]["2x"]["compress_ms"]
    del Kd, Vd
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------------------------------
def main():
    args = parse()
    from kv_cache_compression_group_b200 import ranks
    rank, world, local = ranks.dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.profile_case:
        return profile_case(args)
    if args.sweep:
        return sweep(args)

    import torch
    from kv_cache_compression_group_b200 import synth, jolt as J

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks.init(world, "nccl", dev)

    w = synth.WORKLOADS[args.workload]
    opts = J.default_options(w.T, w.D, args.method)
    seed = ranks.rank_seed(rank)
    K, V = synth.make_cache(w, seed)
    Kd, Vd = K.to(dev), V.to(dev)
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts, dev)
    budgets = [int(w.bf16_bytes() / r) for r in RATIOS]
    blobs = [torch.empty(min(b, comp.blob_max), dtype=torch.uint8, device=dev) for b in budgets]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(Ks, Vs):
        for b, blob in zip(budgets, blobs):
            comp.compress(Ks, Vs, b, seed, blob=blob)

    def barrier():
        ranks.barrier(world)

    for _ in range(args.warmup):
        flush.zero_()
        step(Kd, Vd)
    torch.cuda.synchronize()
    # validity of what is timed: the blobs decode and respect their budgets
    chosen = []
    for b, blob in zip(budgets, blobs):
        _, total, recs = J.read_header(blob)
        assert total <= b
        chosen.append(recs)

    # ---- timed region: device-resident inputs ------------------------------------------
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    n0 = J.launch_count()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step(Kd, Vd)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    launches = J.launch_count() - n0
    barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    t_ms = sum(step_ms)
    t_ms = ranks.max_over_ranks(t_ms, world, dev)
    in_bytes = w.input_bytes()
    value = ranks.aggregate_gbs(world, args.steps * len(RATIOS) * in_bytes, t_ms)

    # ---- end to end through the public API: pinned host in, blobs out ---------------------
    # Every step copies its cache in from pinned host memory and its blobs out, inside the
    # timed region. The copies run on a second stream, double-buffered: step i + 1's upload and
    # step i's download overlap the compress of the neighbouring step. Events order every
    # buffer reuse: an upload waits for the compress that last read its buffers, a download for
    # the compress that wrote its blobs, and a compress for its upload. The upload into a slot
    # is issued after that slot's previous download on the copy stream, so it also orders the
    # compress that overwrites those blobs.
    Kh, Vh = K.pin_memory(), V.pin_memory()
    Kb = [torch.empty_like(Kd), torch.empty_like(Kd)]
    Vb = [torch.empty_like(Vd), torch.empty_like(Vd)]
    dblobs = [blobs, [torch.empty_like(bl) for bl in blobs]]
    host_blobs = [[torch.empty(bl.numel(), dtype=torch.uint8).pin_memory() for bl in blobs] for _ in range(2)]
    cstream = torch.cuda.Stream(device=dev)
    h2d_ev = [torch.cuda.Event(), torch.cuda.Event()]
    done_ev = [torch.cuda.Event(), torch.cuda.Event()]
    d2h = sum(bl.numel() for bl in blobs)

    def upload(slot):
        with torch.cuda.stream(cstream):
            cstream.wait_event(done_ev[slot])
            Kb[slot].copy_(Kh, non_blocking=True)
            Vb[slot].copy_(Vh, non_blocking=True)
            h2d_ev[slot].record(cstream)

    def download(slot):
        with torch.cuda.stream(cstream):
            cstream.wait_event(done_ev[slot])
            for bl, hb in zip(dblobs[slot], host_blobs[slot]):
                hb.copy_(bl, non_blocking=True)

    def compute(slot):
        stream.wait_event(h2d_ev[slot])
        for b, bl in zip(budgets, dblobs[slot]):
            comp.compress(Kb[slot], Vb[slot], b, seed, blob=bl)
        done_ev[slot].record(stream)

    def e2e_run(nsteps, start=None):
        if start is not None:
            cstream.wait_event(start)
        upload(0)
        for i in range(nsteps):
            s = i % 2
            if i + 1 < nsteps:
                upload(1 - s)
            compute(s)
            download(s)
        fin = torch.cuda.Event()
        fin.record(cstream)
        stream.wait_event(fin)

    # each buffer slot's argument set runs directly once, is captured once, then replays
    e2e_run(max(6, args.warmup))
    torch.cuda.synchronize()
    for slot in range(2):
        for b, bl in zip(budgets, dblobs[slot]):
            _, total, _ = J.read_header(bl)
            assert total <= b
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps, start=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = ranks.max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = {"value": ranks.aggregate_gbs(world, args.steps * len(RATIOS) * in_bytes, e_ms), "unit": "GB/s",
           "h2d_bytes_per_step": 2 * K.numel() * K.element_size(), "d2h_bytes_per_step": d2h,
           "ms_per_step": e_ms / args.steps,
           "note": "copies on a second stream, double-buffered: step i+1's upload and step i's download "
                   "overlap the neighbouring compress; all bytes of every step inside the timed region"}

    # ---- stage breakdown: a separate pass with per-stage events (these calls run without
    # the CUDA graphs of the timed region, so stage sums exceed the timed step) ------------
    J.profile_begin()
    for _ in range(2):
        flush.zero_()
        step(Kd, Vd)
    torch.cuda.synchronize()
    prof = J.profile_end()

    # ---- measured FP32-pipe peak (scalar FFMA and packed FFMA2 probes) -------------------
    alu = fp32_peak(J, dev, stream)

    # ---- roofline of every stage above 5 % of a compress ---------------------------------
    peaks, peak_src = load_peaks()
    stages = {k: {"ms_total": v[0], "launches": v[1], "ms_per_launch": v[0] / max(1, v[1])} for k, v in prof.items()}
    n_calls = 2 * len(RATIOS)
    per_call_ms = t_ms / args.steps / len(RATIOS)
    lines = stage_rooflines(w, opts, comp.n_units, prof, n_calls, per_call_ms, peaks, peak_src, alu, chosen)
    leaf = [l for l in lines if l.get("bound") in ("alu", "tensor", "hbm")]
    dom = max(leaf, key=lambda l: l["ms_per_launch"]) if leaf else None
    roofline = None
    if dom is not None:
        roofline = dict(dom)
        roofline["traffic"] = KERNEL_TRAFFIC_BYTES.get((w.name, dom["kernel"]))
        if roofline["traffic"] is not None:
            roofline["traffic_source"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the "
                                          "current kernel on this workload (one-pass metrics, full size)")
        roofline["timing"] = ("per-launch time from a separate pass with CUDA events around the stage on its "
                              "launch stream (the timed steps replay CUDA graphs, which hold no events)")

    out = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, args.method, opts),
        "e2e": e2e, "gpu_launches": int(launches), "clocks": clk, "roofline": roofline,
        "stage_rooflines": lines, "alu_peak": alu, "stages": stages,
    }

    if rank == 0 and not args.no_extras:
        out["mistral7b"] = mistral_extras(J, synth, dev, stream, flush)
        # decompress of the headline cache (output GB/s) and its relative errors
        Ko, Vo = comp.decompress(blobs[0])
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        Ko, Vo = comp.decompress(blobs[0], K_out=Ko, V_out=Vo)
        b.record(stream)
        torch.cuda.synchronize()
        dms = a.elapsed_time(b)
        ek, evv = J.relative_errors(Kd, Vd, Ko, Vo, w.layers_per_group)
        out["decompress_2x"] = {"ms": dms, "out_gbs": in_bytes / dms / 1e6, "rel_err_K": ek, "rel_err_V": evv}
        del Ko, Vo
        out["attend_2x"] = attend_extras(J, comp, blobs[0], w, dev, stream)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Ks = oracle_sample_input(w, 0)
        dt, nb = oracle_sample(w, opts, 0, RATIOS[0], Ks)
        threads, cores = cpu_threads()
        out["cpu_baseline"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "host_cores": cores,
                               "kind": "oracle", "sample": sample_text(w, Ks, f", 2x budget, {dt:.1f} s")}
    ranks.barrier(world)
    ranks.shutdown(world)
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
