#!/usr/bin/env python
"""Benchmark of the JoLT codec's hot path on B200.

One step = one pass of the whole path over one batch of synthetic input resident in HBM:
  jolt_analyze (spectra of every cell) -> jolt_allocate (host, one multiplier per sequence at the
  workload's byte budget) -> jolt_compress (factors + packed residuals) -> jolt_decode_attn (one
  query token per (sequence, layer, query head) over every cached token of every layer).
Throughput unit: context tokens (B*T per rank) through the step per second. The JSON line also
breaks the step down (compress raw GB/s; decode context tokens/s and HBM GB/s) and carries the
live roofline of the dominant kernel family and of the decode kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl jolt|reference]
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import get_workload, make_kv, make_queries, make_inv_freq  # noqa: E402

METRIC = ("decode-attn context tokens/s & HBM GB/s over compressed cache; compress raw GB/s")
DEFAULT_WORKLOAD = "llama70b_128k"
# the metric's other workloads in the default run: the HBM-bound non-RoPE decode (8B, 32K) and the
# batch-4 pre-RoPE 64K workload at its tighter budget
DEFAULT_ALSO = "llama8b_32k:3,llama8b_64k_b4:5"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--ratio", type=float, default=None)
    ap.add_argument("--impl", default="jolt", choices=["jolt", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=4096)
    ap.add_argument("--layers", type=int, default=None, help="override n_layers (small profiling cases)")
    ap.add_argument("--seqlen", type=int, default=None, help="override T (small profiling cases)")
    ap.add_argument("--nvtx", action="store_true", help="NVTX range 'jolt_step' around each timed step")
    ap.add_argument("--no-count", action="store_true", help="skip the CUPTI kernel count")
    ap.add_argument("--no-grouping", action="store_true", help="skip the layer-grouping report")
    ap.add_argument("--cells-per-pass", type=int, default=0,
                    help="cells jolt_analyze batches per pass (0: every cell of a kind in one pass)")
    ap.add_argument("--also", default=None,
                    help="extra workloads name[:ratio],... timed after the headline (default: the metric's "
                         "other workloads when --workload is the default; '' for none)")
    ap.add_argument("--exact", action="store_true",
                    help="exact token-mode SVD (sketch width = L_g*n_kv*d_h: the JoLT backbone FlashJoLT replaces)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """nvidia-smi sampling (200 ms) of SM clock and throttle reasons during the timed region."""

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ---------------------------------------------------------------------------------------------
# oracle (CPU) leg: bounded sample of the same workload
# ---------------------------------------------------------------------------------------------

def oracle_sample(w, choices_by_cell, T_s, K=None, V=None):
    """Time the CPU oracle on one layer group (its K and V cells) over the first T_s tokens:
    exact ST-HOSVD compression with the given choices, then decode attention for the group's
    layers. Returns (seconds, description)."""
    import oracle
    from oracle.codec import compress_cell, decompress_cell, decode_attention, rope
    Lg, d = w.layers_per_group, w.d_h
    T_s = min(T_s, w.T)
    ws = get_workload(w.name, T=T_s, n_layers=Lg, batch=1)
    if K is None:
        Kc, Vc = make_kv(ws, device="cpu", dtype=torch.float32)
    else:
        Kc = K[:1, :Lg, :, :T_s].float().cpu()
        Vc = V[:1, :Lg, :, :T_s].float().cpu()
    q = make_queries(ws, device="cpu", dtype=torch.float32).double().numpy()
    inv = make_inv_freq(d, w.rope_theta)
    t0 = time.perf_counter()
    cells = []
    for kv, X in ((0, Kc), (1, Vc)):
        rT, rd, b = choices_by_cell[kv]
        rT = min(rT, (min(T_s, Lg * w.n_kv * d) // 16) * 16)
        rd = rd if rT else 0
        cells.append(compress_cell(X[0].double().numpy(), rT, rd, b, 1234, w.factor_dtype))
    for ll in range(Lg):
        Kh = decompress_cell(cells[0], 1234)[ll]
        Vh = decompress_cell(cells[1], 1234)[ll]
        if w.keys_pre_rope:
            Kh = rope(Kh, np.arange(T_s), inv)
        decode_attention(Kh, Vh, q[0, ll], 1.0 / math.sqrt(d))
    dt = time.perf_counter() - t0
    desc = (f"oracle (float64 NumPy) on one {Lg}-layer group (its K and V cells) of the first {T_s} "
            f"tokens: exact ST-HOSVD compress + decode of {Lg} layers; full-step time extrapolated "
            f"linearly in T and in the {w.n_groups} groups x {w.batch} sequences")
    return dt, desc


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [os.cpu_count()])
    except Exception:
        return os.cpu_count()


def run_reference(args, w, rank, world):
    """--impl reference: the CPU oracle, as it stands, on bounded samples of the workload. Each step
    is one sample (one layer group's K and V cells over the first --cpu-tokens tokens: exact
    ST-HOSVD compression and the group's decode attention); ms_per_step is that sample's measured
    time and value its context tokens per second, a group of L_g layers being L_g / L of a token's
    pass through the model."""
    if rank != 0:
        return
    choices = {0: (256, 128, 4), 1: (256, 128, 4)} if not w.fixed_choice else {0: w.fixed_choice, 1: w.fixed_choice}
    T_s = min(args.cpu_tokens, w.T)
    for _ in range(args.warmup):
        oracle_sample(w, choices, T_s)
    times = []
    for _ in range(args.steps):
        dt, desc = oracle_sample(w, choices, T_s)
        times.append(dt)
    t_sample = float(np.mean(times))
    value = T_s * (w.layers_per_group / w.n_layers) / t_sample
    desc = (f"oracle (float64 NumPy) on one {w.layers_per_group}-layer group (its K and V cells) of the first "
            f"{T_s} tokens: exact ST-HOSVD compress + decode of {w.layers_per_group} layers per step; context "
            f"tokens counted as {T_s} x {w.layers_per_group}/{w.n_layers} of a full pass")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "context tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_sample * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "T": w.T, "n_layers": w.n_layers,
                       "sample": {"tokens": T_s, "layers": w.layers_per_group, "sequences": 1},
                       "budget": "fixed sample ranks (256, 128, 4)" if not w.fixed_choice else "fixed"},
            "cpu_baseline": {"value": value, "unit": "context tokens/s", "cores": cpu_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "context tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------------------------

class Step:
    def __init__(self, w, ratio, device, seed_shift=0, exact=False, cells_per_pass=0):
        from long_context_st_b200 import api
        self.api = api
        self.w = w
        over = {"cells_per_pass": cells_per_pass or w.batch * w.n_groups}
        if exact:
            over["sketch_cols"] = w.n_cols
        self.shape = api.make_shape(w, **over)
        self.dev = device
        self.K, self.V = make_kv(w, device=device)
        self.q = make_queries(w, device=device)
        self.inv = torch.from_numpy(make_inv_freq(w.d_h, w.rope_theta)).to(device)
        self.cws = api.new_workspace(self.shape, api.JOLT_OP_COMPRESS, device)
        self.dws = api.new_workspace(self.shape, api.JOLT_OP_DECODE, device)
        self.out = torch.empty_like(self.q)
        self.phi = api.phi(w.d_h)
        self.ratio = ratio
        self.cache = None
        self.choices = None
        raw = 2 * w.n_layers * w.n_kv * w.d_h * w.T * w.io_bytes
        self.budget = int(raw / ratio) if ratio else None

    def allocate(self, tables):
        w, api = self.w, self.api
        n2, tT, td = tables
        if w.fixed_choice:
            return [tuple(w.fixed_choice)] * len(n2)
        G = w.n_layers // w.layers_per_group
        out = []
        for b in range(w.batch):
            sl = slice(b * 2 * G, (b + 1) * 2 * G)
            ch, lam, tot = api.allocate(self.shape, n2[sl], tT[sl], td[sl], self.phi, self.budget)
            out.extend(ch)
        return out

    def run(self, events=None, K=None, V=None, host=None):
        """One step. host = (K_host, V_host): the inputs are copied from (pinned) host memory into
        K, V inside the analyze call (the value copy overlapping the key cells' analysis)."""
        api = self.api
        K = self.K if K is None else K
        V = self.V if V is None else V
        ev = events or {}
        if "start" in ev:
            ev["start"].record()
        if host is not None:
            tables = api.analyze_from_host(self.shape, host[0], host[1], K, V, self.cws)
        else:
            tables = api.analyze(self.shape, K, V, self.cws)
        self.tables = tables
        if "analyzed" in ev:
            ev["analyzed"].record()
        choices = self.allocate(tables)
        if self.cache is None or choices != self.choices:
            _, total = api.cache_layout(self.shape, choices)
            if self.cache is None or self.cache.numel() < total:
                self.cache = torch.empty(total, dtype=torch.uint8, device=self.dev)
            self.choices = choices
            self.choices_c = api.choices_array(choices)
        if "allocated" in ev:
            ev["allocated"].record()
        api.compress(self.shape, K, V, choices, self.cache, self.cws)
        if "compressed" in ev:
            ev["compressed"].record()
        api.decode_attn(self.shape, choices, self.cache, self.q, self.out, self.dws, inv_freq=self.inv,
                        choices_c=self.choices_c)
        if "decoded" in ev:
            ev["decoded"].record()
        return choices


def surrogate_error(tables, choices, phi):
    """The allocator's summed error model for a choice vector: phi(b) times the discarded mass."""
    n2, tT, td = tables
    bits = {0: 0, 2: 1, 4: 2, 8: 3}
    e = 0.0
    for c, (rT, rd, b) in enumerate(choices):
        D = n2[c] if rT == 0 else min(n2[c], tT[c][rT // 16] + td[c][rd // 16])
        e += phi[bits[b]] * D
    return e


def allocator_ablation(step):
    """The pages' allocation ablations on this step's own tables at its budget (first sequence):
    joint (one multiplier, exact per-cell search), K/V-decoupled, uniform ranks, and the pages'
    coordinate-wise rank search under the same multiplier — summed surrogate error / ||X||^2, bytes
    used and the share of the budget they use."""
    api, w = step.api, step.w
    if w.fixed_choice or step.budget is None:
        return None
    G = w.n_layers // w.layers_per_group
    n2, tT, td = (np.asarray(a)[:2 * G] for a in step.tables)
    out = {"budget_bytes": step.budget}
    for name, mode in (("joint", api.JOLT_ALLOC_JOINT), ("kv_split", api.JOLT_ALLOC_KV_SPLIT),
                       ("uniform", api.JOLT_ALLOC_UNIFORM), ("coordinate", api.JOLT_ALLOC_COORD)):
        try:
            t0 = time.perf_counter()
            ch, tot = api.allocate_variant(step.shape, n2, tT, td, step.phi, step.budget, mode)
            out[name] = {"rel_error": surrogate_error((n2, tT, td), ch, step.phi) / float(np.sum(n2)),
                         "bytes": tot, "budget_use": tot / step.budget,
                         "host_ms": (time.perf_counter() - t0) * 1e3}
        except api.JoltError as e:
            out[name] = {"error": str(e)}
    return out


def layer_grouping(step, rank=32, tau=0.5):
    """The pages' layer-grouping step ([v4] §3) on this step's own K/V, outside the timed step:
    alignment of consecutive layers' top-`rank` token subspaces (jolt_layer_align, averaged over
    the sequences), the consecutive groups at tau, the uniform group size a fixed-L_g shape could
    use, and the device time of one call."""
    api, w = step.api, step.w
    if w.n_layers < 2:
        return None
    try:
        ws = torch.zeros(api.layer_align_workspace(step.shape, rank), dtype=torch.uint8, device=step.K.device)
        api.layer_align(step.shape, step.K, step.V, rank, ws=ws)  # warm-up
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        a = api.layer_align(step.shape, step.K, step.V, rank, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        del ws
        mean = a.mean(axis=0)
        groups = api.group_layers(mean, tau)
        return {"rank": rank, "tau": tau, "ms": e0.elapsed_time(e1), "align_min": float(mean.min()),
                "align_max": float(mean.max()), "n_groups": len(groups), "groups": groups,
                "uniform_L_g": api.uniform_group(mean, tau)}
    except Exception as e:  # reported, not fatal: the step's own numbers stand
        return {"error": str(e)}


def decode_work(w, shape, choices):
    """Algorithmic work of one decode step over every layer: (bytes, flops).

    Bytes: the compressed cache read once (each cell's U_T, U_d, cores, codes and scale/zero
    pairs) plus q and the output. Flops: each contraction of the method once per (token, layer):
    scores 2 r_T^K per query head (non-RoPE: U_T^K against P = G^K U_d^K^T q) or the key rebuild
    2 r_T^K d_h per KV head plus q.k 2 d_h per query head (pre-RoPE), values 2 r_T^V per query head,
    and 2 d_h per query head for each residual that is stored (the key residual of non-RoPE keys,
    the value residual). bf16 hi/lo terms that only restore an operand's precision are not
    algorithmic work (the kernels report them as issued flops)."""
    from long_context_st_b200 import api
    G = w.n_layers // w.layers_per_group
    nbytes = sum(api.cell_bytes(shape, tuple(c)) for c in choices)
    nbytes += w.batch * w.n_layers * 2 * w.n_q * w.d_h * w.io_bytes
    flops = 0.0
    for b in range(w.batch):
        for g in range(G):
            rk, _, bk = choices[(b * G + g) * 2]
            rv, _, bv = choices[(b * G + g) * 2 + 1]
            per_layer = 0.0
            if w.keys_pre_rope:
                per_layer += 2.0 * rk * w.d_h * w.n_kv + 2.0 * w.d_h * w.n_q
            else:
                per_layer += 2.0 * rk * w.n_q + (2.0 * w.d_h * w.n_q if bk else 0.0)
            per_layer += 2.0 * rv * w.n_q + (2.0 * w.d_h * w.n_q if bv else 0.0)
            flops += per_layer * w.T * w.layers_per_group
    return nbytes, flops


def count_kernels(step):
    """Kernels of this library launched by one step (CUPTI trace of one untimed step)."""
    try:
        from torch.profiler import profile, ProfilerActivity
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step.run()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
        ours = [n for n in names if "jolt" in n or n.startswith("k_") or "k_gemm" in n]
        return len(ours), sorted(set(ours))
    except Exception as ex:  # profiler unavailable: no claim
        return None, [f"profiler unavailable: {ex}"]


def rank_workload(name, rank, over):
    """Weak scaling: every rank compresses and decodes its own sequences — the same shape, its own
    seed (no data-path collective)."""
    w = get_workload(name, **over)
    return get_workload(name, seed=w.seed + 1000 * rank, **over) if rank else w


def max_over_ranks(ms, device):
    """The step time of the slowest rank (every rank calls this at the same point)."""
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def e2e_over_ranks(e_ms, err, device):
    """Slowest rank's end-to-end step time; None (with a reason) when any rank's leg failed.
    Every rank calls this at the same point, whatever happened to its own leg."""
    t = max_over_ranks(e_ms if e_ms is not None else float("inf"), device)
    if not math.isfinite(t):
        return None, err or "the end-to-end leg failed on another rank"
    return t, err


def measure(args, w, ratio, dev, world, steps, warmup, peaks, secondary=False):
    """Time `steps` steps of workload w after `warmup` untimed ones (barrier and synchronize on both
    sides, max over ranks). Returns (line fields, step) for the JSON line."""
    from long_context_st_b200 import api
    hbm_peak, tc_burst, tc_sust, peak_src = peaks
    step = Step(w, ratio, dev, exact=args.exact and not secondary, cells_per_pass=args.cells_per_pass)
    torch.cuda.synchronize()
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    n_kernels, kernel_names = (None, []) if (args.no_count or secondary) else count_kernels(step)
    names = ["start", "analyzed", "allocated", "compressed", "decoded"]
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in names} for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    api.stats_read(reset=True)
    api.stats_enable(True)
    with Clocks(dev.index) as clk:
        t_start.record()
        for i in range(steps):
            if args.nvtx:
                torch.cuda.nvtx.range_push("jolt_step")
            step.run(evs[i])
            if args.nvtx:
                torch.cuda.nvtx.range_pop()
        t_end.record()
        torch.cuda.synchronize()
    api.stats_enable(False)
    stats = api.stats_read(reset=True)
    total_ms = t_start.elapsed_time(t_end)
    if world > 1:
        import torch.distributed as dist
        total_ms = max_over_ranks(total_ms, dev)
        dist.barrier()
    ms_step = total_ms / steps
    ph = {k: float(np.mean([e["start"].elapsed_time(e[k]) if k != "start" else 0.0 for e in evs]))
          for k in names}
    t_an = ph["analyzed"]
    t_alloc = ph["allocated"] - ph["analyzed"]
    t_cmp = ph["compressed"] - ph["allocated"]
    t_dec = ph["decoded"] - ph["compressed"]

    tokens = w.batch * w.T
    raw = 2 * w.batch * w.n_layers * w.n_kv * w.T * w.d_h * w.io_bytes
    dbytes, dflops = decode_work(w, step.shape, step.choices)
    _, cache_total = api.cache_layout(step.shape, step.choices)

    def fam_roof(name, bound, peak):
        st = stats[name]
        if not st["launches"] or st["ms"] <= 0:
            return None
        sec = st["ms"] / st["launches"] / 1e3
        if bound == "tensor":
            ach = st["flops"] / st["launches"] / sec / 1e12
            unit = "TFLOP/s"
        else:
            ach = st["bytes"] / st["launches"] / sec / 1e9
            unit = "GB/s"
        r = {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
             "traffic": None, "kernel": name, "launches_per_step": st["launches"] / steps,
             "ms_per_step": st["ms"] / steps, "peak_source": peak_src}
        if bound == "tensor" and st.get("flops_issued", 0.0) > st["flops"]:
            r["issued_tflops"] = st["flops_issued"] / st["launches"] / sec / 1e12
        return r

    def binding(name):
        # a family that reports both flops and bytes is bound by the resource it uses the larger
        # fraction of (the pre-RoPE key rebuild is a tensor-core contraction, the rest streams HBM)
        t = fam_roof(name, "tensor", tc_sust) if stats[name]["flops"] > 0 else None
        h = fam_roof(name, "hbm", hbm_peak) if stats[name]["bytes"] > 0 else None
        if t and h:
            other = h if t["frac"] >= h["frac"] else t
            best = t if t["frac"] >= h["frac"] else h
            best["other"] = {"bound": other["bound"], "achieved": other["achieved"], "peak": other["peak"],
                             "unit": other["unit"], "frac": other["frac"]}
            return best
        return t or h

    fams = ["gemm", "decode_main", "residual"]
    dom = max(fams, key=lambda k: stats[k]["ms"])
    dec = {"context_tokens_per_s": tokens * w.n_layers / (t_dec / 1e3) if t_dec > 0 else None,
           "context_tokens_per_s_per_layer_step": tokens / (t_dec / 1e3) if t_dec > 0 else None,
           "ms": t_dec,
           "hbm_gbs": dbytes / (t_dec / 1e3) / 1e9 if t_dec > 0 else None,
           "alg_bytes": dbytes, "frac_of_hbm": dbytes / (t_dec / 1e3) / 1e9 / hbm_peak if t_dec > 0 else None,
           "tensor_flops": dflops,
           "tensor_tflops": dflops / (t_dec / 1e3) / 1e12 if t_dec > 0 else None,
           # the step's own roofline: the slower of its HBM bytes and its tensor flops
           "roofline_ms": max(dbytes / hbm_peak / 1e6, dflops / tc_sust / 1e9),
           "bound": "tensor" if dflops / tc_sust / 1e9 > dbytes / hbm_peak / 1e6 else "hbm",
           "frac_of_roofline": max(dbytes / hbm_peak / 1e6, dflops / tc_sust / 1e9) / t_dec if t_dec > 0 else None}
    out = {"value": tokens * world / (ms_step / 1e3), "ms_per_step": ms_step,
           "config": {"workload": w.name, "batch": w.batch, "n_layers": w.n_layers,
                      "layers_per_group": w.layers_per_group, "n_kv": w.n_kv, "n_q": w.n_q, "T": w.T,
                      "d_h": w.d_h, "keys_pre_rope": w.keys_pre_rope, "budget_ratio": ratio,
                      "q_cap": step.shape.q_cap, "sketch_cols": step.shape.sketch_cols,
                      "power_iters": step.shape.power_iters, "l2": "inputs larger than L2 (no flush)",
                      "token_svd": "exact" if step.shape.sketch_cols == w.n_cols else "randomized",
                      "cells_per_pass": step.shape.cells_per_pass,
                      "parallelism": f"dp{world}" if world > 1 else "single-gpu"},
           "decode_attn_context_tokens_per_s": dec["context_tokens_per_s"],
           "decode_hbm_gbs": dec["hbm_gbs"], "decode_frac_of_hbm": dec["frac_of_hbm"],
           "compress_raw_gbs": raw / ((t_an + t_alloc + t_cmp) / 1e3) / 1e9,
           "breakdown_ms": {"analyze": t_an, "allocate_host": t_alloc, "compress": t_cmp, "decode": t_dec},
           "compress": {"raw_gbs": raw / ((t_an + t_alloc + t_cmp) / 1e3) / 1e9,
                        "raw_bytes": raw, "cache_bytes": cache_total, "ratio": raw / cache_total},
           "decode": dec, "roofline": binding(dom), "roofline_decode": binding("decode_main"),
           "kernel_stats": {k: {kk: (float(vv) if isinstance(vv, float) else int(vv)) for kk, vv in v.items()}
                            for k, v in stats.items()},
           "allocator_ablation": allocator_ablation(step),
           "clocks": clk.summary(), "choices": sorted(set(map(tuple, step.choices)))}
    if not secondary:
        out["gpu_launches"] = n_kernels * steps if n_kernels is not None else None
        out["kernels"] = kernel_names
    return out, step


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    over = {}
    if args.layers:
        over["n_layers"] = args.layers
    if args.seqlen:
        over["T"] = args.seqlen
    w = get_workload(args.workload, **over)
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() and args.impl == "jolt" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = rank_workload(args.workload, rank, over)
    ratio = args.ratio if args.ratio else (w.budget_ratios[0] if w.budget_ratios else None)
    peaks = load_peaks()
    res, step = measure(args, w, ratio, dev, world, args.steps, max(3, args.warmup), peaks)
    tokens = w.batch * w.T
    line = {"metric": METRIC, "value": res["value"], "unit": "context tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (planted low-rank + noise K/V, seeded)"}
    line.update({k: v for k, v in res.items() if k not in ("value", "ms_per_step")})
    line["layer_grouping"] = None if args.no_grouping else layer_grouping(step)

    # e2e: same step through the C ABI with host buffers: H2D of K and V and D2H of the outputs.
    # Every rank takes the same collective steps whether or not its own leg worked.
    if not args.no_e2e:
        e_ms, err, h2d, d2h = None, None, 0, 0
        n_e2e = max(1, min(args.steps, 3))
        try:
            Kh = step.K.cpu().pin_memory()
            Vh = step.V.cpu().pin_memory()
            outh = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
            Kd = torch.empty_like(step.K)
            Vd = torch.empty_like(step.V)
            h2d = Kh.numel() * Kh.element_size() * 2
            d2h = outh.numel() * outh.element_size()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            step.run(K=Kd, V=Vd, host=(Kh, Vh))
            outh.copy_(step.out, non_blocking=True)
            torch.cuda.synchronize()
        except (RuntimeError, MemoryError) as ex:
            err = str(ex)[:200]
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        if err is None:
            try:
                e0.record()
                for _ in range(n_e2e):
                    # the H2D copies of K and V run inside the analyze call (jolt_analyze_from_host)
                    step.run(K=Kd, V=Vd, host=(Kh, Vh))
                    outh.copy_(step.out, non_blocking=True)
                e1.record()
                torch.cuda.synchronize()
                e_ms = e0.elapsed_time(e1) / n_e2e
            except (RuntimeError, MemoryError) as ex:
                err = str(ex)[:200]
        if world > 1:
            e_ms, err = e2e_over_ranks(e_ms, err, dev)
        if e_ms is not None:
            line["e2e"] = {"value": tokens * world / (e_ms / 1e3), "unit": "context tokens/s",
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                           "steps": n_e2e}
        else:
            line["e2e"] = {"value": None, "unit": "context tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0, "error": err}
        Kh = Vh = Kd = Vd = None

    # CPU oracle on a bounded sample (rank 0, N = 1 only)
    if rank == 0 and world == 1 and not args.no_cpu:
        G = w.n_layers // w.layers_per_group
        ch = {0: step.choices[0], 1: step.choices[1]}
        dt, desc = oracle_sample(w, ch, min(args.cpu_tokens, w.T), step.K, step.V)
        t_full = dt * G * w.batch * (w.T / min(args.cpu_tokens, w.T))
        line["cpu_baseline"] = {"value": tokens / t_full, "unit": "context tokens/s", "cores": cpu_threads(),
                                "kind": "oracle", "sample": desc, "sample_seconds": dt}
    # the metric's other workloads, timed the same way in the same run (decode and compress
    # figures; the headline's buffers are released first)
    also = args.also if args.also is not None else (DEFAULT_ALSO if args.workload == DEFAULT_WORKLOAD else "")
    if also and not (args.layers or args.seqlen):
        step = None
        torch.cuda.empty_cache()
        sec = {}
        for spec in [x for x in also.split(",") if x]:
            name, r = (spec.split(":") + [None])[:2]
            w2 = rank_workload(name, rank, {})
            r2 = float(r) if r else (w2.budget_ratios[0] if w2.budget_ratios else None)
            try:
                res2, st2 = measure(args, w2, r2, dev, world, 3, 3, peaks, secondary=True)
                sec[f"{name}@{r2:g}x" if r2 else name] = {
                    k: res2[k] for k in ("value", "ms_per_step", "config", "decode_attn_context_tokens_per_s",
                                         "decode_hbm_gbs", "decode_frac_of_hbm", "compress_raw_gbs", "breakdown_ms",
                                         "compress", "decode", "roofline", "roofline_decode", "allocator_ablation",
                                         "clocks")}
                sec[f"{name}@{r2:g}x" if r2 else name]["steps"] = 3
            except (RuntimeError, MemoryError) as ex:
                sec[spec] = {"error": str(ex)[:200]}
            st2 = None
            torch.cuda.empty_cache()
        line["workloads"] = sec
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
