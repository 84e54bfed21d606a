"""Benchmark of one Medusa verification step (heads + top-k, tree build, tree
attention, posterior, KV compaction) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-graph]

A step is one ``medusa_step`` call over one batch of synthetic inputs already
resident in HBM (the Vicuna-7B-shaped batch-1 workload by default).  Each
rank runs its own replica (sequences are independent, so the path shards
with no exchange: weak scaling).  Rank 0 prints one JSON line.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only) and prints the same metric.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

REPO = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, REPO)

METRIC = "Medusa step µs (heads+tree-attn+posterior) at 7B shape; % of HBM roofline"
NOMINAL_HBM_GBS = 8000.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default=None)
    p.add_argument("--no-graph", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true",
                   help="skip the timing of the base model's forward over the tree (tree_decoding)")
    p.add_argument("--shrink", default=None,
                   help="a smaller variant of the workload for profiling one kernel on a small case, "
                        "e.g. layers=1 (comma-separated field=value; the line's config names the variant)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(REPO, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def subseeds(name):
    path = os.path.join(REPO, "tests", "golden", "subseeds.json")
    if os.path.exists(path):
        d = json.load(open(path))
        if name in d:
            return d[name]["sub_h"], d[name]["sub_logits"]
    return 0, 0


L2_BYTES = 126 * 1024 * 1024


def l2_note(nbytes):
    """How the timed loop stands to the 126 MB L2 (no flush is done either way)."""
    if nbytes > L2_BYTES:
        return "inputs larger than L2 (%.2f GB read per step vs 126 MB L2); no flush" % (nbytes / 1e9)
    return ("inputs fit in L2 (%.1f MB read per step vs 126 MB L2); no flush, so steps after the first "
            "read from L2: a latency-bound case, not an HBM measurement" % (nbytes / 1e6))


def workload_config(w, graph=None):
    cfg = {"workload": w.name, "B": w.B, "d": w.d, "V": w.V, "K": w.K, "topk": w.topk, "T": w.T,
           "layers": w.layers, "H": w.H, "hd": w.hd,
           "L": int(w.prefix) if w.prefix is not None else list(w.prefix_range),
           "mode": w.modes[0], "metric_bytes": w.metric_bytes(), "l2": l2_note(w.metric_bytes())}
    if graph is not None:
        cfg["graph"] = graph
    return cfg


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# oracle on a bounded sample (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------


class OracleSample:
    """The fp64 oracle on one bounded sample of a step, extrapolated to a full step.

    Heads, top-k, candidate assembly and the posterior run in full; tree
    attention and KV compaction run on ``n_slices`` (layer, sequence, head)
    slices spread over the cache and are scaled by total/sampled slices.
    """

    def __init__(self, w, n_slices=8):
        import numpy as np
        import oracle.medusa_oracle as O
        from synth import inputs as I
        self.np, self.O, self.I, self.w = np, O, I, w
        sub_h, sub_l = subseeds(w.name)
        self.tr = O.tree_tables(O.ranksum_choices(w.K, w.topk, w.n_nodes), w.K, w.topk)
        self.h = I.values(I.hidden(w, sub_h))
        self.b1 = I.values(I.b1(w))
        self.W1 = [I.values(I.w1(w, k)) for k in range(w.K)]
        self.Wo = [I.values(I.wout(w, k)) for k in range(w.K)]
        self.root = I.root_tokens(w)
        self.lens = w.prefix_lens()
        total = w.layers * w.B * w.H
        rng = np.random.default_rng(0)
        picks = sorted(set([0, total - 1] + list(rng.choice(total, size=min(total, n_slices) - 2, replace=False))))
        self.slices = []
        for s in picks:
            e, lb = s % w.H, s // w.H
            l, b = lb // w.B, lb % w.B
            n = int(self.lens[b]) + w.T
            self.slices.append((l, b, e, I.q_slice(w, l, b, e), I.values(I.kv_slice(w, "k", l, b, e, n)),
                                I.values(I.kv_slice(w, "v", l, b, e, n))))
        self.scale_slices = total / len(self.slices)
        self.sub_l = sub_l
        self.logits = None
        self.cores = 1
        self.sample_times = []      # measured seconds of each sampled step, before the scaling
        self.desc = (f"heads, top-k, tree and posterior in full; attention and KV compaction on "
                     f"{len(self.slices)} of {total} (layer, seq, head) slices, scaled x{self.scale_slices:.0f}; "
                     f"fp64, 1 BLAS thread")

    def step_seconds(self):
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            return self._step_seconds()

    def _step_seconds(self):
        np, O, w = self.np, self.O, self.w
        t0 = time.perf_counter()
        zs = [O.medusa_head_one(self.h, self.W1[k], self.b1[k], self.Wo[k])[1] for k in range(w.K)]
        z = np.stack(zs, 1)
        ids, _ = O.topk_desc(z, w.topk)
        toks, cand, _ = O.build_tree(self.tr, self.root, ids, self.lens)
        t_full = time.perf_counter() - t0
        if self.logits is None:      # input synthesis, not timed
            self.logits = self.I.base_logits(w, toks, self.tr["parent"], self.sub_l)
        t1 = time.perf_counter()
        post = O.evaluate_posterior(self.tr, self.logits, cand, w.modes[0], w.temperature, w.eps, w.alpha)
        t_full += time.perf_counter() - t1
        t2 = time.perf_counter()
        for (l, b, e, q, k, v) in self.slices:
            O.tree_attention_slice(self.tr, q, k, v, int(self.lens[b]), O.attention_scale(w.hd))
            a = int(post["accept_len"][b])
            L = int(self.lens[b])
            rows = [L + int(self.tr["retrieve"][post["best_path"][b], j]) for j in range(a + 1)]
            k2, v2 = k.copy(), v.copy()
            k2[L:L + a + 1] = k[rows]
            v2[L:L + a + 1] = v[rows]
        t_sample = time.perf_counter() - t2
        self.sample_times.append(t_full + t_sample)
        return t_full + t_sample * self.scale_slices


def expected_launches(w, T):
    """Kernel launches of one medusa_step by the library's launch plan: the heads
    (one launch per group of <= 4 sequences on the CUDA cores at batch 1 or
    fp32, two per pass of <= 16 sequences on the tensor cores), tree attention
    (one launch, two when a tree above 64 tokens leaves 1-64 rows after its
    128-row groups) and the posterior with the compaction (one)."""
    if w.dtype == "bf16" and w.B >= 2 and w.d % 128 == 0:
        heads = 2 * ((w.B + 15) // 16)
    else:
        heads = (w.B + 3) // 4
    attn = 1
    if w.dtype == "bf16" and w.hd == 128 and T > 64 and 0 < T % 128 <= 64:
        attn = 2
    return heads + attn + 1


def _kernel_short_name(mangled):
    """The innermost identifier of an Itanium-mangled kernel name (the kernel's own name)."""
    if not mangled.startswith("_Z"):
        return mangled
    i, last = 2, mangled
    if i < len(mangled) and mangled[i] == "N":
        i += 1
    while i < len(mangled) and mangled[i].isdigit():
        j = i
        while j < len(mangled) and mangled[j].isdigit():
            j += 1
        n = int(mangled[i:j])
        last = mangled[j:j + n]
        i = j + n
    return last


def graph_kernels(g):
    """Names of the kernel nodes of a captured CUDA graph (kept with keep_graph=True), in
    node order; None when the driver API cannot be queried."""
    try:
        from cuda.bindings import driver as drv
        graph = drv.CUgraph(int(g.raw_cuda_graph()))
        err, _, n = drv.cuGraphGetNodes(graph, 0)
        if err != drv.CUresult.CUDA_SUCCESS:
            return None
        err, nodes, n = drv.cuGraphGetNodes(graph, n)
        if err != drv.CUresult.CUDA_SUCCESS:
            return None
        names = []
        for node in nodes:
            err, ty = drv.cuGraphNodeGetType(node)
            if err != drv.CUresult.CUDA_SUCCESS:
                return None
            if ty != drv.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
                continue
            name = "?"
            try:
                err, p = drv.cuGraphKernelNodeGetParams(node)
                if err == drv.CUresult.CUDA_SUCCESS:
                    if int(p.func):
                        err, nm = drv.cuFuncGetName(p.func)
                    else:
                        err, nm = drv.cuKernelGetName(p.kern)
                    if err == drv.CUresult.CUDA_SUCCESS:
                        name = _kernel_short_name(nm.decode() if isinstance(nm, bytes) else str(nm))
            except Exception:
                pass
            names.append(name)
        return names
    except Exception as ex:
        print(f"# graph node query failed: {ex}", file=sys.stderr)
        return None


def reduce_max(x, world, device):
    """The largest of a per-rank scalar over all ranks (every rank receives it)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(a, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    samp = OracleSample(w)
    for _ in range(a.warmup):
        samp.step_seconds()
    times = [samp.step_seconds() for _ in range(a.steps)]
    us = statistics.median(times) * 1e6
    line = {"metric": METRIC, "impl": "reference", "value": us, "unit": "us", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            # the value is a full step's time extrapolated from a sampled one (see "sample")
            "extrapolated": True, "measured_sample_us": statistics.median(samp.sample_times) * 1e6,
            "cpu_baseline": {"value": us, "unit": "us", "cores": samp.cores, "host_cores": os.cpu_count(),
                             "kind": "oracle", "sample": samp.desc},
            "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def run_ours(a, w):
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev_index = torch.cuda.current_device()

    import importlib.util
    spec = importlib.util.spec_from_file_location("medusa_b200_build",
                                                  os.path.join(REPO, "speculative_decoding_heads_b200", "_build.py"))
    bmod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bmod)
    if rank == 0 or world == 1:
        bmod.build_all()
    if world > 1:
        dist.barrier()
    import speculative_decoding_heads_b200 as mb
    from synth import device, workloads as W

    sub_h, sub_l = subseeds(w.name)
    choices = mb.medusa_tree_choices_ranksum(w.K, w.topk, w.n_nodes)
    tree = mb.Tree(choices, w.K, w.topk)
    t = device.materialise(w, sub_h=sub_h, sub_logits=sub_l, with_head_logits=False)
    device.tree_outputs(t, w.B, tree.T, tree.P, tree.D)
    mode = mb.MEDUSA_TYPICAL if w.modes[0] == "typical" else mb.MEDUSA_GREEDY
    args = mb.make_step_args(tree, t, mode, w.temperature, w.eps, w.alpha)
    ws = mb.workspace(mb.medusa_step_workspace_size(args))
    # Plant head/base agreement once the tree tokens are known (input synthesis).
    hws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], hws)
    mb.medusa_build_tree(tree, t["root_tokens"], t["topk_ids"], t["seq_lens"], t["tree_tokens"], t["candidates"],
                         t["position_ids"])
    parent = device.parent_tensor(tree.tables()["parent"])
    device.plant(t["base_logits"], t["tree_tokens"], parent, w.agreement, w.seed + 7919 * sub_l)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    launches_per_step = expected_launches(w, tree.T)
    kernels = None

    def step():
        t["seq_lens"].copy_(t["seq_lens0"])
        mb.medusa_step(args, ws)

    with torch.cuda.stream(stream):
        for _ in range(max(3, a.warmup)):
            step()
    torch.cuda.synchronize()
    st, det = mb.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} detail {det} after warm-up")

    graph = None
    if not a.no_graph:
        try:
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g, stream=stream):
                step()
            g.instantiate()
            graph = g
            kernels = graph_kernels(g)
            if kernels is not None:
                launches_per_step = len(kernels)
            with torch.cuda.stream(stream):
                for _ in range(a.warmup):
                    graph.replay()
            torch.cuda.synchronize()
        except Exception as ex:   # capture not possible: time eager launches
            print(f"# graph capture failed, timing eager launches: {ex}", file=sys.stderr)
            graph = None
            torch.cuda.synchronize()

    def run_k(k):
        with torch.cuda.stream(stream):
            for _ in range(k):
                graph.replay() if graph is not None else step()

    # ---- timed region --------------------------------------------------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev_index)
    with sampler:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        run_k(a.steps)
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ms = reduce_max(ev0.elapsed_time(ev1) / a.steps, world, "cuda")
    clocks = sampler.summary()
    st, det = mb.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} detail {det} after the timed region")

    # ---- per-step distribution, graph replay and eager launches side by side ----
    def per_step_pair(fns, k):
        # The launch forms alternate step by step, so clock and power drift
        # over the run affects both alike.
        evs = {n: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
               for n in fns}
        with torch.cuda.stream(stream):
            for i in range(k):
                for n, fn in fns.items():
                    evs[n][i][0].record(stream)
                    fn()
                    evs[n][i][1].record(stream)
        torch.cuda.synchronize()
        out = {}
        for n in fns:
            xs = sorted(e0.elapsed_time(e1) * 1e3 for e0, e1 in evs[n])
            out[n] = {"mean": statistics.mean(xs), "median": statistics.median(xs), "min": xs[0],
                      "p90": xs[min(k - 1, int(round(0.9 * (k - 1))))], "n": k}
        return out

    dist_steps = max(a.steps, 20)
    forms = {"eager": step}
    if graph is not None:
        forms["graph"] = graph.replay
    step_us = per_step_pair(forms, dist_steps)
    step_us["note"] = "graph and eager steps alternate"

    # ---- per-stage breakdown (standalone calls, CUDA events on the launching stream) ----
    peak, peak_kind = load_peaks()
    stage = {}
    reps = max(5, min(a.steps, 30))
    with torch.cuda.stream(stream):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        acc = [0.0] * 5
        attn_ws = mb.workspace(mb.medusa_attention_workspace_size(tree, w.layers, w.B, w.H, w.hd,
                                                                   mb.MEDUSA_BF16 if w.dtype == "bf16" else mb.MEDUSA_F32))
        pws = mb.workspace(mb.medusa_posterior_workspace_size(tree, w.B))
        for _ in range(reps):
            t["seq_lens"].copy_(t["seq_lens0"])
            # A spin ahead of the stages keeps the host ahead of the GPU, so the
            # events bracket each stage's kernels, not the host's launch latency.
            torch.cuda._sleep(2_000_000)
            evs[0].record(stream)
            mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], hws)
            evs[1].record(stream)
            mb.medusa_build_tree(tree, t["root_tokens"], t["topk_ids"], t["seq_lens"], t["tree_tokens"],
                                 t["candidates"], t["position_ids"])
            evs[2].record(stream)
            mb.medusa_tree_attention(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], w.hd ** -0.5,
                                     t["attn_out"], attn_ws)
            evs[3].record(stream)
            mb.medusa_evaluate_posterior(tree, t["base_logits"], t["candidates"], mode, t["best_path"],
                                         t["accept_len"], t["accepted_tokens"], t["next_token"], pws,
                                         w.temperature, w.eps, w.alpha)
            evs[4].record(stream)
            mb.medusa_accept_kv(tree, t["k_cache"], t["v_cache"], t["seq_lens"], t["best_path"], t["accept_len"])
            evs[5].record(stream)
            torch.cuda.synchronize()
            for i in range(5):
                acc[i] += evs[i].elapsed_time(evs[i + 1])
    names = ["heads_topk", "build_tree", "tree_attention", "posterior", "accept_kv"]
    stage = {n: acc[i] / reps * 1e3 for i, n in enumerate(names)}
    esz = 2 if w.dtype == "bf16" else 4
    head_bytes = w.K * (w.d * w.d + w.d + w.V * w.d) * esz
    kv_bytes = w.metric_bytes() - head_bytes
    # Algorithmic bytes: the head weights once per step, whatever the batch.
    heads_gbs = head_bytes / (stage["heads_topk"] * 1e-6) / 1e9
    attn_gbs = kv_bytes / (stage["tree_attention"] * 1e-6) / 1e9
    traffic = None
    tpath = os.path.join(REPO, "profiles", "heads_topk_traffic.json")
    if os.path.exists(tpath):
        tj = json.load(open(tpath))
        if tj.get("workload") == w.name and tj.get("kernel_rev") == kernel_revision():
            traffic = tj.get("dram_bytes_per_launch")

    peak_desc = (f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                 else "fallback 6650 GB/s")
    heads_line = {"bound": "hbm", "kernel": "heads_topk", "achieved": heads_gbs, "peak": peak, "peak_kind": peak_desc,
                  "unit": "GB/s", "frac": heads_gbs / peak, "traffic": traffic,
                  "algorithmic_bytes_per_launch": head_bytes}
    attn_line = {"bound": "hbm", "kernel": "tree_attention", "achieved": attn_gbs, "peak": peak,
                 "peak_kind": peak_desc, "unit": "GB/s", "frac": attn_gbs / peak, "traffic": None,
                 "algorithmic_bytes_per_launch": kv_bytes}

    # ---- end to end through the public API with host buffers ----------
    e2e = None
    if not a.no_e2e:
        pin = lambda x: x.cpu().pin_memory()
        host_in = {"h": pin(t["h"]), "root_tokens": pin(t["root_tokens"]), "seq_lens": pin(t["seq_lens0"]),
                   "q": pin(t["q"]), "base_logits": pin(t["base_logits"])}
        lens = t["seq_lens0"].cpu()
        kt = torch.stack([t["k_cache"][:, b, :, int(lens[b]):int(lens[b]) + w.T] for b in range(w.B)], 1)
        vt = torch.stack([t["v_cache"][:, b, :, int(lens[b]):int(lens[b]) + w.T] for b in range(w.B)], 1)
        host_in["k_tree"], host_in["v_tree"] = pin(kt), pin(vt)
        host_out = {k: torch.empty_like(t[k], device="cpu").pin_memory()
                    for k in ("best_path", "accept_len", "accepted_tokens", "next_token", "seq_lens")}
        h2d = sum(x.numel() * x.element_size() for x in host_in.values())
        d2h = sum(x.numel() * x.element_size() for x in host_out.values())
        e_ms = []
        for i in range(a.warmup + a.steps):
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            mb.medusa_step_host(args, ws, host_in, host_out, stream)
            s1.record(stream)
            s1.synchronize()
            if i >= a.warmup:
                e_ms.append(s0.elapsed_time(s1))
        e_ms_max = reduce_max(statistics.mean(e_ms), world, "cuda")
        e2e = {"value": e_ms_max * 1e3, "unit": "us", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # ---- the base model's forward over the tree (tree_decoding) -------
    decode = None
    if not a.no_decode and w.dtype == "bf16" and w.hd == 128 and w.d // 128 == w.H and w.d in VICUNA_FFN:
        decode = time_tree_decode(a, w, t, tree, mb, stream, peak, world)

    # ---- CPU baseline (rank 0, N = 1 only) -----------------------------
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        samp = OracleSample(w)
        secs = [samp.step_seconds() for _ in range(2)]
        cpu = {"value": min(secs) * 1e6, "unit": "us", "cores": samp.cores, "host_cores": os.cpu_count(),
               "kind": "oracle", "sample": samp.desc, "extrapolated": True}

    if world > 1:
        dist.barrier()
        del graph
        dist.destroy_process_group()
    if rank != 0:
        return 0
    us = ms * 1e3
    line = {
        "metric": METRIC, "value": us, "unit": "us", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded counter-based generator; Vicuna-shaped random weights and KV)",
        "config": workload_config(w, graph is not None),
        "hbm_roofline_frac_8tbs": w.metric_bytes() / (us * 1e-6) / 1e9 / NOMINAL_HBM_GBS,
        "achieved_step_gbs": w.metric_bytes() / (us * 1e-6) / 1e9,
        "tree_tokens_per_s": world * w.B * w.T / (us * 1e-6),
        "stage_us": stage,
        "step_us": step_us,
        # `roofline` is the dominant kernel's (the larger per-call stage time).
        "roofline": heads_line if stage["heads_topk"] >= stage["tree_attention"] else attn_line,
        "heads_roofline": heads_line,
        "attention_roofline": attn_line,
        "tree_decode": decode,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * a.steps,
        "launches_per_step": {"count": launches_per_step,
                              "source": "kernel nodes of the captured step graph" if kernels is not None
                              else "launch plan", "kernels": kernels},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


# Feed-forward width of the Vicuna (LLaMA) base models by hidden size.
VICUNA_FFN = {4096: 11008, 5120: 13824, 6656: 17920}


def time_tree_decode(a, w, t, tree, mb, stream, peak, world):
    """The base model's forward over the step's tree tokens (every layer of the workload's shape,
    random bf16 weights from the counter-based generator), timed alone and inside a full
    verification step (heads, tree, forward, posterior, compaction).  Overwrites the tree rows of
    the caches, so it runs after every other measurement."""
    import torch
    from synth import device, gen
    D, F, V, H = w.d, VICUNA_FFN[w.d], w.V, w.H
    bf = torch.bfloat16

    def rnd(shape, tid, sigma):
        x = torch.empty(shape, dtype=bf, device="cuda")
        device.fill_normal(x, w.seed, tid, sigma)
        return x

    s = D ** -0.5
    layers = []
    for l in range(w.layers):
        tid = gen.TID_DECODER + 9 * l
        layers.append({"attn_norm": rnd((D,), tid, 0.1) + 1.0, "Wq": rnd((D, D), tid + 1, s),
                       "Wk": rnd((D, D), tid + 2, s), "Wv": rnd((D, D), tid + 3, s), "Wo": rnd((D, D), tid + 4, s),
                       "mlp_norm": rnd((D,), tid + 5, 0.1) + 1.0, "W_gate": rnd((F, D), tid + 6, s),
                       "W_up": rnd((F, D), tid + 7, s), "W_down": rnd((D, F), tid + 8, F ** -0.5)})
    tid = gen.TID_DECODER + 9 * w.layers
    model = mb.Decoder(rnd((V, D), tid, 1.0), layers, rnd((D,), tid + 1, 0.1) + 1.0, rnd((V, D), tid + 2, s))
    del layers
    torch.cuda.synchronize()
    ntok = w.B * w.T
    logits = torch.empty((ntok, V), device="cuda")
    ws = mb.workspace(mb.medusa_tree_decode_workspace_size(tree, model, w.B))
    lens = t["seq_lens0"]

    def fwd():
        mb.medusa_tree_decode(tree, model, t["tree_tokens"], t["k_cache"], t["v_cache"], lens, logits, ws)

    def full_step():
        # the whole verification step with the base model's forward producing the base logits
        t["seq_lens"].copy_(lens)
        hws = t["_hws"]
        mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], hws)
        mb.medusa_build_tree(tree, t["root_tokens"], t["topk_ids"], t["seq_lens"], t["tree_tokens"],
                             t["candidates"], t["position_ids"])
        mb.medusa_tree_decode(tree, model, t["tree_tokens"], t["k_cache"], t["v_cache"], t["seq_lens"], logits, ws)
        mb.medusa_evaluate_posterior(tree, logits.view(w.B, w.T, V), t["candidates"], mb.MEDUSA_GREEDY, t["best_path"],
                                     t["accept_len"], t["accepted_tokens"], t["next_token"], t["_pws"])
        mb.medusa_accept_kv(tree, t["k_cache"], t["v_cache"], t["seq_lens"], t["best_path"], t["accept_len"])

    # plain decoding's step for comparison: the base model's forward over one token per sequence
    root_tree = mb.Tree([], 1, 1)
    one_tok = t["tree_tokens"][:, :1].contiguous()
    one_logits = torch.empty((w.B, V), device="cuda")
    one_ws = mb.workspace(mb.medusa_tree_decode_workspace_size(root_tree, model, w.B))

    def one_token():
        mb.medusa_tree_decode(root_tree, model, one_tok, t["k_cache"], t["v_cache"], lens, one_logits, one_ws)

    t["_hws"] = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    t["_pws"] = mb.workspace(mb.medusa_posterior_workspace_size(tree, w.B))
    res = {}
    with torch.cuda.stream(stream):
        for name, fn in (("forward", fwd), ("full_step", full_step), ("one_token", one_token)):
            for _ in range(max(3, a.warmup)):
                fn()
            torch.cuda.synchronize()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(a.steps + 1)]
            evs[0].record(stream)
            for i in range(a.steps):
                fn()
                evs[i + 1].record(stream)
            torch.cuda.synchronize()
            xs = sorted(evs[i].elapsed_time(evs[i + 1]) * 1e3 for i in range(a.steps))
            res[name] = {"median": statistics.median(xs), "min": xs[0], "p90": xs[min(a.steps - 1, int(0.9 * (a.steps - 1)))]}
    st, det = mb.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} detail {det} after the tree-decode timing")
    wbytes = sum(x.numel() * 2 for ly in model.tensors for x in ly.values()) + model.lm_head.numel() * 2
    kv_bytes = 2 * w.layers * w.H * w.hd * int((w.prefix_lens() + w.T).sum()) * 2
    fwd_us = res["forward"]["median"]
    return {"layers": w.layers, "D": D, "F": F, "V": V, "tokens": ntok, "weights_bytes": wbytes, "kv_bytes": kv_bytes,
            "forward_us": res["forward"], "full_step_us": res["full_step"],
            "one_token_forward_us": res["one_token"],
            # accepted tokens per step (the root included) above which a Medusa step beats plain decoding
            "break_even_tokens_per_step": res["full_step"]["median"] / res["one_token"]["median"],
            "forward_gbs": (wbytes + kv_bytes) / (fwd_us * 1e-6) / 1e9,
            "forward_frac": (wbytes + kv_bytes) / (fwd_us * 1e-6) / 1e9 / peak,
            "note": "random bf16 weights of the base model's shape; the full step's acceptance is meaningless "
                    "with random weights, so tokens per step are not reported; one_token_forward is plain "
                    "decoding's step (one token per sequence at the same cache length)"}


def kernel_revision():
    """Hash of the heads kernel's sources; its ncu traffic figure holds only for that revision."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(REPO, "speculative_decoding_heads_b200", "csrc")
    for f in ("heads.cu", "heads_common.cuh", "common.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


def main():
    a = parse()
    from synth import workloads as W
    w = W.get(a.workload or W.BENCH_WORKLOAD)
    if a.shrink:
        kv = dict(x.split("=") for x in a.shrink.split(","))
        w = W.shrink(w, name=f"{w.name}[{a.shrink}]", **{k: int(v) for k, v in kv.items()})
    if a.impl == "reference":
        return run_reference(a, w)
    return run_ours(a, w)


if __name__ == "__main__":
    sys.exit(main())
