"""Benchmark of the Medusa verify step (heads + top-s, tree expansion, tree
attention, acceptance, KV compaction) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Every rank runs its own replica
of the step on its own sequences (data parallel, no collective on the data
path: weak scaling).  Rank 0 prints one JSON line.  `--impl reference` times
the plain fp64 CPU oracle on sampled slices of the same workload.

The timed region is K verify steps back to back, with no event between
them.  The per-kernel figures (heads, tree attention, acceptance) come from
separate loops of back-to-back calls of each entry point after it
(medusa_head_speculative_02_b200.kernel_bench); the dominant kernel of the
step is the `roofline` object.  The other workloads' step rates and kernel
figures follow under `configs`.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from medusa_head_speculative_02_b200.synthetic import CONFIG_ORDER, CONFIGS, gen_inputs  # noqa: E402

# the largest workload that fits one GPU: B = 4 sequences of 32K-token prefixes,
# 256-node trees, d = 6656
DEFAULT_CONFIG = "longctx_b4"
METRIC = "verify steps/s"
KERNEL_CALLS = 50   # back-to-back calls per entry point for the per-kernel figures
EXTRA_STEPS = 50    # timed steps of each of the other workloads
DECODE_STEPS = 128  # chained steps of the decode-loop measurement
SAMPLE_REPS = 50    # timed calls of the sampled-next-token measurement
SHARD_REPS = 50     # timed calls per shard count of the vocabulary-sharded heads
SHARD_COUNTS = (2, 4, 8)
E2E_GRAPH_STEPS = 8  # end-to-end steps per captured CUDA graph


# ---------------------------------------------------------------------------- helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized():
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, seconds_per_rank: float, world: int, device) -> dict:
    """Whole-job throughput: units all ranks processed / max time over ranks."""
    t = max_over_ranks(seconds_per_rank, device)
    return {"seconds": t, "value": units_per_rank * world / t if t > 0 else 0.0}


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


class ClockSampler:
    """nvidia-smi clocks / throttle reasons of this rank's GPU while running."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.bus = None
        try:
            p = torch.cuda.get_device_properties(device_index)
            self.bus = "%08X:%02X:%02X.0" % (getattr(p, "pci_domain_id", 0),
                                              getattr(p, "pci_bus_id", 0),
                                              getattr(p, "pci_device_id", 0))
        except Exception:
            pass
        self.rows, self.proc, self.thread = [], None, None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        rows = [r for r in self.rows if len(r) >= 10]
        if self.bus:
            mine = [r for r in rows if r[1].upper().endswith(self.bus[-7:])]
            rows = mine or rows
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        reasons = set()
        for r in rows:
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                "sw_power_cap"), r[6:10]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- oracle sampler
class OracleSampler:
    """Times the fp64 CPU oracle on bounded slices of one verify step and
    scales each slice by its share of the step (units of that operation)."""

    def __init__(self, cfg, x, vlogits, target_ms: float):
        from oracle import medusa_oracle as O
        self.O, self.cfg = O, cfg
        self.x = {k: v.cpu() for k, v in x.items()}
        self.vlog = vlogits.cpu()
        self.plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
        g = torch.Generator().manual_seed(1)
        self.topk = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.K * cfg.s]
                                 .view(cfg.K, cfg.s) for _ in range(cfg.B)])
        self.tok, _ = O.build_tree(self.plan, self.x["root_tok"], self.topk, self.x["prefix_len"])
        self.u = O.heads_hidden(self.x["h"], self.x["W1"], self.x["b1"], 0, rows=None)
        # (name, full units, slice units); slices sized by a calibration pass
        self.ops = {"stage1": [cfg.K * cfg.d, 64], "stage2": [cfg.K * cfg.V, 512],
                    "topk": [cfg.B * cfg.K, 1], "tree": [1, 1],
                    "attention": [cfg.B * cfg.N * cfg.Hq, 16], "accept": [cfg.B, 1],
                    "compact": [cfg.B, 1]}
        self.times = {k: [] for k in self.ops}
        self.names = list(self.ops)
        self.j = 0
        self._calibrate(target_ms / 1000.0)

    def _run(self, name, n):
        O, c, x = self.O, self.cfg, self.x
        j = self.j
        if name == "stage1":
            k = j % c.K
            lo = (j * n) % c.d
            O.heads_hidden(x["h"], x["W1"], x["b1"], k, rows=np.arange(lo, min(c.d, lo + n)))
        elif name == "stage2":
            k = j % c.K
            lo = (j * n) % c.V
            O.heads_logits(self.u, x["W2"], k, vocab=np.arange(lo, min(c.V, lo + n)))
        elif name == "topk":
            # one (sequence, head) row of V logits; any length-V row costs the same
            O.topk_row(self.vlog[j % c.B, 0], c.s)
        elif name == "tree":
            O.build_tree(self.plan, x["root_tok"], self.topk, x["prefix_len"])
        elif name == "attention":
            rows = [((j + r) % c.B, ((j + r) // c.B) % c.N, (j * 7 + r) % c.Hq) for r in range(n)]
            O.tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], self.plan,
                             1.0 / np.sqrt(c.dh), rows=rows)
        elif name == "accept":
            b = j % c.B
            if c.accept in ("greedy", "both"):
                O.accept_greedy(self.vlog[b:b + 1], self.tok[b:b + 1], self.plan)
            if c.accept in ("typical", "both"):
                O.accept_typical(self.vlog[b:b + 1], self.tok[b:b + 1], self.plan, c.temperature,
                                 c.eps, c.delta)
        elif name == "compact":
            b = j % c.B
            O.kv_compact(x["k_cache"][b:b + 1], x["v_cache"][b:b + 1], x["prefix_len"][b:b + 1],
                         torch.tensor([2]), torch.tensor([[0, 1, 2] + [-1] * (c.K - 2)]))

    def _calibrate(self, target_s):
        for name, (full, n) in self.ops.items():
            t0 = time.perf_counter()
            self._run(name, n)
            dt = time.perf_counter() - t0
            if name in ("stage1", "stage2", "attention") and dt > 0:
                n2 = int(max(1, min(full, n * target_s / dt)))
                self.ops[name][1] = n2

    def step(self):
        name = self.names[self.j % len(self.names)]
        full, n = self.ops[name]
        t0 = time.perf_counter()
        self._run(name, n)
        self.times[name].append((time.perf_counter() - t0) * full / n)
        self.j += 1

    def estimate_step_seconds(self) -> float:
        return sum(statistics.mean(v) for v in self.times.values() if v)

    def sample_desc(self) -> str:
        d = {k: f"{v[1]}/{v[0]}" for k, v in self.ops.items()}
        return ("per step one op slice, round robin; slice/full units: " +
                ", ".join(f"{k} {v}" for k, v in d.items()) +
                "; each op's mean slice time scaled by full/slice units and summed")


def oracle_full_step_seconds(cfg) -> float:
    """Wall time of one whole verify step of the oracle on the host (every
    head logit, every attention row, both acceptance rules where the workload
    has them, the compaction), inputs generated beforehand."""
    from oracle import medusa_oracle as O
    from medusa_head_speculative_02_b200.synthetic import plant_verify_logits
    x = gen_inputs(cfg, "cpu", seed=0)
    t0 = time.perf_counter()
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    logits = O.heads_forward(x["h"], x["W1"], x["b1"], x["W2"])
    tk = O.topk(logits, cfg.s)
    tok, _ = O.build_tree(plan, x["root_tok"], tk, x["prefix_len"])
    O.tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], plan,
                     1.0 / np.sqrt(cfg.dh))
    t1 = time.perf_counter()
    vlog = plant_verify_logits(cfg, plan["parent"], tok, "cpu", 0)   # input, not timed
    t2 = time.perf_counter()
    if cfg.accept in ("greedy", "both"):
        alen, anodes, _ = O.accept_greedy(vlog, tok, plan)
    if cfg.accept in ("typical", "both"):
        alen, anodes, _, _ = O.accept_typical(vlog, tok, plan, cfg.temperature, cfg.eps,
                                              cfg.delta)
    O.kv_compact(x["k_cache"], x["v_cache"], x["prefix_len"], alen, anodes)
    return (t1 - t0) + (time.perf_counter() - t2)


FULL_STEP_WORKLOADS = ("tiny_f32", "7b_b1")


def cpu_baseline(S, seconds: float) -> dict:
    """The oracle on this host: the headline workload extrapolated from timed
    slices, and whole steps of the two smallest workloads measured in full."""
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        S.step()
    est = S.estimate_step_seconds()
    full = {}
    for name in FULL_STEP_WORKLOADS:
        sec = oracle_full_step_seconds(CONFIGS[name])
        full[name] = {"wall_s": sec, "steps_per_s": 1.0 / sec}
    return {"value": 1.0 / est if est > 0 else 0.0, "unit": "steps/s", "cores": blas_threads(),
            "kind": "oracle",
            "method": "extrapolated: each operation timed on a slice of its rows and scaled "
                      "to the whole step (a full step of this workload takes the oracle "
                      f"~{est / 60:.0f} min)",
            "sample": S.sample_desc(), "host_cores_available": cpu_cores(),
            "full_step": dict(full, note="whole oracle steps measured end to end on the same "
                                         "host, not extrapolated")}


# ---------------------------------------------------------------------------- arms
def run_reference(args, cfg, world, rank):
    if rank != 0:
        return 0
    t_setup = time.perf_counter()
    x = gen_inputs(cfg, "cpu", seed=0)
    from oracle import medusa_oracle as O
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    from medusa_head_speculative_02_b200.synthetic import plant_verify_logits
    g = torch.Generator().manual_seed(1)
    topk = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.K * cfg.s].view(cfg.K, cfg.s)
                        for _ in range(cfg.B)])
    tok, _ = O.build_tree(plan, x["root_tok"], topk, x["prefix_len"])
    vlog = plant_verify_logits(cfg, plan["parent"], tok, "cpu", 0)
    budget_s = float(os.environ.get("MEDUSA_REF_BUDGET_S", "150"))
    target_ms = max(2.0, min(40.0, 1000.0 * budget_s / max(1, args.steps + args.warmup)))
    S = OracleSampler(cfg, x, vlog, target_ms)
    for _ in range(args.warmup):
        S.step()
    S.times = {k: [] for k in S.ops}
    t0 = time.perf_counter()
    for _ in range(args.steps):
        S.step()
    wall = time.perf_counter() - t0
    est = S.estimate_step_seconds()
    value = 1.0 / est if est > 0 else 0.0
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": est * 1000.0, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.B, "d": cfg.d, "vocab": cfg.V,
                       "heads": cfg.K, "top_s": cfg.s, "tree_nodes": cfg.N, "q_heads": cfg.Hq,
                       "kv_heads": cfg.Hkv, "head_dim": cfg.dh, "prefix": [cfg.L_lo, cfg.L_hi],
                       "accept": cfg.accept},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                             "sample": S.sample_desc(), "wall_s": wall,
                             "setup_s": t0 - t_setup,
                             "method": "extrapolated: each operation timed on a slice of its "
                                       "rows and scaled to the whole step"},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _source_digest(*paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# kernel -> sources whose change makes a stored DRAM-traffic figure stale
TRAFFIC_SOURCES = {
    "tree_attention": ("medusa_head_speculative_02_b200/csrc/attention_tc.cu",
                       "medusa_head_speculative_02_b200/csrc/common.cuh"),
    "heads": ("medusa_head_speculative_02_b200/csrc/heads_tc.cu",
              "medusa_head_speculative_02_b200/csrc/topk.cu",
              "medusa_head_speculative_02_b200/csrc/common.cuh"),
}


def stored_traffic(workload: str, kernel: str, path: str | None = None):
    """DRAM bytes (read + write) of one call of `kernel` at `workload`, from the
    ncu capture summarised in profiles/dram_traffic.json; None when there is
    none, or when the kernel's sources changed since it was taken."""
    path = path or os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        e = json.load(open(path))[workload][kernel]
    except Exception:
        return None
    if e.get("sources_sha16") != _source_digest(*TRAFFIC_SOURCES[kernel]):
        return None
    return e.get("bytes_per_call")


def kernel_figures(cfg, st, calls, pk) -> dict:
    """Back-to-back loops of the step's entry points on its own tensors."""
    from medusa_head_speculative_02_b200 import kernel_bench as KB
    out = {"heads": KB.time_heads(cfg, st.x, calls, ws=st.ws_heads, pk=pk),
           "tree_attention": KB.time_attention(cfg, st.x, st.tree, calls, ws=st.ws_attn, pk=pk)}
    if cfg.accept in ("greedy", "both"):
        out["accept_greedy"] = KB.time_accept(cfg, st.vlogits, st.tree_tok, st.tree, calls,
                                              typical=False, ws=st.ws_acc, pk=pk)
    if cfg.accept in ("typical", "both"):
        out["accept_typical"] = KB.time_accept(cfg, st.vlogits, st.tree_tok, st.tree, calls,
                                               typical=True, ws=st.ws_acc, pk=pk)
    for r in out.values():
        classify(r, pk)
    return out


def classify(r: dict, pk: dict) -> dict:
    """Adds to a kernel figure the bound that sets its floor (HBM bytes or
    tensor-core flops, whichever takes longer at the peaks), the floor time,
    `frac` against the peak of that bound, `hbm_frac`, and `roofline_frac`
    = floor time / measured time."""
    hbm_frac = r["algorithmic_bytes"] / (r["avg_ms"] / 1e3) / 1e9 / pk["hbm_gbs"]
    t_hbm = r["algorithmic_bytes"] / (pk["hbm_gbs"] * 1e9)
    t_tc = r["algorithmic_flops"] / (pk["bf16_tflops"] * 1e12) if "algorithmic_flops" in r else 0.0
    r["bound"] = "tensor" if t_tc > t_hbm else "hbm"
    r["floor_ms"] = 1e3 * max(t_hbm, t_tc)
    r["hbm_frac"] = hbm_frac
    r["frac"] = r["tensor_frac"] if r["bound"] == "tensor" else hbm_frac
    r["roofline_frac"] = r["floor_ms"] / r["avg_ms"]
    return r


def roofline_of(name: str, r: dict, pk: dict, workload: str) -> dict:
    """The JSON `roofline` object of kernel `name` from its kernel_figures entry."""
    if r["bound"] == "tensor":
        ach, peak, unit = r["tflops"], pk["bf16_tflops"], "TFLOP/s"
    else:
        ach, peak, unit = r["achieved"], pk["hbm_gbs"], "GB/s"
    traffic = stored_traffic(workload, name)
    line = {"kernel": name, "bound": r["bound"], "achieved": ach, "peak": peak, "unit": unit,
            "frac": ach / peak, "traffic": traffic, "peak_src": pk["src"],
            "avg_ms": r["avg_ms"], "calls": r["calls"],
            "algorithmic_bytes": r["algorithmic_bytes"], "floor_ms": r.get("floor_ms"),
            "roofline_frac": r.get("roofline_frac"),
            "timing": f"CUDA events around {r['calls']} back-to-back calls on the launching "
                      f"stream, after the timed steps"}
    if "algorithmic_flops" in r:
        line.update({"algorithmic_flops": r["algorithmic_flops"], "tflops": r["tflops"],
                     "tensor_frac": r["tensor_frac"],
                     "tensor_frac_sustained": r["tensor_frac_sustained"],
                     "hbm_frac": r["hbm_frac"]})
    if traffic:
        line["traffic_over_algorithmic"] = traffic / r["algorithmic_bytes"]
    return line


def time_steps(st, K, dev):
    """Device time of K back-to-back verify steps (barrier + sync both sides)."""
    stream = torch.cuda.current_stream(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(K):
        st.run()
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    return start.elapsed_time(end) / 1000.0


def other_workloads(args, headline, dev, rank, pk) -> dict:
    """Step rate and per-kernel figures of every other workload, one at a time
    (each rank runs its own replica; figures are this rank's)."""
    from medusa_head_speculative_02_b200.step import VerifyStep
    names = CONFIG_ORDER if args.extra_configs == "all" else \
        [n for n in args.extra_configs.split(",") if n and n != "none"]
    res = {}
    for name in names:
        if name == headline:
            continue
        cfg = CONFIGS[name]
        st = VerifyStep(cfg, dev, seed=rank)
        for _ in range(5):
            st.run()
        torch.cuda.synchronize(dev)
        t = time_steps(st, EXTRA_STEPS, dev)
        kern = kernel_figures(cfg, st, KERNEL_CALLS, pk)
        res[name] = {"steps_per_s": EXTRA_STEPS / t, "ms_per_step": 1e3 * t / EXTRA_STEPS,
                     "steps": EXTRA_STEPS, "dtype": cfg.dtype, "batch": cfg.B,
                     "kernels": {k: dict({kk: v[kk] for kk in (
                         "avg_ms", "achieved", "unit", "frac", "bound", "floor_ms",
                         "roofline_frac", "hbm_frac", "tflops", "tensor_frac", "key_chunks",
                         "query_tiles_per_cta") if kk in v},
                         traffic=stored_traffic(name, k) if k in TRAFFIC_SOURCES else None)
                         for k, v in kern.items()}}
        del st
        torch.cuda.empty_cache()
    return res


MULTI_LAYER = ("7b_b1", 32)   # workload and layer count of the multi-layer verification figure
LARGE_BATCH = ("7b_b1", 256)  # workload shape and batch of the compute-bound heads figure


def heads_large_batch_figure(dev, pk) -> dict:
    """The heads at B = 256 sequences with the 7B shapes (d = 4096, V =
    32000, K = 5): tensor-bound GEMMs.  `tflops` counts the method's
    multiply-adds x 2; `executed_tflops` also the second GEMM's doubled
    columns (u as the bf16 hi/lo pair), which is what the tensor pipe runs."""
    from medusa_head_speculative_02_b200 import kernel_bench as KB
    from medusa_head_speculative_02_b200.synthetic import gen_head_inputs
    name, B = LARGE_BATCH
    c = CONFIGS[name].scaled(B=B)
    x = gen_head_inputs(c, dev, 0)
    r = classify(KB.time_heads(c, x, 20, pk=pk), pk)
    exe = 2 * c.B * c.K * c.d * c.d + 2 * (2 * c.B) * c.K * c.V * c.d
    r.update({"workload": f"{name} heads at B = {B}", "batch": B,
              "executed_flops": exe,
              "executed_tflops": exe / (r["avg_ms"] / 1e3) / 1e12,
              "executed_tensor_frac_sustained": exe / (r["avg_ms"] / 1e3) / 1e12
              / pk["bf16_tflops_sustained"],
              "kernel": "heads_big2_kernel (cta_group::2, M = 256, N = 256) x 2 + SiLU + top-s merge"})
    del x
    torch.cuda.empty_cache()
    return r


def multi_layer_figure(dev, rank, pk) -> dict:
    """A verify step through 32 attention layers at the 7B shape: heads,
    tree, one tree-attention call per layer (each on its own queries and
    cache), acceptance, one compaction over every layer's cache."""
    from medusa_head_speculative_02_b200 import kernel_bench as KB
    from medusa_head_speculative_02_b200.step import MultiLayerStep
    name, layers = MULTI_LAYER
    cfg = CONFIGS[name]
    ml = MultiLayerStep(cfg, layers, dev, seed=rank)
    for _ in range(3):
        ml.run()
    torch.cuda.synchronize(dev)
    steps = 20
    barrier()
    t = time_steps(ml, steps, dev)
    prefix_sum = int(ml.st.x["prefix_len"].sum().item())
    ab = KB.attention_bytes(cfg, prefix_sum) * layers
    att_ms = KB.time_calls(lambda i: ml.attention(), 10, device=dev)
    res = {"workload": name, "layers": layers, "steps": steps,
           "steps_per_s": steps / t, "ms_per_step": 1e3 * t / steps,
           "attention_ms_all_layers": att_ms,
           "attention_achieved_gbs": ab / (att_ms / 1e3) / 1e9,
           "attention_frac": ab / (att_ms / 1e3) / 1e9 / pk["hbm_gbs"],
           "launches_per_step": ml.launches_per_step(),
           "note": "one medusa_tree_attention call per layer on its own cache, then one "
                   "medusa_kv_compact_layers over all layers"}
    del ml
    torch.cuda.empty_cache()
    return res


def run_tensor_parallel(args, cfg, world, rank, local):
    """--heads vocab-shard: one batch of B sequences served by all ranks.
    The heads' second projection is split by vocabulary rows (one NCCL
    all-gather of every rank's [values; ids] candidate planes, B * K * s * 8
    bytes per rank, then the merge kernel), the tree attention and the
    compaction by kv-head (Hkv / N heads of every sequence per rank, no
    exchange), the acceptance replicated.  Whole-job throughput = verify
    steps/s of the one batch (strong scaling: the work per step is fixed)."""
    from medusa_head_speculative_02_b200 import kernel_bench as KB
    from medusa_head_speculative_02_b200.sharded import ShardedHeads, shard_w2, vocab_shard
    from medusa_head_speculative_02_b200.step import VerifyStep
    if cfg.Hkv % world or cfg.Hq % world:
        raise SystemExit(f"--heads vocab-shard: {world} ranks must divide the kv-heads ({cfg.Hkv})")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = KB.peaks(ROOT)
    lcfg = cfg.scaled(Hq=cfg.Hq // world, Hkv=cfg.Hkv // world)
    st = VerifyStep(lcfg, dev, seed=0)   # identical heads inputs and verify logits on every rank
    v0, v1 = vocab_shard(cfg.V, world, rank)
    st.x["W2"] = shard_w2(st.x["W2"], world, rank)
    torch.cuda.empty_cache()
    sh = ShardedHeads(st.x["W1"], st.x["b1"], st.x["W2"], cfg.V, cfg.B, cfg.s)
    # the step's heads call becomes this rank's slice + all-gather + merge,
    # writing the same top-s buffers the rest of the step reads
    st.heads = lambda: sh(st.x["h"], out=(st.topk_idx, st.topk_val))
    for _ in range(args.warmup):
        st.run()
    torch.cuda.synchronize(dev)
    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    elapsed_s = time_steps(st, K, dev)
    t = max_over_ranks(elapsed_s, dev)
    attn = classify(KB.time_attention(lcfg, st.x, st.tree, KERNEL_CALLS, ws=st.ws_attn, pk=pk), pk)
    heads = classify(KB.time_heads(lcfg.scaled(V=v1 - v0), st.x, KERNEL_CALLS, pk=pk), pk)
    clk = clocks.stop()
    if rank == 0:
        line = {"metric": METRIC, "value": K / t, "unit": "steps/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": 1e3 * t / K, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": cfg.name, "batch": cfg.B, "d": cfg.d, "vocab": cfg.V,
                           "heads": cfg.K, "top_s": cfg.s, "tree_nodes": cfg.N,
                           "q_heads": cfg.Hq, "kv_heads": cfg.Hkv, "head_dim": cfg.dh,
                           "prefix": [cfg.L_lo, cfg.L_hi], "accept": cfg.accept,
                           "parallelism": f"tp{world}: W2 split by vocabulary (one all-gather of "
                                          f"{cfg.B * cfg.K * cfg.s * 8} B per rank per step), "
                                          f"attention and compaction by kv-head "
                                          f"({cfg.Hkv // world} per rank), acceptance replicated"},
                "tokens_per_s": K / t * cfg.B * (1.0 + st.accept_len.float().mean().item()),
                "roofline": roofline_of("tree_attention", attn, pk, cfg.name + f"/tp{world}"),
                "kernels": {"heads_rank_share": heads, "tree_attention_rank_share": attn},
                "gpu_launches": (st.launches_per_step() + 1) * K,
                "clocks": dict(clk, window="timed steps and the per-kernel loops after them")}
        print(json.dumps(line), flush=True)
    return 0


def run_ours(args, cfg, world, rank, local):
    from medusa_head_speculative_02_b200 import kernel_bench as KB
    from medusa_head_speculative_02_b200.step import PipelinedHostIO, VerifyStep
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = KB.peaks(ROOT)
    st = VerifyStep(cfg, dev, seed=rank)
    for _ in range(args.warmup):
        st.run()
    torch.cuda.synchronize(dev)

    # timed region: K steps back to back; clocks are sampled from just before
    # it to the end of the per-kernel loops that follow
    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    elapsed_s = time_steps(st, K, dev)
    agg = aggregate(K, elapsed_s, world, dev)
    ms_per_step = agg["seconds"] * 1000.0 / K
    alen = st.accept_len.float().mean().item()
    kern = kernel_figures(cfg, st, KERNEL_CALLS, pk)
    clk = clocks.stop()
    dominant = max(("heads", "tree_attention"), key=lambda k: kern[k]["avg_ms"])

    # end to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory (the next step's on a copy stream,
    # overlapped with this step's kernels, its tree K/V slots ahead of the
    # rest) and reads its results back
    io = PipelinedHostIO(st)
    io.capture(E2E_GRAPH_STEPS)     # E2E_GRAPH_STEPS steps per graph launch
    Ke = E2E_GRAPH_STEPS * max(2, K // (8 * E2E_GRAPH_STEPS))
    for _ in range(2):
        io.replay()
    torch.cuda.synchronize(dev)
    barrier()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke // E2E_GRAPH_STEPS):
        io.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e = aggregate(Ke, e0.elapsed_time(e1) / 1000.0, world, dev)

    # Sampled next token on this step's verify rows and accepted paths (one
    # row of V logits per sequence), CUDA events around SAMPLE_REPS calls.
    from medusa_head_speculative_02_b200 import api as _api
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tok_buf = torch.empty(cfg.B, dtype=torch.int32, device=dev)
    for i in range(3):
        _api.medusa_sample_next(st.vlogits, st.accept_len, st.accept_nodes, 0.7, rank, i,
                                out=tok_buf)
    torch.cuda.synchronize(dev)
    s0.record(stream)
    for i in range(SAMPLE_REPS):
        _api.medusa_sample_next(st.vlogits, st.accept_len, st.accept_nodes, 0.7, rank, 3 + i,
                                out=tok_buf)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    sample_ms = s0.elapsed_time(s1) / SAMPLE_REPS

    # Vocabulary-sharded heads, one rank's share of the work for G shards:
    # the replicated first projection, the second over the first (largest)
    # W2 shard, and the merge of G candidate lists, CUDA events around
    # SHARD_REPS calls.  The all-gather between them needs G GPUs and is not
    # in this figure.
    from medusa_head_speculative_02_b200.sharded import shard_offsets, shard_w2, vocab_shard
    sharded = {}
    R = cfg.B * cfg.K
    elt = 4 if cfg.dtype == "f32" else 2
    for G in SHARD_COUNTS:
        v0, v1 = vocab_shard(cfg.V, G, 0)
        if v1 - v0 < cfg.s:
            continue
        W2g = shard_w2(st.x["W2"], G, 0)
        cand = torch.zeros(G, 2, R, cfg.s, dtype=torch.int32, device=dev)
        offs = torch.tensor(shard_offsets(cfg.V, G), dtype=torch.int32, device=dev)
        ws = torch.empty(max(256, _api.heads_workspace_size(cfg.B, cfg.d, v1 - v0, cfg.K, cfg.s,
                                                            st.x["h"].dtype)),
                         dtype=torch.uint8, device=dev)
        outs = (torch.empty(R, cfg.s, dtype=torch.int32, device=dev),
                torch.empty(R, cfg.s, dtype=torch.float32, device=dev))
        pl = (None, cand[0, 1].view(cfg.B, cfg.K, cfg.s),
              cand[0, 0].view(torch.float32).view(cfg.B, cfg.K, cfg.s))

        def one_rank(_i=0):
            _api.medusa_heads_forward(st.x["h"], st.x["W1"], st.x["b1"], W2g, s=cfg.s,
                                      want_logits=False, out=pl, ws=ws)
            _api.medusa_topk_merge_planes(cand, cfg.s, offs, out=outs)

        one_rank()
        cand[1:] = cand[0]          # every shard's list slot holds a real list
        ms = KB.time_calls(one_rank, SHARD_REPS, device=dev)
        nbytes = st.heads_bytes() - elt * cfg.K * (cfg.V - (v1 - v0)) * cfg.d
        sharded[str(G)] = {"avg_ms": ms, "algorithmic_bytes": nbytes,
                           "achieved": nbytes / (ms / 1e3) / 1e9, "vocab_rows": v1 - v0}
        del W2g, cand, ws
    torch.cuda.empty_cache()

    # Multi-step decode: the next token of each step is the next root and its
    # new lengths the next prefix lengths; one step is captured into a CUDA
    # graph and DECODE_STEPS replays run back to back.  Every rank takes the
    # same collective steps whether or not its capture worked.
    dec_err, dec_s, dec_alen = None, 0.0, 0.0
    loop = None
    try:
        from medusa_head_speculative_02_b200.decode import DecodeLoop
        loop = DecodeLoop(cfg, dev, seed=rank, max_steps=DECODE_STEPS)
        loop.capture()
        torch.cuda.synchronize(dev)
    except Exception as ex:  # reported in the JSON line, the main result stands
        dec_err = f"{type(ex).__name__}: {ex}"[:300]
    barrier()
    if dec_err is None:
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(DECODE_STEPS):
            loop.step()
        d1.record(stream)
        torch.cuda.synchronize(dev)
        dec_s = d0.elapsed_time(d1) / 1000.0
        grown = (loop.st.x["prefix_len"].long() - loop._init["prefix_len"].long()).float()
        dec_alen = (grown.mean().item() / DECODE_STEPS) - 1.0
    dec = aggregate(DECODE_STEPS, dec_s if dec_err is None else 1.0, world, dev)
    del loop
    torch.cuda.empty_cache()

    sample_bytes = cfg.B * cfg.V * (4 if cfg.dtype == "f32" else 2)
    hb = st.heads_bytes()
    ab = st.attention_bytes()
    launches = st.launches_per_step()
    io_h2d, io_d2h = io.h2d_bytes(), io.d2h_bytes()
    # the oracle sampler takes host copies of this step's inputs
    sampler = (OracleSampler(cfg, st.x, st.vlogits, target_ms=40.0)
               if rank == 0 and world == 1 and not args.no_cpu_baseline else None)
    del io, st
    torch.cuda.empty_cache()
    extra = other_workloads(args, cfg.name, dev, rank, pk)
    try:
        big = heads_large_batch_figure(dev, pk)
    except Exception as ex:  # reported in the line, the main result stands
        big = {"error": f"{type(ex).__name__}: {ex}"[:300]}
    multi = None
    if not args.no_multi_layer:
        try:
            multi = multi_layer_figure(dev, rank, pk)
        except Exception as ex:  # reported in the line, the main result stands
            multi = {"error": f"{type(ex).__name__}: {ex}"[:300]}

    line = None
    if rank == 0:
        line = {"metric": METRIC, "value": agg["value"], "unit": "steps/s", "n_gpus": world,
                "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
                "config": {"workload": cfg.name, "batch": cfg.B, "d": cfg.d, "vocab": cfg.V,
                           "heads": cfg.K, "top_s": cfg.s, "tree_nodes": cfg.N,
                           "q_heads": cfg.Hq, "kv_heads": cfg.Hkv, "head_dim": cfg.dh,
                           "prefix": [cfg.L_lo, cfg.L_hi], "accept": cfg.accept,
                           "parallelism": f"dp{world} (independent replicas)",
                           "l2": "inputs larger than L2: each step streams "
                                 f"{hb / 1e9:.2f} GB of head weights and "
                                 f"{ab / 1e9:.2f} GB of K/V, evicting the 126 MB L2"},
                "tokens_per_s": agg["value"] * cfg.B * (1.0 + alen),
                "mean_accept_len": alen,
                "roofline": roofline_of(dominant, kern[dominant], pk, cfg.name),
                "kernels": dict(kern, **{
                    "sample_next": {"avg_ms": sample_ms, "temperature": 0.7,
                                    "algorithmic_bytes": sample_bytes,
                                    "achieved": sample_bytes / (sample_ms / 1e3) / 1e9,
                                    "unit": "GB/s",
                                    "note": "one verify row per sequence; latency-bound at "
                                            "small batch"},
                    "heads_large_batch": big,
                    "sharded_heads": {"per_shard_count": sharded, "unit": "GB/s",
                                      "note": "one rank's heads for G vocabulary shards: "
                                              "replicated first projection, its W2 rows, "
                                              "merge of G candidate lists; the all-gather of "
                                              "G * B * K * s * 8 bytes between them is not "
                                              "included (needs G GPUs)"}}),
                "decode_loop": ({"steps": DECODE_STEPS, "cuda_graph": True,
                                 "steps_per_s": dec["value"],
                                 "tokens_per_s": dec["value"] * cfg.B * (1.0 + dec_alen),
                                 "mean_accept_len": dec_alen,
                                 "note": "next token -> next root, new lengths -> next prefix "
                                         "lengths; one captured step replayed per step"}
                                if dec_err is None else {"error": dec_err}),
                "e2e": {"value": e2e["value"], "unit": "steps/s",
                        "h2d_bytes_per_step": io_h2d, "d2h_bytes_per_step": io_d2h,
                        "steps": Ke,
                        "copies": "pinned host -> device every step; the next step's "
                                  "tree K/V slots, then its hidden state, queries, verify "
                                  "logits, roots and lengths, on a copy stream overlapping "
                                  "this step",
                        "launch": f"API calls and copies of {E2E_GRAPH_STEPS} steps captured "
                                  f"once into a CUDA graph, replayed"},
                "gpu_launches": launches * K,
                "clocks": dict(clk, window="timed steps and the per-kernel loops after them"),
                "configs": extra,
                "multi_layer": multi}
    # CPU baseline: the oracle on rank 0 at N = 1 only
    if sampler is not None:
        line["cpu_baseline"] = cpu_baseline(sampler, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--heads", choices=["replicas", "vocab-shard"], default="replicas",
                    help="replicas: every rank serves its own sequences (weak scaling); "
                         "vocab-shard: all ranks serve one batch, heads split by vocabulary "
                         "and attention by kv-head (strong scaling)")
    ap.add_argument("--no-multi-layer", action="store_true",
                    help="skip the multi-layer verification figure")
    ap.add_argument("--extra-configs", default="all",
                    help="other workloads to report under `configs`: all, none, or a "
                         "comma-separated list")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = CONFIGS[args.config]
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, cfg, world, rank)
    # vocab-shard needs a process group even on one rank (G = 1: the whole
    # vocabulary on one GPU, the all-gather a copy)
    use_pg = world > 1 or args.heads == "vocab-shard"
    if use_pg:
        import datetime
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(_free_port()))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        if args.heads == "vocab-shard":
            return run_tensor_parallel(args, cfg, world, rank, local)
        return run_ours(args, cfg, world, rank, local)
    finally:
        if use_pg:
            torch.distributed.destroy_process_group()


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


if __name__ == "__main__":
    sys.exit(main())
