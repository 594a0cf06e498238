"""Per-call timing of the library's entry points on a workload, and the
algorithmic work each call has to do.

Each entry point is called back to back ``calls`` times on one stream with
one CUDA event before the first call and one after the last, so no event
sits between the kernels of consecutive calls.  Inputs smaller than about
three times the L2 cache are rotated through enough copies that every call
reads its operands from HBM.

Command line (one entry point alone, e.g. for a profiler capture of one
launch):

    python -m medusa_head_speculative_02_b200.kernel_bench \\
        --config longctx_b4 --kernel attention --calls 3 [--batch B]

``--batch`` runs the workload with fewer sequences (a slice of it: every
sequence is an independent unit of the same size).  Prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

import torch

from . import api
from .synthetic import (CONFIGS, MedusaConfig, gen_attention_inputs, gen_head_inputs,
                        plant_verify_logits)

L2_BYTES = 126 * 2 ** 20
ROTATE_BYTES = 3 * L2_BYTES


# ---------------------------------------------------------------- algorithmic work per call
def heads_bytes(c: MedusaConfig) -> int:
    """Weights (W1, b1, W2), hidden state and the top-s output of one heads call."""
    e = 4 if c.dtype == "f32" else 2
    return e * (c.K * c.d * c.d + c.K * c.d + c.K * c.V * c.d + c.B * c.d) + 8 * c.B * c.K * c.s


def heads_flops(c: MedusaConfig) -> int:
    """Multiply-adds x 2 of both projections (the second one on the bf16 hi/lo
    pair of u counts once: the pair is the arithmetic's own precision choice)."""
    return 2 * c.B * c.K * (c.d * c.d + c.V * c.d)


def attention_bytes(c: MedusaConfig, prefix_sum: int) -> int:
    """K and V of every visible slot (prefix and tree) read once, Q read, O written."""
    e = 4 if c.dtype == "f32" else 2
    kv = 2 * (prefix_sum + c.B * c.N) * c.Hkv * c.dh * e
    return kv + 2 * c.B * c.N * c.Hq * c.dh * e


def attention_flops(c: MedusaConfig, prefix_sum: int) -> int:
    """S = Q K^T and O = P V over every key of a sequence's prefix and tree
    slots, per query row."""
    return 4 * c.Hq * c.N * (prefix_sum + c.B * c.N) * c.dh


def accept_bytes(c: MedusaConfig) -> int:
    """Verify logits read once per acceptance pass."""
    e = 4 if c.dtype == "f32" else 2
    return c.B * c.N * c.V * e


# ---------------------------------------------------------------- timing
def time_calls(fn, calls: int, warmup: int = 3, device=None) -> float:
    """Milliseconds per call of ``fn`` over ``calls`` back-to-back calls."""
    stream = torch.cuda.current_stream(device)
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(calls):
        fn(warmup + i)
    e1.record(stream)
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / calls


def _copies(nbytes: int) -> int:
    return max(1, min(16, math.ceil(ROTATE_BYTES / max(1, nbytes))))


def peaks(root: str | None = None) -> dict:
    """Denominators: MEASURED_PEAKS.json at the repository root when present
    (HBM copy GB/s, cuBLAS bf16 TF/s burst and sustained), else the fallback
    figures measured earlier on the same kind of part."""
    root = root or os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    path = os.path.join(root, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": float(d.get("hbm_gbs", 6650.0)),
                "bf16_tflops": float(d.get("bf16_tflops", 1590.0)),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", 1400.0)),
                "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "src": "fallback"}


def _rates(ms: float, nbytes: int, flops: int | None, pk: dict) -> dict:
    r = {"avg_ms": ms, "algorithmic_bytes": nbytes, "achieved": nbytes / (ms / 1e3) / 1e9,
         "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"]}
    if flops is not None:
        tf = flops / (ms / 1e3) / 1e12
        r.update({"algorithmic_flops": flops, "tflops": tf,
                  "tensor_frac": tf / pk["bf16_tflops"],
                  "tensor_frac_sustained": tf / pk["bf16_tflops_sustained"]})
    return r


def time_heads(c: MedusaConfig, x: dict, calls: int, ws=None, pk=None) -> dict:
    """medusa_heads_forward with fused top-s (no logits), as the step calls it.
    The weights of every bf16 workload exceed the L2 cache several times."""
    pk = pk or peaks()
    dev = x["h"].device
    idx = torch.empty(c.B, c.K, c.s, dtype=torch.int32, device=dev)
    val = torch.empty(c.B, c.K, c.s, dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(256, api.heads_workspace_size(c.B, c.d, c.V, c.K, c.s,
                                                           c.torch_dtype)),
                         dtype=torch.uint8, device=dev)

    def one(_i):
        api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=c.s, want_logits=False,
                                 out=(None, idx, val), ws=ws)

    ms = time_calls(one, calls, device=dev)
    r = _rates(ms, heads_bytes(c), heads_flops(c), pk)
    r.update({"calls": calls, "launches_per_call": 4})
    return r


def time_attention(c: MedusaConfig, x: dict, tree, calls: int, ws=None, pk=None) -> dict:
    """medusa_tree_attention on the workload's cache, rotated through copies
    of the cache when it is smaller than ~3x the L2 cache."""
    pk = pk or peaks()
    dev = x["q"].device
    prefix_sum = int(x["prefix_len"].sum().item())
    nb = attention_bytes(c, prefix_sum)
    n = _copies(nb)
    ks = [x["k_cache"]] + [x["k_cache"].clone() for _ in range(n - 1)]
    vs = [x["v_cache"]] + [x["v_cache"].clone() for _ in range(n - 1)]
    out = torch.empty_like(x["q"])
    if ws is None:
        ws = torch.empty(max(256, api.attention_workspace_size(tree, c.B, c.Hq, c.Hkv, c.dh,
                                                               c.Lcap)),
                         dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(c.dh)

    def one(i):
        api.medusa_tree_attention(x["q"], ks[i % n], vs[i % n], x["prefix_len"], tree, scale,
                                  out=out, ws=ws)

    ms = time_calls(one, calls, device=dev)
    r = _rates(ms, nb, attention_flops(c, prefix_sum), pk)
    r.update({"calls": calls, "cache_copies": n,
              "key_chunks": api.attention_chunks(tree, c.B, c.Hq, c.Hkv, c.dh, c.Lcap,
                                                 c.torch_dtype),
              "query_tiles_per_cta": api.attention_tiles_per_cta(tree, c.B, c.Hq, c.Hkv, c.dh,
                                                                 c.Lcap, c.torch_dtype),
              "launches_per_call": api.attention_launches(tree, c.B, c.Hq, c.Hkv, c.dh, c.Lcap,
                                                          c.torch_dtype)})
    del ks, vs
    return r


def time_accept(c: MedusaConfig, vlogits, tree_tok, tree, calls: int, typical: bool, ws=None,
                pk=None) -> dict:
    """One acceptance pass (verify-row reduction + walk) over the verify logits."""
    pk = pk or peaks()
    dev = vlogits.device
    nb = accept_bytes(c)
    n = _copies(nb)
    vls = [vlogits] + [vlogits.clone() for _ in range(n - 1)]
    outs = (torch.empty(c.B, dtype=torch.int32, device=dev),
            torch.empty(c.B, c.K + 1, dtype=torch.int32, device=dev),
            torch.empty(c.B, dtype=torch.int32, device=dev))
    if ws is None:
        ws = torch.empty(max(256, api.accept_workspace_size(tree, c.B, c.V)), dtype=torch.uint8,
                         device=dev)

    def one(i):
        if typical:
            api.medusa_accept_typical(vls[i % n], tree_tok, tree, c.temperature, c.eps, c.delta,
                                      out=outs, ws=ws)
        else:
            api.medusa_accept_greedy(vls[i % n], tree_tok, tree, out=outs, ws=ws)

    ms = time_calls(one, calls, device=dev)
    r = _rates(ms, nb, None, pk)
    r.update({"calls": calls, "logit_copies": n, "rule": "typical" if typical else "greedy",
              "launches_per_call": 2})
    del vls
    return r


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--config", default="longctx_b4", choices=list(CONFIGS))
    ap.add_argument("--kernel", default="attention",
                    choices=["heads", "attention", "accept_greedy", "accept_typical"])
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--batch", type=int, default=0, help="sequences (0: the workload's)")
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args(argv)
    c = CONFIGS[a.config]
    if a.batch > 0:
        c = c.scaled(B=a.batch)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    tree = api.Tree(c.K, c.s, c.N)
    if a.kernel == "heads":
        r = time_heads(c, gen_head_inputs(c, dev, a.seed), a.calls)
    elif a.kernel == "attention":
        r = time_attention(c, gen_attention_inputs(c, dev, a.seed), tree, a.calls)
    else:
        g = torch.Generator().manual_seed(a.seed)
        tok = torch.randint(0, c.V, (c.B, c.N), generator=g, dtype=torch.int32)
        vlog = plant_verify_logits(c, tree.info()[0], tok, dev, a.seed)
        r = time_accept(c, vlog, tok.to(dev), tree, a.calls, a.kernel == "accept_typical")
    r.update({"config": a.config, "batch": c.B, "kernel": a.kernel})
    print(json.dumps(r), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
