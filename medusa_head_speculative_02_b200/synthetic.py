"""Seeded synthetic inputs for the Medusa verify step (workload shapes only).

This module generates tensors; it holds none of the method's arithmetic.
Both the CUDA library and the CPU oracle consume the tensors it returns, so
parity never depends on two random generators agreeing.  Every tensor draws
from its own ``torch.Generator`` seeded by (seed, tensor id), so the values
do not depend on generation order.

Distributions (the five workload configurations): head weights W1, b1, W2
~ N(0, 0.02^2); hidden state h ~ N(0, 1); Q, K, V ~ N(0, 1); verify logits
~ N(0, sigma^2) with a planted accepted prefix (``plant_verify_logits``);
ragged prefix lengths ~ U[lo, hi] inclusive; root tokens ~ U[0, V).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class MedusaConfig:
    name: str
    dtype: str          # "f32" or "bf16": storage/compute dtype of the path
    B: int              # sequences
    d: int              # model dim
    V: int              # vocab
    K: int              # Medusa heads
    s: int              # top-s per head
    N: int              # tree nodes, root included
    Hq: int             # query heads
    Hkv: int            # kv heads
    dh: int             # head dim
    L_lo: int           # prefix length range (inclusive); fixed when lo == hi
    L_hi: int
    sigma: float = 1.0  # verify-logit std
    accept: str = "greedy"   # "greedy", "typical" or "both"
    temperature: float = 0.7
    eps: float = 0.09
    delta: float = 0.6
    plant_p: float = 0.4     # Geometric(p) planted accept length
    boost: float = 8.0
    headroom: int = 0        # extra cache slots (room for the prefix to grow across steps)

    @property
    def Lcap(self) -> int:
        return self.L_hi + self.N + self.headroom

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "MedusaConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny_f32": MedusaConfig("tiny_f32", "f32", B=1, d=256, V=1024, K=4, s=3, N=16,
                             Hq=4, Hkv=4, dh=64, L_lo=128, L_hi=128),
    "7b_b1": MedusaConfig("7b_b1", "bf16", B=1, d=4096, V=32000, K=5, s=10, N=64,
                          Hq=32, Hkv=32, dh=128, L_lo=2048, L_hi=2048),
    "13b_b8": MedusaConfig("13b_b8", "bf16", B=8, d=5120, V=32000, K=5, s=10, N=64,
                           Hq=40, Hkv=40, dh=128, L_lo=1024, L_hi=4096),
    "8b_gqa_b16": MedusaConfig("8b_gqa_b16", "bf16", B=16, d=4096, V=128256, K=5, s=8,
                               N=128, Hq=32, Hkv=8, dh=128, L_lo=8192, L_hi=8192,
                               sigma=1.5, accept="typical", temperature=0.7),
    "longctx_b4": MedusaConfig("longctx_b4", "bf16", B=4, d=6656, V=32000, K=5, s=3,
                               N=256, Hq=52, Hkv=52, dh=128, L_lo=32768, L_hi=32768,
                               accept="both"),
}
CONFIG_ORDER = ["tiny_f32", "7b_b1", "13b_b8", "8b_gqa_b16", "longctx_b4"]

# tensor ids (distinct generator streams)
_TID = dict(h=1, W1=2, b1=3, W2=4, root=5, L=6, q=7, k=8, v=9, vlog=10, plant=11)


def generator(seed: int, tid: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + tid * 7919 + 17)
    return g


def randn(shape, std: float, dtype, seed: int, tid: int, device,
          chunk_elems: int = 1 << 28) -> torch.Tensor:
    """N(0, std^2) rounded once to ``dtype``; generated in chunks along dim 0."""
    g = generator(seed, tid, device)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for lo in range(0, n, chunk_elems):
        hi = min(n, lo + chunk_elems)
        tmp = torch.randn(hi - lo, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[lo:hi].copy_(tmp)
    return out


def gen_head_inputs(cfg: MedusaConfig, device="cpu", seed: int = 0) -> dict:
    """Inputs of the heads and the tree expansion: h, W1, b1, W2, root_tok."""
    dt = cfg.torch_dtype
    x = {}
    x["h"] = randn((cfg.B, cfg.d), 1.0, dt, seed, _TID["h"], device)
    x["W1"] = randn((cfg.K, cfg.d, cfg.d), 0.02, dt, seed, _TID["W1"], device)
    x["b1"] = randn((cfg.K, cfg.d), 0.02, dt, seed, _TID["b1"], device)
    x["W2"] = randn((cfg.K, cfg.V, cfg.d), 0.02, dt, seed, _TID["W2"], device)
    g = generator(seed, _TID["root"], device)
    x["root_tok"] = torch.randint(0, cfg.V, (cfg.B,), generator=g, device=device,
                                  dtype=torch.int64).to(torch.int32)
    return x


def gen_attention_inputs(cfg: MedusaConfig, device="cpu", seed: int = 0) -> dict:
    """Inputs of the tree attention and the compaction: prefix_len, q, k_cache,
    v_cache (the same values gen_inputs gives for the same seed)."""
    dt = cfg.torch_dtype
    x = {}
    g = generator(seed, _TID["L"], device)
    x["prefix_len"] = torch.randint(cfg.L_lo, cfg.L_hi + 1, (cfg.B,), generator=g,
                                    device=device, dtype=torch.int64).to(torch.int32)
    x["q"] = randn((cfg.B, cfg.N, cfg.Hq, cfg.dh), 1.0, dt, seed, _TID["q"], device)
    x["k_cache"] = randn((cfg.B, cfg.Lcap, cfg.Hkv, cfg.dh), 1.0, dt, seed, _TID["k"], device)
    x["v_cache"] = randn((cfg.B, cfg.Lcap, cfg.Hkv, cfg.dh), 1.0, dt, seed, _TID["v"], device)
    return x


def gen_inputs(cfg: MedusaConfig, device="cpu", seed: int = 0) -> dict:
    """All inputs of one verify step except the verify logits."""
    x = gen_head_inputs(cfg, device, seed)
    x.update(gen_attention_inputs(cfg, device, seed))
    return x


def planted_walk(cfg: MedusaConfig, parent, seed: int = 0) -> list[list[int]]:
    """Per sequence, the node path (root first) along which logits get boosted.

    Planted length A ~ Geometric(p) counted as failures before the first
    success (support 0, 1, ...), capped at K; from the root a child is picked
    uniformly at each step until depth A or a leaf.
    """
    parent = [int(p) for p in parent]
    children = [[] for _ in parent]
    for n, p in enumerate(parent):
        if p >= 0:
            children[p].append(n)
    g = generator(seed, _TID["plant"], "cpu")
    paths = []
    for _ in range(cfg.B):
        A = 0
        while A < cfg.K and torch.rand((), generator=g).item() >= cfg.plant_p:
            A += 1
        path = [0]
        while len(path) - 1 < A and children[path[-1]]:
            ch = children[path[-1]]
            path.append(ch[int(torch.randint(0, len(ch), (), generator=g).item())])
        paths.append(path)
    return paths


def plant_verify_logits(cfg: MedusaConfig, parent, tree_tok, device="cpu",
                        seed: int = 0) -> torch.Tensor:
    """Verify logits [B][N][V] ~ N(0, sigma^2), +boost on l[b][parent][tok[child]]
    for every step parent->child of the planted walk, then rounded to the
    storage dtype.  ``parent``/``tree_tok`` describe the tree being verified."""
    tok = torch.as_tensor(tree_tok).to("cpu").long()
    logits = randn((cfg.B, cfg.N, cfg.V), cfg.sigma, torch.float32, seed,
                   _TID["vlog"], device)
    for b, path in enumerate(planted_walk(cfg, parent, seed)):
        for par, child in zip(path[:-1], path[1:]):
            logits[b, par, int(tok[b, child])] += cfg.boost
    return logits.to(cfg.torch_dtype)
