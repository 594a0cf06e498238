"""CPU: the seeded synthetic inputs follow the stated recipe (they stand in
for the trained weights and the benchmark traffic the pages measure with).

Weights N(0, 0.02^2), hidden state and Q/K/V N(0, 1), rounded once to the
storage dtype; prefix lengths in [L_lo, L_hi]; root tokens in [0, V); the
planted accept length A ~ Geometric(p) counted as failures before the first
success, capped at K, walked from the root through uniformly chosen
children; verify logits N(0, sigma^2) plus the boost on l[parent][tok[child]]
along that walk.  Every tensor is a pure function of (seed, tensor id).
"""
import math

import numpy as np
import torch

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200.synthetic import (CONFIGS, MedusaConfig, gen_inputs,
                                                       plant_verify_logits, planted_walk)


def _cfg(**kw):
    base = dict(name="syn", dtype="bf16", B=3, d=256, V=4000, K=5, s=3, N=64, Hq=4, Hkv=2,
                dh=64, L_lo=100, L_hi=300)
    base.update(kw)
    return MedusaConfig(**base)


def test_inputs_are_a_function_of_the_seed():
    c = _cfg()
    a, b, other = gen_inputs(c, "cpu", 5), gen_inputs(c, "cpu", 5), gen_inputs(c, "cpu", 6)
    for k in a:
        assert torch.equal(a[k], b[k]), k
        if a[k].numel() > 8:
            assert not torch.equal(a[k], other[k]), k


def test_value_distributions_and_ranges():
    c = _cfg(d=512, V=8000)
    x = gen_inputs(c, "cpu", 0)
    for k, std in (("W1", 0.02), ("W2", 0.02), ("b1", 0.02), ("h", 1.0), ("q", 1.0),
                   ("k_cache", 1.0), ("v_cache", 1.0)):
        t = x[k].double()
        assert t.dtype == torch.float64 and x[k].dtype == torch.bfloat16
        n = t.numel()
        assert abs(t.mean().item()) < 6 * std / math.sqrt(n), k
        assert abs(t.std().item() / std - 1.0) < max(0.02, 6 / math.sqrt(n)), k
    L = x["prefix_len"]
    assert L.dtype == torch.int32 and int(L.min()) >= c.L_lo and int(L.max()) <= c.L_hi
    r = x["root_tok"]
    assert r.dtype == torch.int32 and int(r.min()) >= 0 and int(r.max()) < c.V
    f = gen_inputs(c.scaled(dtype="f32"), "cpu", 0)
    assert f["W2"].dtype == torch.float32


def test_fixed_prefix_lengths_of_the_workloads():
    for name in ("7b_b1", "8b_gqa_b16", "longctx_b4"):
        c = CONFIGS[name].scaled(d=8, V=16, K=2, s=2, N=4, Hq=1, Hkv=1, dh=8)
        L = gen_inputs(c, "cpu", 0)["prefix_len"]
        assert (L == c.L_hi).all() and c.L_lo == c.L_hi


def test_planted_accept_length_is_capped_geometric():
    K, p, B = 5, 0.4, 6000
    c = _cfg(B=B, K=K, s=3, N=364, plant_p=p)       # the full 3-ary tree of depth 5
    plan = O.tree_plan(K, 3, 364)
    paths = planted_walk(c, plan["parent"], seed=1)
    A = np.array([len(q) - 1 for q in paths])
    expect = [p * (1 - p) ** a for a in range(K)] + [(1 - p) ** K]
    got = np.bincount(A, minlength=K + 1) / B
    for a in range(K + 1):
        sd = math.sqrt(expect[a] * (1 - expect[a]) / B)
        assert abs(got[a] - expect[a]) < 5 * sd, (a, got[a], expect[a])
    # every walk starts at the root and steps from a node to one of its children
    parent = plan["parent"]
    for q in paths[:500]:
        assert q[0] == 0
        assert all(parent[q[i + 1]] == q[i] for i in range(len(q) - 1))


def test_walk_stops_at_a_leaf():
    c = _cfg(B=200, K=5, s=1, N=3, plant_p=0.01)   # a chain of 3 nodes: depth <= 2
    plan = O.tree_plan(5, 1, 3)
    paths = planted_walk(c, plan["parent"], seed=2)
    assert max(len(q) - 1 for q in paths) == 2


def test_verify_logits_carry_the_boost_along_the_walk():
    c = _cfg(dtype="f32", B=4, V=500, N=64)
    plan = O.tree_plan(c.K, c.s, c.N)
    g = torch.Generator().manual_seed(3)
    tok = torch.randint(0, c.V, (c.B, c.N), generator=g)
    boosted = plant_verify_logits(c, plan["parent"], tok, seed=4)
    plain = plant_verify_logits(c.scaled(boost=0.0), plan["parent"], tok, seed=4)
    diff = (boosted - plain).numpy()
    want = np.zeros_like(diff)
    for b, q in enumerate(planted_walk(c, plan["parent"], seed=4)):
        for par, child in zip(q[:-1], q[1:]):
            want[b, par, int(tok[b, child])] += c.boost
    # (l + boost) - l in fp32 is the boost up to one rounding of l + boost
    np.testing.assert_allclose(diff, want, rtol=0, atol=1e-5)
    assert (diff[want == 0] == 0).all()
    assert abs(float(plain.std()) / c.sigma - 1.0) < 0.02
