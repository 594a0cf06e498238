"""Pins of the fp64 oracle against things other than itself.

Each test checks an oracle function against a closed form, a library routine
(torch / scipy), brute force on tiny inputs, or a hand-derived example, so that
a dropped term, a wrong sign or index, or a transposed operand fails one of
them.  CPU only.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200.synthetic import (CONFIGS, MedusaConfig,
                                                       plant_verify_logits, planted_walk)

GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# Tree plan
# ----------------------------------------------------------------------------
def _read_golden_tree(name):
    """Parse tests/golden/<name>: one rank tuple per line, '()' for the root."""
    out = []
    for line in open(f"{GOLDEN}/{name}"):
        line = line.split("#")[0].strip()
        if not line:
            continue
        inner = line.strip("()").strip()
        out.append(tuple(int(x) for x in inner.split(",") if x.strip()))
    return out


def test_tree_plan_tiny_config_worked_example():
    """Hand-derived 16-node tree of the tiny config (K=4, s=3): golden file."""
    plan = O.tree_plan(4, 3, 16)
    expected = _read_golden_tree("tree_tiny_k4_s3_n16.txt")
    assert plan["tuples"] == expected
    assert list(np.bincount(plan["depth"])) == [1, 3, 3, 4, 5]


def test_tree_plan_boundary_tie_breaks_lexicographically():
    """K=2, s=2, N=5 by hand: scores () 1, (0) .8, (0,0) .64, (1) .4, then a tie
    (0,1) = (1,0) = .32 resolved to the lexicographically smaller (0,1)."""
    plan = O.tree_plan(2, 2, 5)
    assert plan["tuples"] == [(), (0,), (1,), (0, 0), (0, 1)]
    assert list(plan["parent"]) == [-1, 0, 0, 1, 1]
    assert list(plan["depth"]) == [0, 1, 1, 2, 2]
    assert list(plan["rank"]) == [-1, 0, 1, 0, 1]
    assert [int(w) for w in plan["anc_mask"][:, 0]] == [0b1, 0b11, 0b101, 0b1011, 0b10011]


def _depth_counts_by_classes(K, s, N):
    """Independent count: group tuples into classes (D, S = sum of ranks), whose
    size is the number of compositions of S into D parts in [0, s) (inclusion-
    exclusion), order classes by exact score 0.8^D 0.5^S (then D), fill N."""
    def compositions(S, D):
        if D == 0:
            return 1 if S == 0 else 0
        return sum((-1) ** j * math.comb(D, j) * math.comb(S - j * s + D - 1, D - 1)
                   for j in range(D + 1) if S - j * s >= 0)
    classes = [(D, S) for D in range(K + 1) for S in range(D * (s - 1) + 1)]
    # exact compare of 0.8^D 0.5^S: 0.8^D 0.5^S = 2^(2D - S) / 5^D
    classes.sort(key=lambda c: (-(2 ** (2 * c[0] - c[1]) / 5 ** c[0]), c[0]))
    counts, left = [0] * (K + 1), N
    for D, S in classes:
        take = min(left, compositions(S, D))
        counts[D] += take
        left -= take
        if left == 0:
            break
    return counts


@pytest.mark.parametrize("name", ["tiny_f32", "7b_b1", "13b_b8", "8b_gqa_b16", "longctx_b4"])
def test_tree_plan_depth_counts_match_class_counting(name):
    cfg = CONFIGS[name]
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    got = list(np.bincount(plan["depth"], minlength=cfg.K + 1))
    assert got == _depth_counts_by_classes(cfg.K, cfg.s, cfg.N)


def test_tree_plan_depth_counts_derived_by_hand():
    # per-depth node counts (root first) worked out from the scoring rule
    assert _depth_counts_by_classes(5, 10, 64) == [1, 4, 10, 13, 15, 21]
    assert _depth_counts_by_classes(5, 8, 128) == [1, 5, 11, 20, 35, 56]
    assert _depth_counts_by_classes(5, 3, 256) == [1, 3, 9, 27, 69, 147]


@pytest.mark.parametrize("K,s", [(3, 2), (2, 3), (4, 3)])
def test_tree_plan_full_product(K, s):
    """N = 1 + s + ... + s^K selects the whole Cartesian product."""
    N = sum(s ** D for D in range(K + 1))
    plan = O.tree_plan(K, s, N)
    allt = [()] + [t for D in range(1, K + 1) for t in itertools.product(range(s), repeat=D)]
    assert set(plan["tuples"]) == set(allt)


@pytest.mark.parametrize("name", ["tiny_f32", "7b_b1", "8b_gqa_b16", "longctx_b4"])
def test_tree_plan_invariants(name):
    cfg = CONFIGS[name]
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    tset = set(plan["tuples"])
    for i, t in enumerate(plan["tuples"]):
        if t:
            assert t[:-1] in tset                        # prefix-closed
            assert plan["parent"][i] < i                 # topological
            assert plan["tuples"][plan["parent"][i]] == t[:-1]
            if t[-1] > 0:
                assert t[:-1] + (t[-1] - 1,) in tset     # rank-closed
        # ancestor mask equals the parent walk
        bits = {j for j in range(cfg.N) if plan["anc_mask"][i, j // 32] >> (j % 32) & 1}
        assert bits == set(O.ancestors_or_self(plan, i))
        assert all(plan["rank_path"][i, :len(t)] == t)
        assert all(plan["rank_path"][i, len(t):] == -1)
    # every unselected tuple scores no better than the worst selected one
    worst = min(O.tree_score(t) for t in plan["tuples"])
    for D in range(1, cfg.K + 1):
        for t in itertools.product(range(cfg.s), repeat=D):
            if t not in tset:
                assert O.tree_score(t) <= worst
                if sum(t) > 4:
                    break


# ----------------------------------------------------------------------------
# Heads
# ----------------------------------------------------------------------------
def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64) * std


def test_heads_zero_w1_reduces_to_lm_projection():
    """W1 = 0, b1 = 0: SiLU(0) = 0 so u = h and logits = W2 h (closed form)."""
    B, d, V, K = 3, 16, 40, 2
    h, W2 = _rand((B, d), 1), _rand((K, V, d), 2, 0.02)
    out = O.heads_forward(h, torch.zeros(K, d, d), torch.zeros(K, d), W2)
    for k in range(K):
        np.testing.assert_allclose(out[:, k], (h @ W2[k].T).numpy(), rtol=1e-12, atol=1e-14)


def test_heads_constant_bias_gives_shifted_residual():
    """W1 = 0, b1 = c: u = h + SiLU(c) (torch's silu), logits = W2 u."""
    B, d, V = 2, 8, 12
    h, W2 = _rand((B, d), 3), _rand((1, V, d), 4)
    c = torch.linspace(-3, 3, d, dtype=torch.float64)
    out = O.heads_forward(h, torch.zeros(1, d, d), c[None], W2)
    u = h + F.silu(c)[None]
    np.testing.assert_allclose(out[:, 0], (u @ W2[0].T).numpy(), rtol=1e-12, atol=1e-13)


def test_heads_match_torch_modules():
    """Random weights: same result as torch Linear -> SiLU -> +residual -> Linear."""
    B, d, V, K = 4, 32, 50, 3
    h, W1, b1, W2 = _rand((B, d), 5), _rand((K, d, d), 6, 0.3), _rand((K, d), 7), _rand((K, V, d), 8)
    out = O.heads_forward(h, W1, b1, W2)
    for k in range(K):
        ref = F.linear(F.silu(F.linear(h, W1[k], b1[k])) + h, W2[k])
        np.testing.assert_allclose(out[:, k], ref.numpy(), rtol=1e-11, atol=1e-12)
    sub = O.heads_forward(h, W1, b1, W2, heads=[2], vocab=[7, 3])
    np.testing.assert_allclose(sub[:, 0], out[:, 2][:, [7, 3]], rtol=1e-13)


# ----------------------------------------------------------------------------
# Top-s
# ----------------------------------------------------------------------------
def test_topk_planted_order_and_ties():
    row = np.array([0.5, 3.0, -1.0, 3.0, 2.0, 9.0])
    assert list(O.topk_row(row, 4)) == [5, 1, 3, 4]     # the tie 3.0 goes to index 1 first
    r = _rand((7, 300), 9)
    ref = torch.topk(r, 5, dim=-1).indices.numpy()       # distinct values: library order
    assert (O.topk(r, 5) == ref).all()


# ----------------------------------------------------------------------------
# Tree expansion
# ----------------------------------------------------------------------------
def test_build_tree_hand_example():
    plan = O.tree_plan(2, 2, 5)                           # (), (0), (1), (0,0), (0,1)
    topk_idx = np.array([[[10, 11], [20, 21]], [[30, 31], [40, 41]]])
    tok, pos = O.build_tree(plan, [7, 8], topk_idx, [100, 5])
    assert tok.tolist() == [[7, 10, 11, 20, 21], [8, 30, 31, 40, 41]]
    assert pos.tolist() == [[100, 101, 101, 102, 102], [5, 6, 6, 7, 7]]


# ----------------------------------------------------------------------------
# Tree attention
# ----------------------------------------------------------------------------
def _chain_plan(N):
    """parent[n] = n - 1: a single path."""
    words = (N + 31) // 32
    m = np.zeros((N, words), dtype=np.uint32)
    for i in range(N):
        for j in range(i + 1):
            m[i, j // 32] |= np.uint32(1 << (j % 32))
    return dict(N=N, K=N - 1, parent=np.arange(N) - 1, depth=np.arange(N), anc_mask=m)


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_attention_chain_tree_equals_causal(Hq, Hkv):
    B, N, dh, L = 2, 6, 8, 5
    q = _rand((B, N, Hq, dh), 10)
    kc, vc = _rand((B, L + N, Hkv, dh), 11), _rand((B, L + N, Hkv, dh), 12)
    scale = 1 / math.sqrt(dh)
    out = O.tree_attention(q, kc, vc, [L, L], _chain_plan(N), scale)
    G = Hq // Hkv
    # causal SDPA over the full sequence; the last N queries are the chain nodes
    qf = torch.zeros(B, Hq, L + N, dh, dtype=torch.float64)
    qf[:, :, L:] = q.permute(0, 2, 1, 3)
    kf = kc.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vf = vc.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    ref = F.scaled_dot_product_attention(qf, kf, vf, is_causal=True, scale=scale)
    np.testing.assert_allclose(out, ref[:, :, L:].permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)


def test_attention_each_node_equals_attention_over_its_path():
    K, s, N = 3, 2, 11
    plan = O.tree_plan(K, s, N)
    B, Hq, Hkv, dh = 2, 3, 3, 16
    Ls = [9, 4]
    q = _rand((B, N, Hq, dh), 13)
    kc, vc = _rand((B, max(Ls) + N, Hkv, dh), 14), _rand((B, max(Ls) + N, Hkv, dh), 15)
    out = O.tree_attention(q, kc, vc, Ls, plan, 0.3)
    for b in range(B):
        for i in range(N):
            path = O.ancestors_or_self(plan, i)
            slots = list(range(Ls[b])) + [Ls[b] + j for j in path]
            for h in range(Hq):
                k, v = kc[b, slots, h][None, None], vc[b, slots, h][None, None]
                ref = F.scaled_dot_product_attention(q[b, i, h][None, None, None], k, v, scale=0.3)
                np.testing.assert_allclose(out[b, i, h], ref[0, 0, 0].numpy(), rtol=1e-10, atol=1e-12)


def test_attention_single_node_is_decode_attention_and_identical_keys_give_mean():
    B, Hq, dh, L = 1, 2, 4, 7
    q = _rand((B, 1, Hq, dh), 16)
    kc, vc = _rand((B, L + 1, Hq, dh), 17), _rand((B, L + 1, Hq, dh), 18)
    plan = _chain_plan(1)
    out = O.tree_attention(q, kc, vc, [L], plan, 0.5)
    ref = F.scaled_dot_product_attention(q.permute(0, 2, 1, 3), kc.permute(0, 2, 1, 3),
                                         vc.permute(0, 2, 1, 3), scale=0.5)
    np.testing.assert_allclose(out[:, 0], ref[:, :, 0].numpy(), rtol=1e-10)
    # identical keys -> uniform weights -> mean of the visible values
    plan = O.tree_plan(2, 2, 5)
    kc = torch.ones(1, L + 5, Hq, dh, dtype=torch.float64)
    vc = _rand((1, L + 5, Hq, dh), 19)
    q = _rand((1, 5, Hq, dh), 20)
    out = O.tree_attention(q, kc, vc, [L], plan, 1.0)
    for i in range(5):
        slots = list(range(L)) + [L + j for j in O.ancestors_or_self(plan, i)]
        np.testing.assert_allclose(out[0, i], vc[0, slots].mean(0).numpy(), rtol=1e-12)


# ----------------------------------------------------------------------------
# Greedy acceptance
# ----------------------------------------------------------------------------
def _sequential_argmax_decode(vlog, tok, plan):
    """Lossless greedy decoding simulated one token at a time: from the root,
    emit t = argmax of the current row; move to the child carrying t if any."""
    children = {n: [c for c in range(plan["N"]) if plan["parent"][c] == n] for n in range(plan["N"])}
    cur, emitted, path = 0, [], [0]
    while True:
        t = int(torch.argmax(vlog[cur]).item()) if isinstance(vlog, torch.Tensor) else int(np.argmax(vlog[cur]))
        emitted.append(t)
        nxt = [c for c in children[cur] if tok[c] == t]
        if not nxt:
            return emitted, path
        cur = nxt[0]
        path.append(cur)


@pytest.mark.parametrize("seed", range(6))
def test_greedy_equals_sequential_argmax(seed):
    cfg = MedusaConfig("t", "f32", B=3, d=8, V=64, K=4, s=3, N=16, Hq=1, Hkv=1, dh=8,
                       L_lo=4, L_hi=4)
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator().manual_seed(seed)
    topk_idx = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.s * cfg.K].view(cfg.K, cfg.s)
                            for _ in range(cfg.B)])
    tok, _ = O.build_tree(plan, torch.randint(0, cfg.V, (cfg.B,), generator=g), topk_idx, [4] * cfg.B)
    vlog = plant_verify_logits(cfg, plan["parent"], tok, seed=seed)
    alen, anodes, nxt = O.accept_greedy(vlog, tok, plan)
    for b in range(cfg.B):
        emitted, path = _sequential_argmax_decode(vlog[b], tok[b], plan)
        assert alen[b] == len(path) - 1
        assert list(anodes[b, :len(path)]) == path and all(anodes[b, len(path):] == -1)
        assert [int(tok[b, n]) for n in path[1:]] + [int(nxt[b])] == emitted
        # the planted walk is followed at least as far as it was planted
        planted = planted_walk(cfg, plan["parent"], seed)[b]
        assert path[:len(planted)] == planted


def test_greedy_tie_goes_to_lowest_index():
    plan = O.tree_plan(1, 2, 3)                          # root, (0), (1)
    vlog = np.zeros((1, 3, 5))
    vlog[0, 0, [2, 4]] = 1.0                             # tie between tokens 2 and 4
    alen, anodes, nxt = O.accept_greedy(vlog, np.array([[0, 4, 2]]), plan)
    assert alen[0] == 1 and anodes[0].tolist() == [0, 2] and nxt[0] == 0


# ----------------------------------------------------------------------------
# Typical acceptance
# ----------------------------------------------------------------------------
def test_typical_entropy_and_threshold_closed_forms():
    n = 50
    p, H = O.typical_row_stats(np.zeros(n), 0.7)
    assert abs(H - math.log(n)) < 1e-12
    assert O.typical_threshold(H, 0.09, 0.6) == pytest.approx(min(0.09, 0.6 / n))
    # against scipy's entropy for random distributions and temperatures
    from scipy.stats import entropy
    from scipy.special import softmax
    r = _rand((5, 40), 21).numpy()
    for T in (0.3, 0.7, 1.0, 2.0):
        for row in r:
            p, H = O.typical_row_stats(row, T)
            np.testing.assert_allclose(p, softmax(row / T), rtol=1e-12)
            assert H == pytest.approx(entropy(softmax(row / T)), rel=1e-12)
    # the threshold switches from eps to delta*e^-H at H = ln(delta/eps)
    Hs = math.log(0.6 / 0.09)
    assert O.typical_threshold(Hs - 1e-6, 0.09, 0.6) == 0.09
    assert O.typical_threshold(Hs + 1e-6, 0.09, 0.6) < 0.09


def _tree_one_level(n_children):
    N = 1 + n_children
    m = np.zeros((N, 1), dtype=np.uint32)
    m[0, 0] = 1
    for c in range(1, N):
        m[c, 0] = 1 | (1 << c)
    return dict(N=N, K=1, parent=np.array([-1] + [0] * n_children), depth=np.array([0] + [1] * n_children),
                anc_mask=m)


def test_typical_hand_cases():
    plan = _tree_one_level(4)
    # p = (0.97, 0.01, 0.01, 0.01): H ~= 0.1677, delta e^-H ~= 0.507 -> thr = 0.09
    p = np.array([0.97, 0.01, 0.01, 0.01])
    vlog = np.zeros((1, 5, 4))
    vlog[0, 0] = np.log(p)
    tok = np.array([[0, 1, 0, 2, 3]])
    alen, anodes, nxt, _ = O.accept_typical(vlog, tok, plan, 1.0)
    assert alen[0] == 1 and anodes[0].tolist() == [0, 2]
    _, H = O.typical_row_stats(vlog[0, 0], 1.0)
    assert H == pytest.approx(-(0.97 * math.log(0.97) + 3 * 0.01 * math.log(0.01)), rel=1e-12)
    # uniform over 4: thr = min(0.09, 0.6/4) = 0.09 < 0.25 -> every child accepted; lowest index wins
    vlog[0, 0] = 0.0
    alen, anodes, _, _ = O.accept_typical(vlog, tok, plan, 1.0)
    assert alen[0] == 1 and anodes[0].tolist() == [0, 1]
    # strictness: a child at exactly the threshold is rejected
    # two tokens: p = (0.91, 0.09) has H > ln(0.6/0.09)? no -> thr = 0.09 -> 0.09 is not > 0.09
    plan2 = _tree_one_level(1)
    v2 = np.zeros((1, 2, 2))
    v2[0, 0] = np.log([0.91, 0.09])
    a, _, _, margin = O.accept_typical(v2, np.array([[0, 1]]), plan2, 1.0)
    assert margin[0, 1] < 1e-12          # a decision on the threshold: flagged as too close to call


def test_typical_low_temperature_reduces_to_greedy():
    cfg = MedusaConfig("t", "f32", B=2, d=8, V=64, K=4, s=3, N=16, Hq=1, Hkv=1, dh=8,
                       L_lo=4, L_hi=4)
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator().manual_seed(3)
    topk_idx = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.s * cfg.K].view(cfg.K, cfg.s)
                            for _ in range(cfg.B)])
    tok, _ = O.build_tree(plan, [1, 2], topk_idx, [4, 4])
    vlog = plant_verify_logits(cfg, plan["parent"], tok, seed=3).double()
    ga = O.accept_greedy(vlog, tok, plan)
    ta = O.accept_typical(vlog, tok, plan, 0.01)
    assert (ga[0] == ta[0]).all() and (ga[1] == ta[1]).all() and (ga[2] == ta[2]).all()


# ----------------------------------------------------------------------------
# Compaction
# ----------------------------------------------------------------------------
def test_kv_compact_equals_gather():
    B, Lcap, H, dh, K = 3, 30, 2, 4, 3
    kc, vc = _rand((B, Lcap, H, dh), 22), _rand((B, Lcap, H, dh), 23)
    L = torch.tensor([5, 10, 0])
    A = torch.tensor([3, 0, 2])
    nodes = torch.tensor([[0, 2, 5, 9], [0, -1, -1, -1], [0, 1, 2, -1]])
    nk, nv, nl = O.kv_compact(kc, vc, L, A, nodes)
    assert nl.tolist() == [9, 11, 3]
    for b in range(B):
        idx = torch.arange(Lcap)
        for j in range(1, int(A[b]) + 1):
            idx[L[b] + j] = L[b] + nodes[b, j]
        np.testing.assert_array_equal(nk[b], kc[b].index_select(0, idx).numpy())
        np.testing.assert_array_equal(nv[b], vc[b].index_select(0, idx).numpy())


# ----------------------------------------------------------------------------
# Sampled next token (Gumbel-max over SplitMix64 noise)
# ----------------------------------------------------------------------------
def test_splitmix64_known_answers():
    """The generator's first outputs from state 0 (tests/golden/splitmix64_seed0.txt)."""
    rows = [ln.split() for ln in open(__import__("os").path.join(GOLDEN, "splitmix64_seed0.txt"))
            if ln.strip() and not ln.startswith("#")]
    idx = np.array([int(r[0]) for r in rows])
    want = [int(r[1], 16) for r in rows]
    assert [int(v) for v in O.splitmix64(0, idx)] == want


def test_splitmix64_counter_form_equals_sequential_generator():
    """Output i of the counter form = the (i+1)-th output of the stepping
    generator (state += gamma, then the finaliser), for an arbitrary seed."""
    M = (1 << 64) - 1
    seed = 0x0123456789ABCDEF
    x, seq = seed, []
    for _ in range(12):
        x = (x + 0x9E3779B97F4A7C15) & M
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        seq.append(z ^ (z >> 31))
    assert [int(v) for v in O.splitmix64(seed, np.arange(12))] == seq


def test_uniform01_extremes_are_exact_and_inside_the_interval():
    """The smallest and largest 23-bit values map exactly to 2^-24 and
    1 - 2^-24 in fp32 (a construction that rounded the top value up to 1
    would give infinite Gumbel noise)."""
    top = np.array([0, 1, (1 << 23) - 2, (1 << 23) - 1], dtype=np.float32)
    u = ((top + np.float32(0.5)) * np.float32(2.0 ** -23)).astype(np.float32)
    assert u[0] == np.float32(2.0 ** -24) and u[-1] == np.float32(1 - 2.0 ** -24)
    assert (u < 1).all() and (u > 0).all() and np.isfinite(O.gumbel32(u)).all()
    # and the oracle's uniforms are exactly of that form
    v = O.uniform01(3, np.arange(1000))
    t = (O.splitmix64(3, np.arange(1000)) >> np.uint64(41)).astype(np.float64)
    np.testing.assert_array_equal(v.astype(np.float64), (t + 0.5) * 2.0 ** -23)


def test_uniform01_range_and_uniformity():
    u = O.uniform01(7, np.arange(200_000))
    assert u.dtype == np.float32 and (u > 0).all() and (u < 1).all()
    counts = np.bincount((u * 64).astype(np.int64), minlength=64)
    exp = len(u) / 64
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert chi2 < 110.0          # df = 63, p ~ 1e-4
    # consecutive counters are uncorrelated
    assert abs(np.corrcoef(u[:-1], u[1:])[0, 1]) < 0.01


def test_gumbel_noise_moments():
    """Standard Gumbel: mean = Euler-Mascheroni constant, variance pi^2 / 6."""
    g = O.gumbel32(O.uniform01(11, np.arange(400_000))).astype(np.float64)
    assert abs(g.mean() - 0.5772156649) < 0.01
    assert abs(g.var() - math.pi ** 2 / 6) < 0.03


def test_sample_next_frequencies_follow_softmax():
    """Draws over many call offsets follow softmax(l / T) (chi-square)."""
    l = np.array([2.0, 1.0, 0.5, 0.0, -1.0, 3.0], dtype=np.float32)
    T = 0.8
    vlog = torch.from_numpy(l).view(1, 1, 6)
    A, nodes = np.array([0]), np.array([[0, -1]])
    n = 20_000
    hits = np.zeros(6)
    for off in range(n):
        t, _ = O.sample_next(vlog, A, nodes, T, seed=5, offset=off)
        hits[t[0]] += 1
    p = np.exp(l / T - (l / T).max())
    p /= p.sum()
    chi2 = float(((hits - n * p) ** 2 / (n * p)).sum())
    assert chi2 < 20.5           # df = 5, p = 0.001


def test_sample_next_temperature_zero_is_argmax_of_last_accepted_row():
    g = torch.Generator().manual_seed(4)
    vlog = torch.randn(3, 5, 50, generator=g)
    A = np.array([0, 2, 1])
    nodes = np.array([[0, -1, -1], [0, 3, 4], [0, 2, -1]])
    t, _ = O.sample_next(vlog, A, nodes, 0.0, seed=1, offset=0)
    assert list(t) == [int(vlog[0, 0].argmax()), int(vlog[1, 4].argmax()), int(vlog[2, 2].argmax())]
    # a tiny temperature with a clear winner also picks the argmax
    t2, _ = O.sample_next(vlog, A, nodes, 1e-3, seed=1, offset=3)
    assert list(t2) == list(t)


# ----------------------------------------------------------------------------
# Typical acceptance with one temperature per head
# ----------------------------------------------------------------------------
def test_typical_per_head_equal_temperatures_is_the_scalar_rule():
    cfg = MedusaConfig("t", "f32", B=2, d=8, V=64, K=4, s=3, N=16, Hq=1, Hkv=1, dh=8,
                       L_lo=4, L_hi=4, plant_p=0.2)
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator().manual_seed(8)
    topk_idx = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.s * cfg.K].view(cfg.K, cfg.s)
                            for _ in range(cfg.B)])
    tok, _ = O.build_tree(plan, [1, 2], topk_idx, [4, 4])
    vlog = plant_verify_logits(cfg, plan["parent"], tok, seed=8).double()
    a = O.accept_typical(vlog, tok, plan, 0.7)
    b = O.accept_typical(vlog, tok, plan, [0.7] * cfg.K)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_typical_per_head_temperature_decides_its_own_depth():
    """Hand case: chain tree (s = 1), V = 8.  The root row favours token 0 by
    3 nats; node 1 carries token 1.  At T = 0.1 its probability is ~e^-30
    (rejected); at T = 10 the row is nearly uniform: H ~ ln 8, threshold
    min(0.09, 0.6 / 8.0...) ~ 0.075 < p(1) = 1 / (7 + e^0.3) ~ 0.12 (accepted).
    Node 2 (depth 2, token 2) sits on node 1's row, which is uniform: p = 1/8
    > min(0.09, 0.6/8) = 0.075 at any temperature."""
    plan = O.tree_plan(2, 1, 3)
    assert [int(x) for x in plan["depth"]] == [0, 1, 2]
    V = 8
    vlog = np.zeros((1, 3, V))
    vlog[0, 0, 0] = 3.0
    tok = np.array([[5, 1, 2]])
    for T, want in (([0.1, 1.0], 0), ([10.0, 1.0], 2), ([10.0, 0.05], 2)):
        alen, nodes, _, _ = O.accept_typical(vlog, tok, plan, T)
        assert int(alen[0]) == want, (T, alen)


# ----------------------------------------------------------------------------
# Merging per-shard top-s lists (vocabulary split across ranks)
# ----------------------------------------------------------------------------
def test_topk_merge_of_shard_lists_is_the_global_topk():
    """Each shard's own top-s, with global indices, merged = top-s of the
    whole row (brute force), for uneven shard sizes and ties."""
    g = torch.Generator().manual_seed(12)
    R, V, s = 7, 1000, 6
    logits = torch.randn(R, V, generator=g, dtype=torch.float64)
    logits[2, 100:110] = 5.0                       # a 10-way tie across shards
    bounds = [0, 137, 500, 501, 1000]              # 4 shards, one of a single column
    vals, idxs = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        k = min(s, b - a)
        loc = O.topk(logits[:, a:b].numpy(), k)
        v = np.take_along_axis(logits[:, a:b].numpy(), loc, axis=1)
        vi = np.full((R, s), -1)
        vv = np.zeros((R, s))
        vi[:, :k], vv[:, :k] = loc + a, v
        vals.append(vv)
        idxs.append(vi)
    mi, mv = O.topk_merge(np.stack(vals), np.stack(idxs), s)
    want = O.topk(logits.numpy(), s)
    np.testing.assert_array_equal(mi, want)
    np.testing.assert_array_equal(mv, np.take_along_axis(logits.numpy(), want, axis=1))


def test_topk_merge_pads_when_candidates_run_out():
    vals = np.array([[[3.0, 1.0]], [[2.0, 0.0]]])
    idxs = np.array([[[4, -1]], [[9, -1]]])
    mi, mv = O.topk_merge(vals, idxs, 3)
    assert mi.tolist() == [[4, 9, -1]] and mv[0, 0] == 3.0 and np.isnan(mv[0, 2])


# ----------------------------------------------------------------------------
# Several layers
# ----------------------------------------------------------------------------
def test_attention_layers_chain_tree_is_causal_attention_per_layer():
    """Three layers, a chain tree (s = 1): each layer's rows equal ordinary
    causal attention (torch SDPA) over that layer's own prefix + chain."""
    nl, B, K, L, Hq, Hkv, dh = 3, 2, 5, 40, 4, 2, 16
    N = K + 1
    g = torch.Generator().manual_seed(21)
    q = torch.randn(nl, B, N, Hq, dh, generator=g, dtype=torch.float64)
    kc = torch.randn(nl, B, L + N, Hkv, dh, generator=g, dtype=torch.float64)
    vc = torch.randn(nl, B, L + N, Hkv, dh, generator=g, dtype=torch.float64)
    plan = O.tree_plan(K, 1, N)
    got = O.tree_attention_layers(q, kc, vc, [L] * B, plan, 0.25)
    G = Hq // Hkv
    for l in range(nl):
        qf = torch.zeros(B, Hq, L + N, dh, dtype=torch.float64)
        qf[:, :, L:] = q[l].permute(0, 2, 1, 3)
        kf = kc[l].repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
        vf = vc[l].repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
        ref = F.scaled_dot_product_attention(qf, kf, vf, is_causal=True, scale=0.25)
        assert np.allclose(got[l], ref[:, :, L:].permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_attention_layers_follow_their_own_caches():
    """Swapping two layers' queries and caches swaps their outputs, and a
    layer's output depends on no other layer (doubling layer 0's V doubles
    its output and leaves layer 1's)."""
    nl, B, L, Hq, dh = 2, 1, 30, 2, 8
    plan = O.tree_plan(3, 2, 9)
    g = torch.Generator().manual_seed(4)
    q = torch.randn(nl, B, 9, Hq, dh, generator=g, dtype=torch.float64)
    kc = torch.randn(nl, B, L + 9, Hq, dh, generator=g, dtype=torch.float64)
    vc = torch.randn(nl, B, L + 9, Hq, dh, generator=g, dtype=torch.float64)
    a = O.tree_attention_layers(q, kc, vc, [L], plan, 0.3)
    b = O.tree_attention_layers(q.flip(0), kc.flip(0), vc.flip(0), [L], plan, 0.3)
    assert np.array_equal(a, b[::-1])
    vc2 = vc.clone()
    vc2[0] *= 2.0          # attention is linear in V: layer 0 doubles, layer 1 stays
    c = O.tree_attention_layers(q, kc, vc2, [L], plan, 0.3)
    assert np.array_equal(a[1], c[1]) and np.allclose(c[0], 2.0 * a[0], atol=1e-12)


def test_kv_compact_layers_equals_gather_in_every_layer():
    """Every layer's slots L_b + j take old slots L_b + nodes[j] (numpy
    fancy-index gather), new_len = L_b + 1 + a, other slots untouched."""
    nl, B, Lcap, Hkv, dh, K = 3, 2, 30, 2, 4, 3
    rng = np.random.default_rng(8)
    kc = rng.standard_normal((nl, B, Lcap, Hkv, dh))
    vc = rng.standard_normal((nl, B, Lcap, Hkv, dh))
    L = np.array([10, 4])
    A = np.array([3, 1])
    nodes = np.array([[0, 2, 5, 9], [0, 1, -1, -1]])
    nk, nv, nlen = O.kv_compact_layers(kc, vc, L, A, nodes)
    assert (nlen == L + 1 + A).all()
    for b in range(B):
        dst = L[b] + np.arange(1, A[b] + 1)
        src = L[b] + nodes[b, 1:A[b] + 1]
        ek, ev = kc.copy(), vc.copy()
        ek[:, b, dst] = kc[:, b, src]
        ev[:, b, dst] = vc[:, b, src]
        assert np.array_equal(nk[:, b], ek[:, b]) and np.array_equal(nv[:, b], ev[:, b])
