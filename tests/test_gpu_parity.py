"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded
inputs (tolerances: indices, tree tokens, accept results and compacted KV
bit-exact; logits and attention outputs max-abs 2e-2; top-s ids exact
wherever the logit gap to the neighbouring rank exceeds 1e-2)."""
import math

import numpy as np
import pytest
import torch

from attn_check import assert_attention_close
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.synthetic import (CONFIGS, MedusaConfig, gen_inputs,
                                                       plant_verify_logits)

pytestmark = pytest.mark.gpu
ATOL = 2e-2
GAP = 1e-2
DEV = "cuda"


def _check_topk(gpu_idx, ref_logits, s):
    """gpu_idx [R][s]; ref_logits [R][V] fp64 (oracle)."""
    gpu_idx = np.asarray(gpu_idx)
    for r in range(ref_logits.shape[0]):
        row = ref_logits[r]
        order = O.topk_row(row, s + 1)
        vals = row[order]
        for j in range(s):
            left_ok = j == 0 or vals[j - 1] - vals[j] > GAP
            right_ok = vals[j] - vals[j + 1] > GAP if j + 1 < len(vals) else True
            if left_ok and right_ok:
                assert gpu_idx[r, j] == order[j], (r, j, gpu_idx[r], order[:s])
        if s < len(vals) and vals[s - 1] - vals[s] > GAP:
            assert set(gpu_idx[r].tolist()) == set(order[:s].tolist())


def _small_cfg(**kw):
    base = dict(name="small", dtype="bf16", B=1, d=256, V=1000, K=3, s=5, N=16, Hq=4, Hkv=4,
                dh=128, L_lo=64, L_hi=64)
    base.update(kw)
    return MedusaConfig(**base)


# ---------------------------------------------------------------------------- heads
@pytest.mark.parametrize("B,d,V,K,s", [(1, 256, 1000, 3, 5), (3, 200, 777, 2, 4),
                                       (16, 1024, 1000, 5, 8), (8, 512, 2048, 4, 10),
                                       (32, 128, 300, 1, 16), (2, 2048, 640, 5, 3)])
def test_heads_bf16_small(B, d, V, K, s):
    cfg = _small_cfg(B=B, d=d, V=V, K=K, s=s)
    x = gen_inputs(cfg, DEV, seed=B + d)
    logits, idx, val = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s)
    torch.cuda.synchronize()
    ref = O.heads_forward(x["h"], x["W1"], x["b1"], x["W2"])
    err = np.abs(logits.double().cpu().numpy() - ref).max()
    assert err <= ATOL, err
    _check_topk(idx.cpu().numpy().reshape(B * K, s), ref.reshape(B * K, V), s)
    # returned values are the GPU logits at those ids
    lg = logits.cpu()
    np.testing.assert_array_equal(val.cpu().numpy(),
                                  torch.gather(lg, 2, idx.long().cpu()).numpy())


def test_heads_bf16_topk_without_logits_and_null_bias():
    cfg = _small_cfg(B=4, d=512, V=1500, K=2, s=6)
    x = gen_inputs(cfg, DEV, seed=7)
    logits, idx, _ = api.medusa_heads_forward(x["h"], x["W1"], None, x["W2"], s=6,
                                              want_logits=False)
    assert logits is None
    ref = O.heads_forward(x["h"], x["W1"], None, x["W2"])
    _check_topk(idx.cpu().numpy().reshape(8, 6), ref.reshape(8, 1500), 6)


def test_heads_f32_tiny_config():
    cfg = CONFIGS["tiny_f32"]
    x = gen_inputs(cfg, DEV, seed=0)
    logits, idx, _ = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=cfg.s)
    ref = O.heads_forward(x["h"], x["W1"], x["b1"], x["W2"])
    assert np.abs(logits.double().cpu().numpy() - ref).max() <= 1e-4
    _check_topk(idx.cpu().numpy().reshape(cfg.K, cfg.s), ref.reshape(cfg.K, cfg.V), cfg.s)


def test_heads_repeatable():
    cfg = _small_cfg(B=8, d=1024, V=3000, K=3, s=8)
    x = gen_inputs(cfg, DEV, seed=3)
    a = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=8)
    b = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=8)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------------------------------------------------- top-s
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("R,V,s", [(1, 10, 10), (7, 1000, 5), (3, 32001, 16), (5, 129, 1)])
def test_topk_rows_exact(dtype, R, V, s):
    g = torch.Generator(device=DEV).manual_seed(R * V + s)
    x = (torch.randn(R, V, generator=g, device=DEV) * 2).to(dtype)   # bf16: many exact ties
    idx, val = api.medusa_topk(x, s)
    ref = O.topk(x, s)
    assert (idx.cpu().numpy() == ref).all()
    np.testing.assert_array_equal(val.cpu().numpy(), x.float().cpu().numpy()[np.arange(R)[:, None], ref])


# ---------------------------------------------------------------------------- tree
@pytest.mark.parametrize("name", list(CONFIGS))
def test_build_tree_exact(name):
    cfg = CONFIGS[name]
    tree = api.Tree(cfg.K, cfg.s, cfg.N)
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator(device=DEV).manual_seed(11)
    topk = torch.randint(0, cfg.V, (cfg.B, cfg.K, cfg.s), generator=g, device=DEV,
                         dtype=torch.int32)
    root = torch.randint(0, cfg.V, (cfg.B,), generator=g, device=DEV, dtype=torch.int32)
    L = torch.randint(cfg.L_lo, cfg.L_hi + 1, (cfg.B,), generator=g, device=DEV, dtype=torch.int32)
    tok, pos = api.medusa_build_tree(tree, root, topk, L)
    rt, rp = O.build_tree(plan, root, topk, L)
    assert (tok.cpu().numpy() == rt).all() and (pos.cpu().numpy() == rp).all()
    p, dpt, rk, anc = tree.info()
    assert (p.numpy() == plan["parent"]).all() and (dpt.numpy() == plan["depth"]).all()


# ---------------------------------------------------------------------------- attention
def _attn_case(B, N_K_s, Hq, Hkv, dh, Ls, dtype, seed):
    K, s, N = N_K_s
    Lcap = max(Ls) + N + 3
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn(B, N, Hq, dh, generator=g, device=DEV).to(dtype)
    kc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    vc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    L = torch.tensor(Ls, dtype=torch.int32, device=DEV)
    return K, s, N, q, kc, vc, L


@pytest.mark.parametrize("B,tree,Hq,Hkv,dh,Ls,dtype", [
    (1, (4, 3, 16), 4, 4, 64, [128], torch.float32),
    (1, (4, 3, 16), 4, 4, 128, [0], torch.bfloat16),
    (3, (3, 2, 7), 8, 2, 128, [1, 63, 129], torch.bfloat16),
    (2, (5, 10, 64), 4, 1, 128, [300, 1000], torch.bfloat16),
    (1, (1, 1, 1), 2, 2, 128, [257], torch.bfloat16),
    (2, (5, 3, 100), 2, 2, 64, [33, 0], torch.float32),
    (2, (5, 8, 128), 8, 2, 128, [1000, 777], torch.bfloat16),    # 4 row tiles, split keys
    (1, (5, 3, 256), 2, 2, 128, [513], torch.bfloat16),          # two tree tiles
    (2, (4, 4, 40), 16, 1, 128, [2100, 64], torch.bfloat16),     # GQA group 16
])
def test_tree_attention_small(B, tree, Hq, Hkv, dh, Ls, dtype):
    K, s, N, q, kc, vc, L = _attn_case(B, tree, Hq, Hkv, dh, Ls, dtype, seed=B * 100 + tree[2])
    t = api.Tree(K, s, N)
    plan = O.tree_plan(K, s, N)
    scale = 1.0 / math.sqrt(dh)
    out = api.medusa_tree_attention(q, kc, vc, L, t, scale)
    ref = O.tree_attention(q, kc, vc, L, plan, scale)
    assert_attention_close(out.double().cpu().numpy(), ref, bf16=dtype == torch.bfloat16,
                           what=f"B={B} tree={tree} Hq={Hq} Hkv={Hkv} dh={dh} L={Ls}")


def test_tree_attention_chain_equals_causal_sdpa():
    """A K-deep chain tree (s = 1) is ordinary causal attention."""
    K, N, Hq, dh, L = 8, 9, 4, 128, 200
    B = 2
    g = torch.Generator(device=DEV).manual_seed(5)
    q = torch.randn(B, N, Hq, dh, generator=g, device=DEV).bfloat16()
    kc = torch.randn(B, L + N, Hq, dh, generator=g, device=DEV).bfloat16()
    vc = torch.randn(B, L + N, Hq, dh, generator=g, device=DEV).bfloat16()
    t = api.Tree(K, 1, N)
    out = api.medusa_tree_attention(q, kc, vc, torch.full((B,), L, dtype=torch.int32, device=DEV),
                                    t, 1 / math.sqrt(dh))
    qf = torch.zeros(B, Hq, L + N, dh, dtype=torch.float64)
    qf[:, :, L:] = q.double().cpu().permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qf, kc.double().cpu().permute(0, 2, 1, 3), vc.double().cpu().permute(0, 2, 1, 3),
        is_causal=True, scale=1 / math.sqrt(dh))[:, :, L:].permute(0, 2, 1, 3)
    assert_attention_close(out.double().cpu().numpy(), ref.numpy(), what="chain tree")


def test_tree_attention_rejects_overflowing_sequence_rows():
    """L_b + N > Lcap: that sequence's rows are written as zeros."""
    K, s, N, q, kc, vc, L = _attn_case(2, (2, 2, 5), 2, 2, 128, [10, 10], torch.bfloat16, 1)
    L[1] = kc.shape[1] - 2
    t = api.Tree(K, s, N)
    out = api.medusa_tree_attention(q, kc, vc, L, t, 0.1)
    assert out[1].abs().max().item() == 0.0
    ref = O.tree_attention(q[:1], kc[:1], vc[:1], L[:1], O.tree_plan(K, s, N), 0.1)
    assert_attention_close(out[:1].double().cpu().numpy(), ref, what="valid sequence")


# ---------------------------------------------------------------------------- acceptance
def _accept_inputs(cfg, seed):
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator().manual_seed(seed)
    topk = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.K * cfg.s].view(cfg.K, cfg.s)
                        for _ in range(cfg.B)])
    root = torch.randint(0, cfg.V, (cfg.B,), generator=g)
    tok, _ = O.build_tree(plan, root, topk, [0] * cfg.B)
    vlog = plant_verify_logits(cfg, plan["parent"], tok, device=DEV, seed=seed)
    return plan, torch.as_tensor(tok, dtype=torch.int32, device=DEV), vlog


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,K,s,N,V", [(1, 4, 3, 16, 1024), (5, 5, 10, 64, 3001),
                                       (3, 5, 3, 256, 500), (2, 1, 4, 5, 64)])
def test_accept_greedy_exact(dtype, B, K, s, N, V):
    cfg = _small_cfg(dtype=dtype, B=B, K=K, s=s, N=N, V=V)
    plan, tok, vlog = _accept_inputs(cfg, seed=B * 7 + N)
    t = api.Tree(K, s, N)
    alen, anodes, nxt = api.medusa_accept_greedy(vlog, tok, t)
    ra, rn, rx = O.accept_greedy(vlog, tok, plan)
    assert (alen.cpu().numpy() == ra).all()
    assert (anodes.cpu().numpy() == rn).all()
    assert (nxt.cpu().numpy() == rx).all()


def _check_typical(alen, anodes, nxt, ref, plan, B):
    ra, rn, rx, margin = ref
    for b in range(B):
        path = [int(n) for n in rn[b] if n >= 0]
        # decisions too close to call in any finite precision are don't-cares
        close = any(margin[b, n] < 1e-5 for n in range(1, plan["N"]))
        if close:
            continue
        assert alen[b] == ra[b], b
        assert anodes[b].tolist() == rn[b].tolist(), b
        assert nxt[b] == rx[b], b
        assert len(path) == ra[b] + 1


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,K,s,N,V,sigma,T", [(4, 5, 8, 128, 4096, 1.5, 0.7),
                                               (3, 4, 3, 16, 1024, 1.0, 1.0),
                                               (2, 5, 3, 256, 777, 1.0, 0.3)])
def test_accept_typical(dtype, B, K, s, N, V, sigma, T):
    cfg = _small_cfg(dtype=dtype, B=B, K=K, s=s, N=N, V=V, sigma=sigma)
    plan, tok, vlog = _accept_inputs(cfg, seed=B * 13 + N)
    t = api.Tree(K, s, N)
    alen, anodes, nxt = api.medusa_accept_typical(vlog, tok, t, T, 0.09, 0.6)
    ref = O.accept_typical(vlog, tok, plan, T, 0.09, 0.6)
    _check_typical(alen.cpu().numpy(), anodes.cpu().numpy(), nxt.cpu().numpy(), ref, plan, B)


@pytest.mark.parametrize("dtype,B,K,s,N,V,temps", [
    (torch.bfloat16, 4, 5, 10, 64, 32000, (0.5, 0.7, 1.0, 1.2, 1.5)),
    (torch.float32, 3, 4, 3, 16, 1000, (2.0, 0.3, 1.0, 0.6)),
    (torch.bfloat16, 2, 3, 4, 40, 5000, (0.7, 0.7, 0.7)),
])
def test_accept_typical_per_head(dtype, B, K, s, N, V, temps):
    """One temperature per head: node of depth D verified at temps[D-1]."""
    cfg = _small_cfg(dtype=dtype, B=B, K=K, s=s, N=N, V=V, sigma=1.0)
    plan, tok, vlog = _accept_inputs(cfg, seed=B * 7 + N)
    t = api.Tree(K, s, N)
    alen, anodes, nxt = api.medusa_accept_typical_per_head(vlog, tok, t, temps, 0.09, 0.6)
    ref = O.accept_typical(vlog, tok, plan, list(temps), 0.09, 0.6)
    _check_typical(alen.cpu().numpy(), anodes.cpu().numpy(), nxt.cpu().numpy(), ref, plan, B)
    if len(set(temps)) == 1:   # equal temperatures: the scalar entry point
        a2, n2, x2 = api.medusa_accept_typical(vlog, tok, t, temps[0], 0.09, 0.6)
        assert torch.equal(a2, alen) and torch.equal(n2, anodes) and torch.equal(x2, nxt)


def test_accept_typical_uniform_rows_accept_lowest_deepest():
    """Uniform verify rows over V = 8: p = 1/8 exceeds min(0.09, 0.6/8) = 0.075,
    so every node is accepted and the deepest node with the lowest index wins."""
    K, s, N, V = 3, 2, 15, 8
    t = api.Tree(K, s, N)
    plan = O.tree_plan(K, s, N)
    vlog = torch.zeros(1, N, V, device=DEV)
    tok = torch.tensor([[n % V for n in range(N)]], dtype=torch.int32, device=DEV)
    alen, anodes, nxt = api.medusa_accept_typical(vlog, tok, t, 1.0)
    ra, rn, rx, _ = O.accept_typical(vlog, tok, plan, 1.0)
    assert alen.item() == ra[0] == K and anodes.cpu().numpy()[0].tolist() == rn[0].tolist()


# ---------------------------------------------------------------------------- compaction
@pytest.mark.parametrize("dtype,Hkv,dh", [(torch.bfloat16, 4, 128), (torch.float32, 3, 64),
                                          (torch.bfloat16, 1, 2)])
def test_kv_compact_exact(dtype, Hkv, dh):
    B, K, Lcap = 4, 5, 120
    g = torch.Generator(device=DEV).manual_seed(9)
    kc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    vc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    L = torch.tensor([10, 0, 50, 100], dtype=torch.int32, device=DEV)
    A = torch.tensor([3, 0, 5, 1], dtype=torch.int32, device=DEV)
    nodes = torch.tensor([[0, 1, 4, 9, -1, -1], [0, -1, -1, -1, -1, -1], [0, 2, 6, 7, 11, 19],
                          [0, 1, -1, -1, -1, -1]], dtype=torch.int32, device=DEV)
    rk, rv, rl = O.kv_compact(kc, vc, L, A, nodes)
    new_len = api.medusa_kv_compact(kc, vc, L, A, nodes, K)
    assert (new_len.cpu().numpy() == rl).all()
    np.testing.assert_array_equal(kc.double().cpu().numpy(), rk)
    np.testing.assert_array_equal(vc.double().cpu().numpy(), rv)


def test_device_status_clean():
    assert api.device_status(clear=True) == 0


@pytest.mark.parametrize("B,K,s,N,V,dtype,T", [
    (4, 5, 3, 256, 32000, "bf16", 0.7),
    (3, 5, 10, 64, 1000, "bf16", 1.3),
    (2, 4, 3, 16, 1024, "f32", 0.5),
])
def test_accept_greedy_typical_in_one_pass_equals_the_two_calls(B, K, s, N, V, dtype, T):
    """medusa_accept_greedy_typical writes what medusa_accept_greedy and
    medusa_accept_typical write for the same arguments, bit for bit, and the
    greedy half equals the oracle's sequential argmax decoding."""
    cfg = MedusaConfig("both", dtype, B=B, d=8, V=V, K=K, s=s, N=N, Hq=1, Hkv=1, dh=64,
                       L_lo=0, L_hi=0)
    plan = O.tree_plan(K, s, N)
    g = torch.Generator().manual_seed(B * N + V)
    topk = torch.stack([torch.randperm(V, generator=g)[:K * s].view(K, s) for _ in range(B)])
    tok, _ = O.build_tree(plan, torch.randint(0, V, (B,), generator=g), topk, [0] * B)
    vlog = plant_verify_logits(cfg, plan["parent"], tok, device=DEV, seed=B + K)
    tok_d = torch.as_tensor(tok, dtype=torch.int32, device=DEV)
    tree = api.Tree(K, s, N)
    rg = api.medusa_accept_greedy(vlog, tok_d, tree)
    rt = api.medusa_accept_typical(vlog, tok_d, tree, T)
    fg, ft = api.medusa_accept_greedy_typical(vlog, tok_d, tree, T)
    torch.cuda.synchronize()
    for a, b in zip(fg + ft, rg + rt):
        assert torch.equal(a, b)
    ref = O.accept_greedy(vlog, tok, plan)
    assert (fg[0].cpu().numpy() == ref[0]).all()
    assert api.device_status() == 0
