"""Full-size parity at the five workload configurations, through the same
calls, workspaces and launch configuration the benchmark times
(medusa_head_speculative_02_b200.step.VerifyStep).  Outputs too large for the
oracle are sampled: logits and top-s on a few (sequence, head) rows over the
whole vocabulary, attention on rows spread over sequences / nodes / heads;
tree expansion, acceptance and compaction are checked completely, with the
acceptance inputs (tree tokens, planted verify logits) built on the oracle
side."""
import math

import numpy as np
import pytest
import torch

from attn_check import assert_attention_close
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.step import VerifyStep
from medusa_head_speculative_02_b200.synthetic import CONFIGS, plant_verify_logits

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
ATOL = 2e-2
GAP = 1e-2


@pytest.fixture(scope="module", params=["tiny_f32", "7b_b1", "13b_b8", "8b_gqa_b16", "longctx_b4"])
def step(request):
    st = VerifyStep(CONFIGS[request.param], "cuda", seed=0)
    yield st
    del st
    torch.cuda.empty_cache()


def _oracle_logits_row(x, b, k, chunk=16384):
    """Oracle logits of head k for sequence b over the whole vocabulary."""
    u = O.heads_hidden(x["h"][b:b + 1], x["W1"], x["b1"], k)
    V = x["W2"].shape[1]
    out = np.empty(V)
    for lo in range(0, V, chunk):
        hi = min(V, lo + chunk)
        out[lo:hi] = O.heads_logits(u, x["W2"][k:k + 1], 0, vocab=np.arange(lo, hi))[0]
    return out


def test_heads_full_size_sampled(step):
    cfg, x = step.cfg, step.x
    logits, idx, val = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=cfg.s,
                                                ws=step.ws_heads)
    # the benchmark's call (top-s only) must agree with this one
    step.heads()
    torch.cuda.synchronize()
    assert torch.equal(step.topk_idx, idx)
    samples = sorted({(0, 0), (cfg.B - 1, cfg.K - 1), (cfg.B // 2, cfg.K // 2)})
    for b, k in samples:
        ref = _oracle_logits_row(x, b, k)
        got = logits[b, k].double().cpu().numpy()
        assert np.abs(got - ref).max() <= ATOL, (b, k, np.abs(got - ref).max())
        order = O.topk_row(ref, cfg.s + 1)
        vals = ref[order]
        gi = idx[b, k].cpu().numpy()
        for j in range(cfg.s):
            left = j == 0 or vals[j - 1] - vals[j] > GAP
            right = vals[j] - vals[j + 1] > GAP
            if left and right:
                assert gi[j] == order[j], (b, k, j)


def test_build_tree_full_size(step):
    cfg, x = step.cfg, step.x
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator(device="cuda").manual_seed(3)
    topk = torch.randint(0, cfg.V, (cfg.B, cfg.K, cfg.s), generator=g, device="cuda",
                         dtype=torch.int32)
    tok, pos = api.medusa_build_tree(step.tree, x["root_tok"], topk, x["prefix_len"])
    rt, rp = O.build_tree(plan, x["root_tok"], topk, x["prefix_len"])
    assert (tok.cpu().numpy() == rt).all() and (pos.cpu().numpy() == rp).all()


def test_attention_full_size_sampled(step):
    cfg, x = step.cfg, step.x
    step.attention()
    torch.cuda.synchronize()
    out = step.attn_out
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    nodes = sorted({0, 1, cfg.N // 2, cfg.N - 1})
    heads = sorted({0, cfg.Hq // 2, cfg.Hq - 1})
    rows = [(b, i, h) for b in range(cfg.B) for i in nodes for h in heads]
    if len(rows) > 96:
        rows = rows[::len(rows) // 96 + 1]
    ref = O.tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], plan,
                           1.0 / math.sqrt(cfg.dh), rows=rows)
    got = np.stack([out[b, i, h].double().cpu().numpy() for (b, i, h) in rows])
    assert_attention_close(got, ref, bf16=cfg.dtype == "bf16", what=f"{cfg.name} sampled rows")


def test_attention_full_size_whole_kv_head(step):
    """Every output row of one (sequence, kv-head): all tree nodes x the GQA
    group, so every query tile of the pair, every key chunk and every tree
    tile is compared, on the sequence with the longest prefix."""
    cfg, x = step.cfg, step.x
    step.attention()
    torch.cuda.synchronize()
    out = step.attn_out
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    b = int(torch.argmax(x["prefix_len"]).item())
    kvh = cfg.Hkv - 1
    G = cfg.Hq // cfg.Hkv
    rows = [(b, i, kvh * G + g) for i in range(cfg.N) for g in range(G)]
    ref = O.tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], plan,
                           1.0 / math.sqrt(cfg.dh), rows=rows)
    got = out[b, :, kvh * G:(kvh + 1) * G].double().cpu().numpy().reshape(-1, cfg.dh)
    assert_attention_close(got, ref, bf16=cfg.dtype == "bf16",
                           what=f"{cfg.name} sequence {b} kv-head {kvh}, {len(rows)} rows")


def _accept_inputs(cfg, tree_parent):
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    g = torch.Generator().manual_seed(5)
    topk = torch.stack([torch.randperm(cfg.V, generator=g)[:cfg.K * cfg.s].view(cfg.K, cfg.s)
                        for _ in range(cfg.B)])
    tok, _ = O.build_tree(plan, torch.randint(0, cfg.V, (cfg.B,), generator=g), topk,
                          [0] * cfg.B)
    vlog = plant_verify_logits(cfg, plan["parent"], tok, device="cuda", seed=5)
    return plan, torch.as_tensor(tok, dtype=torch.int32, device="cuda"), vlog


def test_accept_full_size(step):
    cfg = step.cfg
    plan, tok, vlog = _accept_inputs(cfg, None)
    ws = step.ws_acc
    if cfg.accept in ("greedy", "both"):
        a = api.medusa_accept_greedy(vlog, tok, step.tree, ws=ws)
        r = O.accept_greedy(vlog, tok, plan)
        for got, ref in zip(a, r):
            assert (got.cpu().numpy() == ref).all()
    if cfg.accept in ("typical", "both"):
        a = api.medusa_accept_typical(vlog, tok, step.tree, cfg.temperature, cfg.eps, cfg.delta,
                                      ws=ws)
        ra, rn, rx, margin = O.accept_typical(vlog, tok, plan, cfg.temperature, cfg.eps, cfg.delta)
        alen, anodes, nxt = (t.cpu().numpy() for t in a)
        checked = 0
        for b in range(cfg.B):
            if (margin[b, 1:] < 1e-5).any():
                continue                     # a decision too close to call
            checked += 1
            assert alen[b] == ra[b] and (anodes[b] == rn[b]).all() and nxt[b] == rx[b]
        assert checked >= cfg.B - 1


def test_kv_compact_full_size(step):
    cfg, x = step.cfg, step.x
    g = torch.Generator().manual_seed(7)
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    # an accepted path per sequence: the deepest-first walk of random children
    A, nodes = [], []
    for b in range(cfg.B):
        path = [0]
        for _ in range(int(torch.randint(0, cfg.K + 1, (), generator=g))):
            ch = [c for c in range(cfg.N) if plan["parent"][c] == path[-1]]
            if not ch:
                break
            path.append(ch[int(torch.randint(0, len(ch), (), generator=g))])
        A.append(len(path) - 1)
        nodes.append(path + [-1] * (cfg.K + 1 - len(path)))
    A = torch.tensor(A, dtype=torch.int32, device="cuda")
    nodes = torch.tensor(nodes, dtype=torch.int32, device="cuda")
    L = x["prefix_len"]
    Ls = [int(v) for v in L.tolist()]
    before_k = [x["k_cache"][b, Ls[b]:Ls[b] + cfg.N].clone() for b in range(cfg.B)]
    before_v = [x["v_cache"][b, Ls[b]:Ls[b] + cfg.N].clone() for b in range(cfg.B)]
    edge_k = [x["k_cache"][b, max(0, Ls[b] - 2):Ls[b]].clone() for b in range(cfg.B)]
    new_len = api.medusa_kv_compact(x["k_cache"], x["v_cache"], L, A, nodes, cfg.K)
    torch.cuda.synchronize()
    for b in range(cfg.B):
        # the oracle on this sequence's tree region (prefix length 0 relative to it)
        rk, rv, rl = O.kv_compact(before_k[b][None], before_v[b][None], [0], A[b:b + 1],
                                  nodes[b:b + 1])
        got_k = x["k_cache"][b, Ls[b]:Ls[b] + cfg.N].double().cpu().numpy()
        got_v = x["v_cache"][b, Ls[b]:Ls[b] + cfg.N].double().cpu().numpy()
        assert (got_k == rk[0]).all() and (got_v == rv[0]).all()
        assert int(new_len[b]) == Ls[b] + 1 + int(A[b])
        assert torch.equal(x["k_cache"][b, max(0, Ls[b] - 2):Ls[b]], edge_k[b])
