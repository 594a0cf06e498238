"""The multi-step decode loop: each step's next token is the next root and its
new lengths the next prefix lengths.  Checked against (1) the same chain
replayed from a CUDA graph, bit for bit, and (2) the oracle run as the same
chain on the CPU, step by step."""
import math

import numpy as np
import pytest
import torch

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200.decode import DecodeLoop
from medusa_head_speculative_02_b200.synthetic import MedusaConfig

pytestmark = pytest.mark.gpu

# small bf16 shapes on the tensor-core paths: 128-wide heads tiles, dh = 128,
# GQA group 2, a ragged batch
CFG = MedusaConfig("decode_small", "bf16", B=3, d=512, V=1000, K=4, s=3, N=16, Hq=4, Hkv=2,
                   dh=128, L_lo=100, L_hi=300)


def _outputs(st):
    return {k: getattr(st, k).clone() for k in
            ("topk_idx", "tree_tok", "tree_pos", "attn_out", "accept_len", "accept_nodes",
             "next_tok", "new_len")}


def test_graph_replay_equals_eager_chain():
    steps = 4
    loop = DecodeLoop(CFG, "cuda", seed=1, max_steps=steps + 1)
    eager = []
    for _ in range(steps):
        loop.step()
        eager.append(_outputs(loop.st))
    kc, vc = loop.st.x["k_cache"].clone(), loop.st.x["v_cache"].clone()
    loop.reset()
    loop.capture()
    for i in range(steps):
        loop.step()
        got = _outputs(loop.st)
        for k, v in eager[i].items():
            assert torch.equal(got[k], v), (i, k)
    assert torch.equal(loop.st.x["k_cache"], kc) and torch.equal(loop.st.x["v_cache"], vc)
    # the chain actually advanced: prefix lengths grew by 1 + accept_len per step
    L0 = loop._init["prefix_len"].long()
    total = sum(1 + e["accept_len"].long() for e in eager)
    assert torch.equal(loop.st.x["prefix_len"].long(), L0 + total)


def test_eager_chain_matches_oracle_chain():
    steps = 3
    loop = DecodeLoop(CFG, "cuda", seed=2, max_steps=steps)
    st, cfg = loop.st, loop.cfg
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    x = {k: v.cpu() for k, v in st.x.items()}
    vlog = st.vlogits.cpu()
    L = x["prefix_len"].numpy().astype(np.int64)
    root = x["root_tok"].numpy().astype(np.int64)
    kc, vc = O.f64(x["k_cache"]), O.f64(x["v_cache"])
    logits = O.heads_forward(x["h"], x["W1"], x["b1"], x["W2"])
    ref_idx = O.topk(logits, cfg.s)
    srt = -np.sort(-logits, axis=-1)
    gap = srt[..., :cfg.s] - srt[..., 1:cfg.s + 1]          # gap below each rank
    scale = 1.0 / math.sqrt(cfg.dh)
    rng = np.random.default_rng(0)
    for step in range(steps):
        loop.step()
        torch.cuda.synchronize()
        # heads: the same h every step; top-s exact wherever the order is clear
        idx = st.topk_idx.cpu().numpy()
        clear = np.minimum.accumulate(gap, axis=-1) > 1e-2
        assert (idx[clear] == ref_idx[clear]).all()
        # tree expansion from this step's root and prefix lengths (GPU top-s
        # fed in, so that the rest of the chain compares exactly)
        tok, pos = O.build_tree(plan, root, idx, L)
        assert (st.tree_tok.cpu().numpy() == tok).all()
        assert (st.tree_pos.cpu().numpy() == pos).all()
        # attention on the oracle's own cache state, sampled rows
        rows = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.N)), int(rng.integers(cfg.Hq)))
                for _ in range(24)]
        ref = O.tree_attention(x["q"], kc, vc, L, plan, scale, rows=rows)
        out = st.attn_out.cpu()
        got = np.stack([O.f64(out[b, i, h]) for (b, i, h) in rows])
        assert np.abs(got - ref).max() <= 2e-2
        # greedy acceptance and compaction
        alen, anodes, nxt = O.accept_greedy(vlog, tok, plan)
        assert (st.accept_len.cpu().numpy() == alen).all()
        assert (st.accept_nodes.cpu().numpy() == anodes).all()
        assert (st.next_tok.cpu().numpy() == nxt).all()
        kc, vc, new_len = O.kv_compact(kc, vc, L, alen, anodes)
        assert (st.new_len.cpu().numpy() == new_len).all()
        assert np.array_equal(O.f64(st.x["k_cache"].cpu()), kc)
        assert np.array_equal(O.f64(st.x["v_cache"].cpu()), vc)
        # the chain: next token -> root, new lengths -> prefix lengths
        L, root = new_len, nxt
        assert (st.x["prefix_len"].cpu().numpy() == L).all()
        assert (st.x["root_tok"].cpu().numpy() == root).all()


def test_headroom_bounds_the_step_count():
    loop = DecodeLoop(CFG, "cuda", seed=3, max_steps=2)
    assert loop.cfg.Lcap == CFG.L_hi + CFG.N + 2 * (CFG.K + 1)
    loop.step()
    loop.step()
    with pytest.raises(RuntimeError):
        loop.step()


CFG_TYP = CFG.scaled(name="decode_small_typical", accept="typical", temperature=0.8)


def test_sampling_chain_graph_equals_eager_and_draws_fresh_noise():
    steps = 4
    loop = DecodeLoop(CFG_TYP, "cuda", seed=5, max_steps=steps + 1, sample_temperature=0.9,
                      sample_seed=77)
    eager = []
    for _ in range(steps):
        loop.step()
        eager.append(_outputs(loop.st))
    assert int(loop.draws.item()) == steps
    loop.reset()
    loop.capture()
    for i in range(steps):
        loop.step()
        got = _outputs(loop.st)
        for k, v in eager[i].items():
            assert torch.equal(got[k], v), (i, k)
    assert int(loop.draws.item()) == steps


def test_sampling_chain_matches_oracle_chain():
    """Typical acceptance, then the next token drawn at offset = step index."""
    steps, T_s, seed_s = 3, 0.9, 123
    loop = DecodeLoop(CFG_TYP, "cuda", seed=6, max_steps=steps, sample_temperature=T_s,
                      sample_seed=seed_s)
    st, cfg = loop.st, loop.cfg
    plan = O.tree_plan(cfg.K, cfg.s, cfg.N)
    vlog = st.vlogits.cpu()
    L = st.x["prefix_len"].cpu().numpy().astype(np.int64)
    root = st.x["root_tok"].cpu().numpy().astype(np.int64)
    kc, vc = O.f64(st.x["k_cache"].cpu()), O.f64(st.x["v_cache"].cpu())
    for step in range(steps):
        loop.step()
        torch.cuda.synchronize()
        idx = st.topk_idx.cpu().numpy()
        tok, _ = O.build_tree(plan, root, idx, L)
        assert (st.tree_tok.cpu().numpy() == tok).all()
        alen, anodes, _, margin = O.accept_typical(vlog, tok, plan, cfg.temperature, cfg.eps,
                                                   cfg.delta)
        assert (margin > 1e-5).all()          # no decision too close to call
        assert (st.accept_len.cpu().numpy() == alen).all()
        assert (st.accept_nodes.cpu().numpy() == anodes).all()
        nxt, gap = O.sample_next(vlog, alen, anodes, T_s, seed_s, step)
        got = st.next_tok.cpu().numpy()
        assert ((got == nxt) | (gap < 1e-5)).all() and (gap >= 1e-5).all()
        kc, vc, new_len = O.kv_compact(kc, vc, L, alen, anodes)
        assert (st.new_len.cpu().numpy() == new_len).all()
        assert np.array_equal(O.f64(st.x["k_cache"].cpu()), kc)
        L, root = new_len, nxt
