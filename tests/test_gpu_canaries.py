"""GPU: poisoned canaries around every buffer the verify step's calls write.

Each output tensor, each caller workspace (of exactly the size the library
reports) and each KV cache sits between two 4 KB guard bands filled with a
NaN pattern, and the output tensors themselves start out filled with it.
After each call: both guard bands of every buffer are intact (nothing is
written before or after a buffer, nor into the caches by the calls that
only read them), every element of an output the call must fill has been
written, no written float is NaN, and each output equals, bit for bit, the
same call made on freshly allocated buffers.  The chain is the verify step
of the Medusa paper digest ([MD] "ツリーアテンションによる並列検証"): heads +
top-s, tree expansion, tree attention, acceptance, next-token sampling,
compaction (both acceptance rules separately and in one pass), plus the
shard merge.
"""
import ctypes as C
import math

import pytest
import torch

from canary import Guarded, GuardedWorkspace
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import _lib as L
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.synthetic import (MedusaConfig, gen_inputs,
                                                       plant_verify_logits)

pytestmark = pytest.mark.gpu
DEV = "cuda"
F32, I32 = torch.float32, torch.int32


def _filled(g: Guarded, want_nan_free: bool = True):
    assert g.intact(), "guard band overwritten"
    assert g.untouched() == 0, f"{g.untouched()} elements never written"
    if want_nan_free and g.dtype.is_floating_point:
        assert not torch.isnan(g.t.float()).any()



def _guarded_copy(t):
    g = Guarded(t.shape, t.dtype, t.device)
    g.t.copy_(t)
    return g


CASES = [
    # name, dtype, B, d, V, K, s, N, Hq, Hkv, dh, L_lo, L_hi
    ("b1_gqa", "bf16", 1, 512, 4099, 5, 10, 64, 8, 2, 128, 700, 700),
    ("b4_chunks", "bf16", 4, 256, 1000, 5, 3, 256, 2, 2, 128, 70, 5000),
    ("b40_big_heads", "bf16", 40, 256, 700, 3, 4, 16, 4, 4, 128, 100, 300),
    ("f32_simt", "f32", 2, 128, 1024, 4, 3, 16, 4, 4, 64, 128, 200),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_step_calls_stay_inside_their_buffers(case):
    name, dtype, B, d, V, K, s, N, Hq, Hkv, dh, L_lo, L_hi = case
    cfg = MedusaConfig(name, dtype, B=B, d=d, V=V, K=K, s=s, N=N, Hq=Hq, Hkv=Hkv, dh=dh,
                       L_lo=L_lo, L_hi=L_hi, headroom=3)
    dt = cfg.torch_dtype
    x = gen_inputs(cfg, DEV, seed=len(name))
    tree = api.Tree(K, s, N)

    # heads + top-s (logits and top-s; top-s only)
    ref = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s)
    gl, gi, gv = Guarded((B, K, V), F32, DEV), Guarded((B, K, s), I32, DEV), \
        Guarded((B, K, s), F32, DEV)
    ws = GuardedWorkspace(api.heads_workspace_size(B, d, V, K, s, dt), DEV)
    api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s, out=(gl.t, gi.t, gv.t),
                             ws=ws.t)
    gi2, gv2 = Guarded((B, K, s), I32, DEV), Guarded((B, K, s), F32, DEV)
    api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s, want_logits=False,
                             out=(None, gi2.t, gv2.t), ws=ws.t)
    torch.cuda.synchronize()
    assert ws.intact()
    for g, r in ((gl, ref[0]), (gi, ref[1]), (gv, ref[2]), (gi2, ref[1]), (gv2, ref[2])):
        _filled(g)
        assert torch.equal(g.t, r)

    # top-s of stored logits
    ti, tv = Guarded((B, K, s), I32, DEV), Guarded((B, K, s), F32, DEV)
    L.check(L.lib().medusa_topk(C.c_void_p(ref[0].data_ptr()), L.F32, B * K, V, s,
                                C.c_void_p(ti.t.data_ptr()), C.c_void_p(tv.t.data_ptr()),
                                C.c_void_p(torch.cuda.current_stream().cuda_stream)),
            "medusa_topk")
    # merge of two half-vocabulary candidate lists
    half = V // 2
    c1 = api.medusa_topk(ref[0][..., :half].contiguous(), s)
    c2 = api.medusa_topk(ref[0][..., half:].contiguous(), s)
    vals = torch.stack([c1[1].view(B * K, s), c2[1].view(B * K, s)])
    idxs = torch.stack([c1[0].view(B * K, s), c2[0].view(B * K, s)])
    v0 = torch.tensor([0, half], dtype=I32, device=DEV)
    mi, mv = Guarded((B * K, s), I32, DEV), Guarded((B * K, s), F32, DEV)
    api.medusa_topk_merge(vals, idxs, s, v0, out=(mi.t, mv.t))
    torch.cuda.synchronize()
    for g in (ti, tv, mi, mv):
        _filled(g)
    assert torch.equal(ti.t, ref[1]) and torch.equal(tv.t, ref[2])
    assert torch.equal(mi.t.view(B, K, s), ref[1]) and torch.equal(mv.t.view(B, K, s), ref[2])

    # tree expansion
    rtok, rpos = api.medusa_build_tree(tree, x["root_tok"], ref[1], x["prefix_len"])
    gt, gp = Guarded((B, N), I32, DEV), Guarded((B, N), I32, DEV)
    api.medusa_build_tree(tree, x["root_tok"], ref[1], x["prefix_len"], out=(gt.t, gp.t))
    torch.cuda.synchronize()
    _filled(gt)
    _filled(gp)
    assert torch.equal(gt.t, rtok) and torch.equal(gp.t, rpos)

    # tree attention over guarded caches
    kc, vc = _guarded_copy(x["k_cache"]), _guarded_copy(x["v_cache"])
    scale = 1.0 / math.sqrt(dh)
    ra = api.medusa_tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], tree,
                                   scale)
    go = Guarded(x["q"].shape, dt, DEV)
    wsa = GuardedWorkspace(api.attention_workspace_size(tree, B, Hq, Hkv, dh, cfg.Lcap), DEV)
    api.medusa_tree_attention(x["q"], kc.t, vc.t, x["prefix_len"], tree, scale, out=go.t,
                              ws=wsa.t)
    torch.cuda.synchronize()
    assert wsa.intact() and kc.intact() and vc.intact()
    assert torch.equal(kc.t, x["k_cache"]) and torch.equal(vc.t, x["v_cache"])
    _filled(go)
    assert torch.equal(go.t, ra)

    # acceptance (greedy, typical, typical per head) and the sampled next token
    plan = O.tree_plan(K, s, N)
    vlog = plant_verify_logits(cfg, plan["parent"], rtok.cpu(), DEV, seed=3)
    wsc = GuardedWorkspace(api.accept_workspace_size(tree, B, V), DEV)
    temps = [0.7 + 0.1 * i for i in range(K)]
    calls = [
        lambda out, w: api.medusa_accept_greedy(vlog, rtok, tree, out=out, ws=w),
        lambda out, w: api.medusa_accept_typical(vlog, rtok, tree, 0.7, out=out, ws=w),
        lambda out, w: api.medusa_accept_typical_per_head(vlog, rtok, tree, temps, out=out, ws=w),
    ]
    accepted = None
    for call in calls:
        r = call(None, None)
        g = (Guarded((B,), I32, DEV), Guarded((B, K + 1), I32, DEV), Guarded((B,), I32, DEV))
        call(tuple(q.t for q in g), wsc.t)
        torch.cuda.synchronize()
        assert wsc.intact()
        for q, rr in zip(g, r):
            _filled(q)
            assert torch.equal(q.t, rr)
        accepted = accepted or r
    # both rules from one pass: two guarded output sets
    rg = api.medusa_accept_greedy(vlog, rtok, tree)
    rt = api.medusa_accept_typical(vlog, rtok, tree, 0.7)
    gg = tuple(Guarded(x.shape, I32, DEV) for x in rg)
    gt2 = tuple(Guarded(x.shape, I32, DEV) for x in rt)
    api.medusa_accept_greedy_typical(vlog, rtok, tree, 0.7, out_greedy=tuple(q.t for q in gg),
                                     out_typical=tuple(q.t for q in gt2), ws=wsc.t)
    torch.cuda.synchronize()
    assert wsc.intact()
    for q, rr in zip(gg + gt2, rg + rt):
        _filled(q)
        assert torch.equal(q.t, rr)
    alen, anodes, _ = accepted
    for temp in (0.0, 0.8):
        rn = api.medusa_sample_next(vlog, alen, anodes, temp, seed=5, offset=1)
        gn = Guarded((B,), I32, DEV)
        api.medusa_sample_next(vlog, alen, anodes, temp, seed=5, offset=1, out=gn.t)
        torch.cuda.synchronize()
        _filled(gn)
        assert torch.equal(gn.t, rn)

    # compaction inside the guarded caches
    k2, v2 = x["k_cache"].clone(), x["v_cache"].clone()
    rl = api.medusa_kv_compact(k2, v2, x["prefix_len"], alen, anodes, K)
    gn = Guarded((B,), I32, DEV)
    api.medusa_kv_compact(kc.t, vc.t, x["prefix_len"], alen, anodes, K, new_len=gn.t)
    torch.cuda.synchronize()
    assert kc.intact() and vc.intact()
    _filled(gn)
    assert torch.equal(gn.t, rl)
    assert torch.equal(kc.t, k2) and torch.equal(vc.t, v2)
    assert api.device_status() == 0
