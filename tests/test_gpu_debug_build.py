"""GPU: the MEDUSA_DEBUG build (libmedusa_debug.so, device-side index checks).

Run in a child process with MEDUSA_DEBUG=1, so the binding loads the debug
library.  On valid inputs it must give the release library's results bit
for bit and a clean status word.  Inputs whose indices fall outside the
tree, the cache or the vocabulary are turned into MEDUSA_ERR_BOUNDS by the
kernels' own checks, which skip the access: a tree token outside [0, V) in
the acceptance walk (check site 5) and an accepted node whose slot lies
past the cache in the compaction (site 6).  No access goes out of range:
the release build skips the same entries by its documented rules.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

from medusa_head_speculative_02_b200 import _lib as L
from medusa_head_speculative_02_b200 import api

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, math, sys
import torch
sys.path.insert(0, ROOT)
from medusa_head_speculative_02_b200 import _lib as L, api
from medusa_head_speculative_02_b200.synthetic import MedusaConfig, gen_inputs, plant_verify_logits
out = {"version": api.version()}
cfg = MedusaConfig("dbg", "bf16", B=2, d=512, V=1000, K=4, s=3, N=16, Hq=4, Hkv=2, dh=128,
                   L_lo=100, L_hi=200)
x = gen_inputs(cfg, "cuda", 0)
t = api.Tree(cfg.K, cfg.s, cfg.N)
_, idx, _ = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=cfg.s,
                                     want_logits=False)
tok, pos = api.medusa_build_tree(t, x["root_tok"], idx, x["prefix_len"])
att = api.medusa_tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], t,
                                1 / math.sqrt(cfg.dh))
vlog = plant_verify_logits(cfg, t.info()[0], tok.cpu(), "cuda", 0)
alen, anodes, nxt = api.medusa_accept_greedy(vlog, tok, t)
ta, tn, tx = api.medusa_accept_typical(vlog, tok, t, 0.7)
new_len = api.medusa_kv_compact(x["k_cache"], x["v_cache"], x["prefix_len"], alen, anodes, cfg.K)
torch.cuda.synchronize()
out["valid_status"] = api.device_status()
torch.save({"idx": idx.cpu(), "tok": tok.cpu(), "pos": pos.cpu(), "att": att.cpu(),
            "alen": alen.cpu(), "anodes": anodes.cpu(), "nxt": nxt.cpu(), "ta": ta.cpu(),
            "tn": tn.cpu(), "tx": tx.cpu(), "new_len": new_len.cpu(),
            "k": x["k_cache"].cpu()}, OUT)

# a tree token outside the vocabulary: the walk's check (site 5) reports it
bad = tok.clone()
bad[0, 3] = cfg.V + 5
api.medusa_accept_greedy(vlog, bad, t)
torch.cuda.synchronize()
out["token_status"] = api.device_status()
out["token_error"] = L.lib().medusa_last_error().decode()
# an accepted node whose source slot lies past the cache: skipped, site 6
A = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
nodes = torch.full((2, cfg.K + 1), -1, dtype=torch.int32, device="cuda")
nodes[0, 0], nodes[0, 1] = 0, x["k_cache"].shape[1]
before = x["k_cache"].clone()
api.medusa_kv_compact(x["k_cache"], x["v_cache"], x["prefix_len"], A, nodes, cfg.K)
torch.cuda.synchronize()
out["compact_status"] = api.device_status()
out["compact_error"] = L.lib().medusa_last_error().decode()
out["cache_unchanged"] = bool(torch.equal(before, x["k_cache"]))
out["final_status"] = api.device_status()
print(json.dumps(out))
"""


def _release_results():
    import math
    from medusa_head_speculative_02_b200.synthetic import (MedusaConfig, gen_inputs,
                                                           plant_verify_logits)
    cfg = MedusaConfig("dbg", "bf16", B=2, d=512, V=1000, K=4, s=3, N=16, Hq=4, Hkv=2, dh=128,
                       L_lo=100, L_hi=200)
    x = gen_inputs(cfg, "cuda", 0)
    t = api.Tree(cfg.K, cfg.s, cfg.N)
    _, idx, _ = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=cfg.s,
                                         want_logits=False)
    tok, pos = api.medusa_build_tree(t, x["root_tok"], idx, x["prefix_len"])
    att = api.medusa_tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], t,
                                    1 / math.sqrt(cfg.dh))
    vlog = plant_verify_logits(cfg, t.info()[0], tok.cpu(), "cuda", 0)
    alen, anodes, nxt = api.medusa_accept_greedy(vlog, tok, t)
    ta, tn, tx = api.medusa_accept_typical(vlog, tok, t, 0.7)
    new_len = api.medusa_kv_compact(x["k_cache"], x["v_cache"], x["prefix_len"], alen, anodes,
                                    cfg.K)
    torch.cuda.synchronize()
    return {"idx": idx, "tok": tok, "pos": pos, "att": att, "alen": alen, "anodes": anodes,
            "nxt": nxt, "ta": ta, "tn": tn, "tx": tx, "new_len": new_len, "k": x["k_cache"]}


def test_debug_build_matches_release_and_reports_bad_indices(tmp_path):
    assert not L.DEBUG, "the parent test process uses the release library"
    if not os.path.exists(os.path.join(ROOT, "medusa_head_speculative_02_b200",
                                       "libmedusa_debug.so")):
        pytest.fail("libmedusa_debug.so is missing: build with "
                    "`python -m medusa_head_speculative_02_b200.build`")
    out_file = str(tmp_path / "debug.pt")
    code = f"ROOT = {ROOT!r}\nOUT = {out_file!r}\n" + CHILD
    env = dict(os.environ, MEDUSA_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert "MEDUSA_DEBUG" in res["version"]
    assert res["valid_status"] == L.OK
    assert res["token_status"] == L.ERR_BOUNDS and "site 5" in res["token_error"]
    assert res["compact_status"] == L.ERR_BOUNDS and "site 6" in res["compact_error"]
    assert res["cache_unchanged"] and res["final_status"] == L.OK
    dbg = torch.load(out_file)
    rel = _release_results()
    for k, v in rel.items():
        assert torch.equal(v.cpu(), dbg[k]), k
    assert api.device_status() == L.OK
