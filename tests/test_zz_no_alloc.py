"""medusa_accept_greedy_noalloc: greedy acceptance for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Called through the C ABI directly.  Two calls in a row, on different inputs,
must each reproduce the workspace-taking medusa_accept_greedy exactly (the
shared scratch keeps the previous call's contents, which must not leak into
the next result).  Collected last so a stop-at-first-failure run has already
run every other test.
"""
import ctypes as C

import pytest
import torch

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import _lib as L
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.synthetic import MedusaConfig, plant_verify_logits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, K, s, N, V, dtype, seed):
    cfg = MedusaConfig("na", dtype, B=B, d=8, V=V, K=K, s=s, N=N, Hq=1, Hkv=1, dh=64,
                       L_lo=0, L_hi=0)
    plan = O.tree_plan(K, s, N)
    g = torch.Generator().manual_seed(seed)
    topk = torch.stack([torch.randperm(V, generator=g)[:K * s].view(K, s) for _ in range(B)])
    tok, _ = O.build_tree(plan, torch.randint(0, V, (B,), generator=g), topk, [0] * B)
    vlog = plant_verify_logits(cfg, plan["parent"], tok, device=DEV, seed=seed)
    return vlog, torch.as_tensor(tok, dtype=torch.int32, device=DEV)


def _noalloc(vlog, tok, tree, out):
    alen, anodes, nxt = out
    B, N, V = vlog.shape
    dt = L.F32 if vlog.dtype == torch.float32 else L.BF16
    rc = L.lib().medusa_accept_greedy_noalloc(
        C.c_void_p(vlog.data_ptr()), dt, C.c_void_p(tok.data_ptr()), tree.handle, B, V,
        C.c_void_p(alen.data_ptr()), C.c_void_p(anodes.data_ptr()), C.c_void_p(nxt.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    L.check(rc, "medusa_accept_greedy_noalloc")


@pytest.mark.parametrize("cases", [
    [(4, 5, 10, 64, 32000, "bf16", 1), (2, 4, 3, 16, 1024, "f32", 2)],
    [(16, 5, 8, 128, 128256, "bf16", 3), (16, 5, 8, 128, 128256, "bf16", 4)],
])
def test_noalloc_matches_workspace_entry_point_twice(cases):
    for (B, K, s, N, V, dtype, seed) in cases:
        vlog, tok = _inputs(B, K, s, N, V, dtype, seed)
        tree = api.Tree(K, s, N)
        ref = api.medusa_accept_greedy(vlog, tok, tree)
        out = tuple(torch.full_like(t, -7) for t in ref)
        _noalloc(vlog, tok, tree, out)
        torch.cuda.synchronize()
        for a, b in zip(out, ref):
            assert torch.equal(a, b)


def test_noalloc_rejects_rows_beyond_its_scratch():
    tree = api.Tree(5, 3, 256)
    too_many = 65536 // 256 + 1
    p = C.c_void_p(256)
    rc = L.lib().medusa_accept_greedy_noalloc(p, L.BF16, p, tree.handle, too_many, 1000, p, p, p,
                                              None)
    assert rc == L.ERR_INVALID_ARG
    assert b"scratch" in L.lib().medusa_last_error()
