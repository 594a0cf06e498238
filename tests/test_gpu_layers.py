"""GPU: verification through several layers ([MD] "ツリーアテンションによる並列
検証": the tree is verified in one forward pass of the base model, every
layer attending over its own cache with the same tree, and the accepted
path is then kept in every layer's cache).

Per-layer tree attention (one medusa_tree_attention call per layer, on that
layer's queries and cache) against the oracle's tree_attention_layers, and
medusa_kv_compact_layers (one launch over all layers) against the oracle's
kv_compact_layers bit for bit, with contiguous and padded layer strides.
"""
import ctypes as C
import math

import numpy as np
import pytest
import torch

from attn_check import assert_attention_close
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import _lib as L
from medusa_head_speculative_02_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _paths(plan, B, K, seed):
    """An accepted root-first path per sequence (random children)."""
    g = torch.Generator().manual_seed(seed)
    A, nodes = [], []
    N = plan["N"]
    for _ in range(B):
        path = [0]
        for _ in range(int(torch.randint(0, K + 1, (), generator=g))):
            ch = [c for c in range(N) if plan["parent"][c] == path[-1]]
            if not ch:
                break
            path.append(ch[int(torch.randint(0, len(ch), (), generator=g))])
        A.append(len(path) - 1)
        nodes.append(path + [-1] * (K + 1 - len(path)))
    return (torch.tensor(A, dtype=torch.int32, device=DEV),
            torch.tensor(nodes, dtype=torch.int32, device=DEV))


@pytest.mark.parametrize("nl,B,tree,Hq,Hkv,Ls,dtype", [
    (4, 3, (5, 10, 64), 8, 2, [300, 1000, 77], torch.bfloat16),
    (3, 2, (5, 3, 256), 4, 4, [513, 129], torch.bfloat16),
    (2, 2, (4, 3, 16), 4, 4, [128, 40], torch.float32),
])
def test_layers_attention_and_compaction_match_oracle(nl, B, tree, Hq, Hkv, Ls, dtype):
    K, s, N = tree
    dh = 128 if dtype == torch.bfloat16 else 64
    Lcap = max(Ls) + N + 9
    g = torch.Generator(device=DEV).manual_seed(nl * 100 + N)
    q = torch.randn(nl, B, N, Hq, dh, generator=g, device=DEV).to(dtype)
    kc = torch.randn(nl, B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    vc = torch.randn(nl, B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    Lt = torch.tensor(Ls, dtype=torch.int32, device=DEV)
    t = api.Tree(K, s, N)
    plan = O.tree_plan(K, s, N)
    scale = 1.0 / math.sqrt(dh)
    outs = torch.stack([api.medusa_tree_attention(q[l], kc[l], vc[l], Lt, t, scale)
                        for l in range(nl)])
    torch.cuda.synchronize()
    ref = O.tree_attention_layers(q, kc, vc, Lt, plan, scale)
    for l in range(nl):
        assert_attention_close(outs[l].double().cpu().numpy(), ref[l],
                               bf16=dtype == torch.bfloat16, what=f"layer {l}")

    A, nodes = _paths(plan, B, K, seed=nl + N)
    rk, rv, rl = O.kv_compact_layers(kc, vc, Lt, A, nodes)
    new_len = api.medusa_kv_compact_layers(kc, vc, Lt, A, nodes, K)
    torch.cuda.synchronize()
    assert (new_len.cpu().numpy() == rl).all()
    assert np.array_equal(kc.double().cpu().numpy(), rk)
    assert np.array_equal(vc.double().cpu().numpy(), rv)
    assert api.device_status() == 0


def test_layers_compaction_with_padded_stride_and_one_layer():
    """Layers 1.5 caches apart (padding between them untouched), and one
    layer, which must equal medusa_kv_compact."""
    nl, B, Lcap, Hkv, dh, K = 3, 2, 90, 2, 128, 5
    plan = O.tree_plan(K, 3, 31)
    per = B * Lcap * Hkv * dh
    stride = per + per // 2
    g = torch.Generator(device=DEV).manual_seed(3)
    buf_k = torch.randn(nl * stride, generator=g, device=DEV).bfloat16()
    buf_v = torch.randn(nl * stride, generator=g, device=DEV).bfloat16()
    before_k, before_v = buf_k.clone(), buf_v.clone()
    Lt = torch.tensor([20, 50], dtype=torch.int32, device=DEV)
    A, nodes = _paths(plan, B, K, seed=9)
    new_len = torch.empty(B, dtype=torch.int32, device=DEV)
    rc = L.lib().medusa_kv_compact_layers(
        C.c_void_p(buf_k.data_ptr()), C.c_void_p(buf_v.data_ptr()), nl, stride,
        C.c_void_p(Lt.data_ptr()), C.c_void_p(A.data_ptr()), C.c_void_p(nodes.data_ptr()), B,
        Hkv, dh, Lcap, K, L.BF16, C.c_void_p(new_len.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    L.check(rc, "medusa_kv_compact_layers")
    torch.cuda.synchronize()
    for l in range(nl):
        lk = before_k[l * stride:l * stride + per].view(1, B, Lcap, Hkv, dh)
        lv = before_v[l * stride:l * stride + per].view(1, B, Lcap, Hkv, dh)
        rk, rv, rl = O.kv_compact_layers(lk, lv, Lt, A, nodes)
        assert np.array_equal(buf_k[l * stride:l * stride + per].view(B, Lcap, Hkv, dh)
                              .double().cpu().numpy(), rk[0])
        assert np.array_equal(buf_v[l * stride:l * stride + per].view(B, Lcap, Hkv, dh)
                              .double().cpu().numpy(), rv[0])
        assert torch.equal(buf_k[l * stride + per:(l + 1) * stride],
                           before_k[l * stride + per:(l + 1) * stride])
    assert (new_len.cpu().numpy() == rl).all()
    # one layer == medusa_kv_compact
    k1, v1 = before_k[:per].view(B, Lcap, Hkv, dh).clone(), before_v[:per].view(B, Lcap, Hkv, dh).clone()
    k2, v2 = k1.clone(), v1.clone()
    api.medusa_kv_compact_layers(k1[None], v1[None], Lt, A, nodes, K)
    api.medusa_kv_compact(k2, v2, Lt, A, nodes, K)
    torch.cuda.synchronize()
    assert torch.equal(k1, k2) and torch.equal(v1, v2)


def test_layers_compaction_rejects_overlapping_layers():
    B, Lcap, Hkv, dh, K = 1, 40, 1, 128, 3
    k = torch.zeros(2, B, Lcap, Hkv, dh, dtype=torch.bfloat16, device=DEV)
    z = torch.zeros(B, dtype=torch.int32, device=DEV)
    nodes = torch.zeros(B, K + 1, dtype=torch.int32, device=DEV)
    rc = L.lib().medusa_kv_compact_layers(C.c_void_p(k.data_ptr()), C.c_void_p(k.data_ptr()), 2,
                                          B * Lcap * Hkv * dh - 1, C.c_void_p(z.data_ptr()),
                                          C.c_void_p(z.data_ptr()), C.c_void_p(nodes.data_ptr()),
                                          B, Hkv, dh, Lcap, K, L.BF16, None, None)
    assert rc == L.ERR_INVALID_ARG
