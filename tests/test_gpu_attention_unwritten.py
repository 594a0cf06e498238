"""GPU: cache slots a sequence has not written do not reach the attention
output.

A sequence b attends to its prefix slots 0..L_b-1 and its tree slots
L_b..L_b+N-1 only ([MD] "ツリーアテンションによる並列検証": Mask_ij = 1 only for
ancestors).  The kernels stage whole 128-key tiles, so the tree tiles and
the prefix tile that ends the sequence also bring in slots >= L_b + N: the
caller's unused cache capacity, or the next sequence's slots.  Those must
carry exactly zero weight, and a NaN or Inf stored there must not reach the
output through 0 * NaN in the P.V product.

Every slot >= L_b + N of K and V is filled with NaN, +3e38 or -3e38 (bf16:
-3e38 and 3e38 are finite, their products overflow).  The output must be
bit-identical to the same call with those slots zeroed, and match the fp64
oracle (which reads only the visible slots).  Covered launch shapes: one
query tile per CTA with one key chunk, key chunks merged in-cluster, key
chunks merged by the combine kernel, two query tiles per CTA with one and
with two chunks, and the fp32 / dh = 64 SIMT kernel.
"""
import math

import pytest
import torch

from attn_check import assert_attention_close
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (B, tree (K, s, N), Hq, Hkv, dh, prefix lengths, spare slots past the longest, dtype,
#  expected (query tiles per CTA, key chunks, launches))
CASES = [
    (2, (5, 10, 64), 4, 4, 128, [300, 129], 200, torch.bfloat16, (1, 1, 1)),
    (1, (5, 10, 64), 2, 2, 128, [700], 300, torch.bfloat16, (1, 2, 1)),
    (1, (5, 10, 64), 100, 100, 128, [1000], 100, torch.bfloat16, (1, 3, 2)),
    (16, (5, 8, 128), 32, 8, 128, [50, 400, 120, 333, 7, 260, 199, 380, 0, 64, 128, 129, 255,
                                   256, 300, 1], 150, torch.bfloat16, (2, 1, 1)),
    (4, (5, 3, 256), 52, 52, 128, [2000, 1500, 700, 1999], 300, torch.bfloat16, (2, 2, 1)),
    (2, (4, 3, 16), 4, 4, 64, [128, 45], 70, torch.float32, None),
]
POISON = [math.nan, 3e38, -3e38]


def _case(B, tree, Hq, Hkv, dh, Ls, spare, dtype):
    K, s, N = tree
    Lcap = max(Ls) + N + spare
    g = torch.Generator(device=DEV).manual_seed(B * 31 + N + Hq)
    q = torch.randn(B, N, Hq, dh, generator=g, device=DEV).to(dtype)
    kc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    vc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).to(dtype)
    L = torch.tensor(Ls, dtype=torch.int32, device=DEV)
    return K, s, N, Lcap, q, kc, vc, L


def _fill_unwritten(c, Ls, N, value):
    c = c.clone()
    for b, Lb in enumerate(Ls):
        c[b, Lb + N:] = value
    return c


@pytest.mark.parametrize("B,tree,Hq,Hkv,dh,Ls,spare,dtype,shape", CASES)
def test_unwritten_slots_do_not_reach_the_output(B, tree, Hq, Hkv, dh, Ls, spare, dtype, shape):
    K, s, N, Lcap, q, kc, vc, L = _case(B, tree, Hq, Hkv, dh, Ls, spare, dtype)
    t = api.Tree(K, s, N)
    if shape is not None:
        assert api.attention_tiles_per_cta(t, B, Hq, Hkv, dh, Lcap, dtype) == shape[0]
        assert api.attention_chunks(t, B, Hq, Hkv, dh, Lcap, dtype) == shape[1]
        assert api.attention_launches(t, B, Hq, Hkv, dh, Lcap, dtype) == shape[2]
    scale = 1.0 / math.sqrt(dh)
    clean = api.medusa_tree_attention(q, _fill_unwritten(kc, Ls, N, 0.0),
                                      _fill_unwritten(vc, Ls, N, 0.0), L, t, scale).clone()
    ref = O.tree_attention(q, kc, vc, L, O.tree_plan(K, s, N), scale)
    assert_attention_close(clean.double().cpu().numpy(), ref, bf16=dtype == torch.bfloat16,
                           what="zeroed unwritten slots")
    for value in POISON:
        out = api.medusa_tree_attention(q, _fill_unwritten(kc, Ls, N, value),
                                        _fill_unwritten(vc, Ls, N, value), L, t, scale)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), value
        assert torch.equal(out, clean), (value, (out.float() - clean.float()).abs().max().item())
    # random finite values there give the same bits too (their weight is exactly 0)
    out = api.medusa_tree_attention(q, kc, vc, L, t, scale)
    torch.cuda.synchronize()
    assert torch.equal(out, clean)
    assert api.device_status() == 0
