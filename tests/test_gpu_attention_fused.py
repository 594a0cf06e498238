"""GPU: tree attention whose keys are split into 2 to 8 chunks merged inside
the kernel (the chunks of a query tile run as one thread-block cluster and
merge through distributed shared memory), against the fp64 oracle on every
output row (max-abs 2e-2): MHA and GQA, one and several query tiles, ragged
prefixes, chunks that see no key (a short or empty prefix next to a long
cache), and the launch count the library reports."""
import math

import numpy as np
import pytest
import torch

from attn_check import assert_attention_close
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,tree,Hq,Hkv,Ls", [
    (1, (5, 10, 64), 2, 2, [700]),             # 2 chunks
    (3, (3, 2, 7), 4, 1, [600, 0, 1200]),      # GQA, an empty prefix
    (1, (5, 10, 64), 4, 4, [2048]),            # 7B-like rows, 5 chunks
    (2, (5, 10, 64), 8, 2, [50, 3000]),        # 2 query tiles, keyless chunks
    (1, (4, 4, 32), 2, 2, [4000]),             # 8 chunks
    (2, (5, 8, 128), 8, 2, [1000, 777]),       # 4 query tiles
])
def test_fused_chunk_merge_matches_oracle(B, tree, Hq, Hkv, Ls):
    K, s, N = tree
    dh = 128
    Lcap = max(Ls) + N + 3
    g = torch.Generator(device=DEV).manual_seed(B * 1000 + Lcap)
    q = torch.randn(B, N, Hq, dh, generator=g, device=DEV).bfloat16()
    kc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).bfloat16()
    vc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).bfloat16()
    L = torch.tensor(Ls, dtype=torch.int32, device=DEV)
    t = api.Tree(K, s, N)
    P = api.attention_chunks(t, B, Hq, Hkv, dh, Lcap, torch.bfloat16)
    assert 2 <= P <= 8
    assert api.attention_launches(t, B, Hq, Hkv, dh, Lcap, torch.bfloat16) == 1
    scale = 1.0 / math.sqrt(dh)
    out = api.medusa_tree_attention(q, kc, vc, L, t, scale)
    torch.cuda.synchronize()
    ref = O.tree_attention(q, kc, vc, L, O.tree_plan(K, s, N), scale)
    assert_attention_close(out.double().cpu().numpy(), ref, what=f"B={B} Hq={Hq} L={Ls} P={P}")
    assert api.device_status() == 0


def test_fused_merge_is_repeatable_and_leaves_no_state():
    """Two calls on the same inputs give the same bits (nothing carried over
    between calls), and a call on other inputs in between changes nothing."""
    B, (K, s, N), Hq, Hkv, dh = 2, (5, 10, 64), 8, 2, 128
    Lcap = 3000 + N
    g = torch.Generator(device=DEV).manual_seed(9)
    mk = lambda *shape: torch.randn(*shape, generator=g, device=DEV).bfloat16()
    q, kc, vc = mk(B, N, Hq, dh), mk(B, Lcap, Hkv, dh), mk(B, Lcap, Hkv, dh)
    q2, kc2, vc2 = mk(B, N, Hq, dh), mk(B, Lcap, Hkv, dh), mk(B, Lcap, Hkv, dh)
    L = torch.tensor([2900, 123], dtype=torch.int32, device=DEV)
    t = api.Tree(K, s, N)
    a = api.medusa_tree_attention(q, kc, vc, L, t, 0.1).clone()
    api.medusa_tree_attention(q2, kc2, vc2, L, t, 0.1)
    b = api.medusa_tree_attention(q, kc, vc, L, t, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ---------------------------------------------------------------- two query tiles per CTA
@pytest.mark.parametrize("B,tree,Hq,Hkv,Ls,chunks", [
    # GQA 4: 4 query tiles per (sequence, kv-head), 512 single-tile CTAs
    (16, (5, 8, 128), 32, 8, [50, 400, 120, 333, 7, 260, 199, 380, 0, 64, 128, 129, 255, 256,
                              300, 1], 1),
    # GQA 16: 5 tiles, the last pair has one
    (9, (4, 4, 40), 160, 10, [200, 0, 90, 17, 300, 128, 256, 5, 77], 1),
    # 256 tree nodes, 52 heads (2 tiles): keys split in 2 chunks, merged in-cluster
    (4, (5, 3, 256), 52, 52, [2000, 1500, 700, 1999], 2),
])
def test_two_tiles_per_cta_match_oracle(B, tree, Hq, Hkv, Ls, chunks):
    K, s, N = tree
    dh = 128
    Lcap = max(Ls) + N + 5
    g = torch.Generator(device=DEV).manual_seed(B * 7 + N)
    q = torch.randn(B, N, Hq, dh, generator=g, device=DEV).bfloat16()
    kc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).bfloat16()
    vc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).bfloat16()
    L = torch.tensor(Ls, dtype=torch.int32, device=DEV)
    t = api.Tree(K, s, N)
    assert api.attention_tiles_per_cta(t, B, Hq, Hkv, dh, Lcap, torch.bfloat16) == 2
    assert api.attention_chunks(t, B, Hq, Hkv, dh, Lcap, torch.bfloat16) == chunks
    assert api.attention_launches(t, B, Hq, Hkv, dh, Lcap, torch.bfloat16) == 1
    scale = 1.0 / math.sqrt(dh)
    out = api.medusa_tree_attention(q, kc, vc, L, t, scale)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    rng = np.random.default_rng(B + N)
    rows = [(int(rng.integers(B)), int(rng.integers(N)), int(rng.integers(Hq))) for _ in range(160)]
    # every node of the last rows of each tile pair, on one head of each sequence
    rows += [(b, i, (b * 7) % Hq) for b in range(B) for i in (0, N // 2 - 1, N // 2, N - 1)]
    ref = O.tree_attention(q, kc, vc, L, O.tree_plan(K, s, N), scale, rows=rows)
    got = np.stack([out[b, i, h].double().cpu().numpy() for b, i, h in rows])
    assert_attention_close(got, ref, what=f"B={B} Hq={Hq} Hkv={Hkv} N={N}")
    assert np.isfinite(out.float().cpu().numpy()).all()


def test_plan_queries_reject_bad_shapes():
    t = api.Tree(5, 10, 64)
    for fn in (api.attention_chunks, api.attention_launches, api.attention_tiles_per_cta):
        with pytest.raises(RuntimeError):
            fn(t, 1, 6, 4, 128, 4096, torch.bfloat16)    # Hq not a multiple of Hkv
        with pytest.raises(RuntimeError):
            fn(t, -1, 4, 4, 128, 4096, torch.bfloat16)   # negative batch
        with pytest.raises(RuntimeError):
            fn(t, 1, 4, 4, 128, 32, torch.bfloat16)      # cache shorter than the tree
    # no sequences: no launch
    assert api.attention_launches(t, 0, 4, 4, 128, 4096, torch.bfloat16) == 0
    # the tiny fp32 shape runs on the SIMT kernel and its combine kernel, one tile per CTA
    assert api.attention_launches(t, 1, 4, 4, 64, 4096, torch.float32) == 2
    assert api.attention_tiles_per_cta(t, 1, 4, 4, 64, 4096, torch.float32) == 1
