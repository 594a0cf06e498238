"""GPU: Medusa heads at large batch (bf16, B > 32, the compute-bound
kernels) against the fp64 oracle ([MD] "Medusa Headのアーキテクチャ":
logits_k = W2_k (SiLU(W1_k h + b1_k) + h)).

Logits within max-abs 2e-2; top-s ids exact wherever the oracle's gap to
the neighbouring logits exceeds 1e-2; the top-s-only call returns the same
ids and values as the call that also writes logits.  Shapes with ragged
vocabulary tiles, batches that are not multiples of the 128/256-column
chunks, several K-splits of the first GEMM, and the 7B-shaped heads at
B = 256 (sampled rows of the oracle).
"""
import numpy as np
import pytest
import torch

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.synthetic import MedusaConfig, gen_head_inputs

pytestmark = pytest.mark.gpu
ATOL = 2e-2
GAP = 1e-2


def _check_topk(ref_row, got_ids, s):
    order = O.topk_row(ref_row, s + 1)
    vals = ref_row[order]
    for j in range(s):
        left = j == 0 or vals[j - 1] - vals[j] > GAP
        right = vals[j] - vals[j + 1] > GAP
        if left and right:
            assert got_ids[j] == order[j], (j, got_ids[:s], order[:s])


@pytest.mark.parametrize("B,d,V,K,s", [
    (33, 256, 700, 2, 3),       # just past the small-batch limit
    (64, 512, 1000, 3, 4),
    (200, 1024, 4099, 2, 10),   # ragged tiles and chunks
    (256, 512, 2000, 5, 8),
    (300, 768, 1500, 2, 16),    # three 128-sequence chunks in the second GEMM
])
def test_heads_large_batch_match_oracle(B, d, V, K, s):
    cfg = MedusaConfig("big", "bf16", B=B, d=d, V=V, K=K, s=s, N=1, Hq=1, Hkv=1, dh=128,
                       L_lo=1, L_hi=1)
    x = gen_head_inputs(cfg, "cuda", seed=B + d)
    logits, idx, val = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s)
    _, idx2, val2 = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s,
                                             want_logits=False)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(val, val2)
    ref = O.heads_forward(x["h"], x["W1"], x["b1"], x["W2"])
    got = logits.double().cpu().numpy()
    err = np.abs(got - ref).max()
    assert err <= ATOL, err
    gi = idx.cpu().numpy()
    gv = val.double().cpu().numpy()
    for b in range(B):
        for k in range(K):
            _check_topk(ref[b, k], gi[b, k], s)
            # values are the logits of the returned ids
            assert np.abs(gv[b, k] - got[b, k, gi[b, k]]).max() == 0.0
    assert api.device_status() == 0


def test_heads_large_batch_null_bias_and_repeatable():
    cfg = MedusaConfig("big", "bf16", B=128, d=512, V=777, K=2, s=5, N=1, Hq=1, Hkv=1, dh=128,
                       L_lo=1, L_hi=1)
    x = gen_head_inputs(cfg, "cuda", seed=7)
    a = api.medusa_heads_forward(x["h"], x["W1"], None, x["W2"], s=5)
    b = api.medusa_heads_forward(x["h"], x["W1"], None, x["W2"], s=5)
    torch.cuda.synchronize()
    assert all(torch.equal(p, q) for p, q in zip(a, b))
    ref = O.heads_forward(x["h"], x["W1"], None, x["W2"])
    assert np.abs(a[0].double().cpu().numpy() - ref).max() <= ATOL


@pytest.mark.slow
def test_heads_large_batch_7b_shape_sampled():
    """The 7B-shaped heads (d = 4096, V = 32000, K = 5, s = 10) at B = 256:
    whole-vocabulary oracle rows for a few (sequence, head) pairs."""
    cfg = MedusaConfig("7b_b256", "bf16", B=256, d=4096, V=32000, K=5, s=10, N=1, Hq=1, Hkv=1,
                       dh=128, L_lo=1, L_hi=1)
    x = gen_head_inputs(cfg, "cuda", seed=0)
    logits, idx, _ = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=cfg.s)
    torch.cuda.synchronize()
    for b, k in [(0, 0), (127, 2), (128, 3), (255, 4)]:
        u = O.heads_hidden(x["h"][b:b + 1], x["W1"], x["b1"], k)
        ref = O.heads_logits(u, x["W2"][k:k + 1], 0)[0]
        got = logits[b, k].double().cpu().numpy()
        assert np.abs(got - ref).max() <= ATOL, (b, k, np.abs(got - ref).max())
        _check_topk(ref, idx[b, k].cpu().numpy(), cfg.s)
    assert api.device_status() == 0
