"""GPU: the merge of per-shard top-s candidate lists (bit-exact against the
oracle merge, dense and [values; ids]-plane layouts, ties, empty slots,
padding), and the vocabulary-sharded heads emulated on one device: G shards
of W2 each through the heads kernel, merged, checked against the oracle's
top-s of the whole vocabulary (ids exact wherever the logit gap to the
neighbouring rank exceeds 1e-2)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.sharded import (ShardedHeads, shard_offsets, shard_w2,
                                                     vocab_shard)
from medusa_head_speculative_02_b200.synthetic import MedusaConfig, gen_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
ATOL = 2e-2
GAP = 1e-2


def _lists(G, R, c, Vr, seed, empty=0.0):
    """Per-shard candidate lists: distinct local ids per (g, r), values on a
    coarse grid (many ties across and within shards), a share of empty slots."""
    g = np.random.default_rng(seed)
    vals = (g.integers(-8, 8, (G, R, c)) * 0.5).astype(np.float32)
    idxs = np.stack([np.stack([g.permutation(Vr)[:c] for _ in range(R)]) for _ in range(G)])
    idxs = idxs.astype(np.int32)
    idxs[g.random((G, R, c)) < empty] = -1
    return vals, idxs


def _check_exact(oi, ov, ri, rv):
    np.testing.assert_array_equal(oi.cpu().numpy(), ri)
    got = ov.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(rv))
    np.testing.assert_array_equal(got[~np.isnan(got)], rv[~np.isnan(rv)])


@pytest.mark.parametrize("G,R,c,s,empty", [(1, 1, 1, 1, 0.0), (2, 7, 10, 10, 0.0),
                                           (4, 40, 10, 10, 0.1), (8, 3, 16, 16, 0.3),
                                           (3, 300, 5, 5, 0.0), (5, 2, 20, 6, 0.5),
                                           (64, 4, 12, 12, 0.0)])
def test_topk_merge_exact(G, R, c, s, empty):
    Vr = 1000
    vals, idxs = _lists(G, R, c, Vr, seed=G * 100 + R, empty=empty)
    v0 = np.arange(G, dtype=np.int32) * Vr
    oi, ov = api.medusa_topk_merge(torch.from_numpy(vals).to(DEV), torch.from_numpy(idxs).to(DEV),
                                   s, torch.from_numpy(v0).to(DEV))
    torch.cuda.synchronize()
    shifted = np.where(idxs >= 0, idxs.astype(np.int64) + v0[:, None, None], -1)
    ri, rv = O.topk_merge(vals, shifted, s)
    _check_exact(oi, ov, ri, rv)


def test_topk_merge_without_offsets_and_padding():
    # fewer valid candidates than s in some rows: -1 / NaN padding
    vals, idxs = _lists(3, 9, 4, 50, seed=3, empty=0.6)
    oi, ov = api.medusa_topk_merge(torch.from_numpy(vals).to(DEV), torch.from_numpy(idxs).to(DEV),
                                   12)
    torch.cuda.synchronize()
    ri, rv = O.topk_merge(vals, idxs, 12)
    assert (ri == -1).any()
    _check_exact(oi, ov, ri, rv)


def test_topk_merge_planes_layout_matches_dense():
    G, R, c, s = 4, 11, 8, 8
    vals, idxs = _lists(G, R, c, 500, seed=11, empty=0.05)
    cand = np.empty((G, 2, R, c), dtype=np.int32)
    cand[:, 0] = vals.view(np.int32)
    cand[:, 1] = idxs
    v0 = np.array([0, 500, 1000, 1500], dtype=np.int32)
    oi, ov = api.medusa_topk_merge_planes(torch.from_numpy(cand).to(DEV), s,
                                          torch.from_numpy(v0).to(DEV))
    torch.cuda.synchronize()
    shifted = np.where(idxs >= 0, idxs.astype(np.int64) + v0[:, None, None], -1)
    ri, rv = O.topk_merge(vals, shifted, s)
    _check_exact(oi, ov, ri, rv)


def test_topk_merge_zero_rows_and_bad_args():
    e = torch.empty(2, 0, 4, dtype=torch.float32, device=DEV)
    ei = torch.empty(2, 0, 4, dtype=torch.int32, device=DEV)
    oi, ov = api.medusa_topk_merge(e, ei, 4)
    assert oi.shape == (0, 4)
    x = torch.zeros(2, 3, 4, dtype=torch.float32, device=DEV)
    xi = torch.zeros(2, 3, 4, dtype=torch.int32, device=DEV)
    with pytest.raises(RuntimeError):
        api.medusa_topk_merge(x, xi, 0)                 # s < 1
    with pytest.raises(RuntimeError):
        api.medusa_topk_merge(x, xi, 10 ** 6)           # s > MEDUSA_MAX_S


def _check_topk(gpu_idx, ref_logits, s):
    for r in range(ref_logits.shape[0]):
        row = ref_logits[r]
        order = O.topk_row(row, s + 1)
        vals = row[order]
        for j in range(s):
            left_ok = j == 0 or vals[j - 1] - vals[j] > GAP
            right_ok = vals[j] - vals[j + 1] > GAP
            if left_ok and right_ok:
                assert gpu_idx[r, j] == order[j], (r, j, gpu_idx[r], order[:s])


@pytest.mark.parametrize("G,B,d,V,K,s", [(2, 1, 512, 4000, 3, 8), (4, 4, 256, 5000, 5, 10),
                                         (8, 2, 1024, 3001, 2, 6), (3, 16, 128, 1000, 4, 4)])
def test_sharded_heads_on_one_device(G, B, d, V, K, s):
    cfg = MedusaConfig(name="sharded", dtype="bf16", B=B, d=d, V=V, K=K, s=s, N=16, Hq=4, Hkv=4,
                       dh=128, L_lo=64, L_hi=64)
    x = gen_inputs(cfg, DEV, seed=G + V)
    R = B * K
    cand = torch.empty(G, 2, R, s, dtype=torch.int32, device=DEV)
    for g in range(G):
        W2g = shard_w2(x["W2"], G, g)
        assert W2g.shape[1] == vocab_shard(V, G, g)[1] - vocab_shard(V, G, g)[0]
        val = cand[g, 0].view(torch.float32).view(B, K, s)
        idx = cand[g, 1].view(B, K, s)
        api.medusa_heads_forward(x["h"], x["W1"], x["b1"], W2g, s=s, want_logits=False,
                                 out=(None, idx, val))
    v0 = torch.tensor(shard_offsets(V, G), dtype=torch.int32, device=DEV)
    oi, ov = api.medusa_topk_merge_planes(cand, s, v0)
    _, full_i, full_v = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=s,
                                                 want_logits=False)
    torch.cuda.synchronize()
    ref = O.heads_forward(x["h"], x["W1"], x["b1"], x["W2"]).reshape(R, V)
    got_i = oi.cpu().numpy()
    assert ((got_i >= 0) & (got_i < V)).all()
    assert all(len(set(row)) == s for row in got_i.tolist())
    _check_topk(got_i, ref, s)
    # values are logits at the returned ids
    np.testing.assert_allclose(ov.cpu().numpy(), np.take_along_axis(ref, got_i, 1), atol=ATOL)
    # and agree with the unsharded kernel's wherever the ids agree
    same = got_i == full_i.view(R, s).cpu().numpy()
    assert same.mean() > 0.9
    np.testing.assert_allclose(ov.cpu().numpy()[same], full_v.view(R, s).cpu().numpy()[same],
                               atol=1e-4)


def test_sharded_heads_class_single_rank_matches_unsharded():
    """One NCCL rank: the class's gather and merge reduce to the unsharded
    top-s, id for id and value for value."""
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        cfg = MedusaConfig(name="sharded1", dtype="bf16", B=2, d=512, V=3000, K=4, s=8, N=16,
                           Hq=4, Hkv=4, dh=128, L_lo=64, L_hi=64)
        x = gen_inputs(cfg, DEV, seed=5)
        sh = ShardedHeads(x["W1"], x["b1"], shard_w2(x["W2"], 1, 0), cfg.V, cfg.B, cfg.s)
        oi, ov = sh(x["h"])
        _, ri, rv = api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=cfg.s,
                                             want_logits=False)
        torch.cuda.synchronize()
        assert torch.equal(oi, ri)
        assert torch.equal(ov, rv)
    finally:
        dist.destroy_process_group()
