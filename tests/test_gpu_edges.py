"""Edge cases against the oracle: a running max that grows tile after tile
(the attention kernel's lazy rescaling after the first tile), -inf logits in
the verify rows, and empty batches."""
import math

import numpy as np
import pytest
import torch

from attn_check import assert_attention_close
from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api
from medusa_head_speculative_02_b200.synthetic import MedusaConfig, plant_verify_logits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("Hq,Hkv,L,spike_tree", [(4, 2, 1500, False), (8, 8, 700, True),
                                                 (16, 2, 3000, False)])
def test_tree_attention_running_max_grows_across_tiles(Hq, Hkv, L, spike_tree):
    """Keys scaled up along the sequence (and, optionally, 6x on the tree
    slots): the tile maxima rise by far more than 2^8 over the row, so the
    reference max moves and O is rescaled after the first tile, repeatedly."""
    B, K, s, N, dh = 2, 4, 3, 16, 128
    Lcap = L + N + 5
    g = torch.Generator(device=DEV).manual_seed(L + Hq)
    q = (3.0 * torch.randn(B, N, Hq, dh, generator=g, device=DEV)).bfloat16()
    ramp = torch.linspace(1.0, 5.0, Lcap, device=DEV).view(1, Lcap, 1, 1)
    kc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV) * ramp
    if spike_tree:
        kc[:, L:L + N] *= 6.0
    kc = kc.bfloat16()
    vc = torch.randn(B, Lcap, Hkv, dh, generator=g, device=DEV).bfloat16()
    Ls = torch.tensor([L, L - 37], dtype=torch.int32, device=DEV)
    t = api.Tree(K, s, N)
    plan = O.tree_plan(K, s, N)
    scale = 1.0 / math.sqrt(dh)
    out = api.medusa_tree_attention(q, kc, vc, Ls, t, scale)
    ref = O.tree_attention(q, kc, vc, Ls, plan, scale)
    assert_attention_close(out.double().cpu().numpy(), ref, what=f"Hq={Hq} L={L}")


def _neg_inf_case(dtype, B, K, s, N, V, seed):
    cfg = MedusaConfig("edge", dtype, B=B, d=8, V=V, K=K, s=s, N=N, Hq=1, Hkv=1, dh=8,
                       L_lo=4, L_hi=4)
    plan = O.tree_plan(K, s, N)
    g = torch.Generator().manual_seed(seed)
    topk = torch.stack([torch.randperm(V, generator=g)[:K * s].view(K, s) for _ in range(B)])
    tok, _ = O.build_tree(plan, torch.zeros(B, dtype=torch.long), topk, [0] * B)
    vlog = plant_verify_logits(cfg, plan["parent"], tok, device="cpu", seed=seed).float()
    # mask 90% of every row to -inf, keeping the tree tokens' entries finite
    mask = torch.rand(B, N, V, generator=g) < 0.9
    keep = torch.zeros(B, N, V, dtype=torch.bool)
    for b in range(B):
        keep[b, :, torch.as_tensor(tok[b], dtype=torch.long)] = True
    vlog[mask & ~keep] = -math.inf
    vlog = vlog.to(cfg.torch_dtype).to(DEV)
    return plan, torch.as_tensor(tok, dtype=torch.int32, device=DEV), vlog


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_accept_with_neg_inf_logits(dtype):
    B, K, s, N, V = 3, 4, 3, 16, 2000
    plan, tok, vlog = _neg_inf_case(dtype, B, K, s, N, V, seed=41)
    t = api.Tree(K, s, N)
    alen, anodes, nxt = api.medusa_accept_greedy(vlog, tok, t)
    ra, rn, rx = O.accept_greedy(vlog, tok, plan)
    assert (alen.cpu().numpy() == ra).all() and (anodes.cpu().numpy() == rn).all()
    assert (nxt.cpu().numpy() == rx).all()
    alen, anodes, nxt = api.medusa_accept_typical(vlog, tok, t, 0.8)
    ra, rn, rx, margin = O.accept_typical(vlog, tok, plan, 0.8)
    for b in range(B):
        if (margin[b, 1:] < 1e-5).any():
            continue
        assert alen[b].item() == ra[b] and anodes[b].tolist() == rn[b].tolist()
        assert nxt[b].item() == rx[b]
    # sampling never draws a -inf entry
    for off in range(5):
        drawn = api.medusa_sample_next(vlog, alen, anodes, 1.0, 3, off).cpu()
        ref, _ = O.sample_next(vlog.cpu(), alen.cpu().numpy(), anodes.cpu().numpy(), 1.0, 3, off)
        for b in range(B):
            row = vlog[b, int(anodes[b, int(alen[b])])].float().cpu()
            assert math.isfinite(row[int(drawn[b])].item())
        assert (drawn.numpy() == ref).all()


def test_empty_batch_is_a_no_op():
    K, s, N, V, H, dh, Lcap = 3, 2, 7, 64, 2, 128, 32
    t = api.Tree(K, s, N)
    z32 = lambda *sh: torch.zeros(*sh, dtype=torch.int32, device=DEV)
    q = torch.zeros(0, N, H, dh, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(0, Lcap, H, dh, dtype=torch.bfloat16, device=DEV)
    out = api.medusa_tree_attention(q, kc, kc.clone(), z32(0), t, 0.1)
    assert out.shape[0] == 0
    tok, pos = api.medusa_build_tree(t, z32(0), z32(0, K, s), z32(0))
    assert tok.shape == (0, N)
    vlog = torch.zeros(0, N, V, dtype=torch.bfloat16, device=DEV)
    a, n, x = api.medusa_accept_greedy(vlog, z32(0, N), t)
    assert a.numel() == 0
    a, n, x = api.medusa_accept_typical(vlog, z32(0, N), t, 0.7)
    assert a.numel() == 0
    assert api.medusa_sample_next(vlog, z32(0), z32(0, K + 1), 0.7, 1, 0).numel() == 0
    assert api.medusa_kv_compact(kc, kc.clone(), z32(0), z32(0), z32(0, K + 1), K).numel() == 0
    torch.cuda.synchronize()
    assert api.device_status(clear=True) == 0
