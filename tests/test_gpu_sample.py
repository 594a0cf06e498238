"""Sampled next token on the GPU against the oracle (same inputs, same seed
and offset): the token must be identical except where the oracle's top two
fp32 scores are closer than the rounding of the Gumbel noise (counted; such
draws are too close to call between two log implementations)."""
import numpy as np
import pytest
import torch

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import api

pytestmark = pytest.mark.gpu

NEAR = 1e-5   # |z_1 - z_2| below this (z ~ 10) is a don't-care draw


def _inputs(B, N, V, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    vlog = (torch.randn(B, N, V, generator=g) * 2.0).to(dtype)
    alen = torch.randint(0, K + 1, (B,), generator=g, dtype=torch.int32)
    nodes = torch.full((B, K + 1), -1, dtype=torch.int32)
    for b in range(B):
        path = [0] + sorted(torch.randperm(N - 1, generator=g)[:int(alen[b])].add(1).tolist())
        nodes[b, :len(path)] = torch.tensor(path, dtype=torch.int32)
    return vlog, alen, nodes


def _check(vlog, alen, nodes, T, seed, offset):
    got = api.medusa_sample_next(vlog.cuda(), alen.cuda(), nodes.cuda(), T, seed, offset).cpu()
    ref, gap = O.sample_next(vlog, alen.numpy(), nodes.numpy(), T, seed, offset)
    diff = got.numpy() != ref
    assert not (diff & (gap >= NEAR)).any(), (got, ref, gap)
    return int((diff & (gap < NEAR)).sum())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sample_next_matches_oracle_small(dtype):
    vlog, alen, nodes = _inputs(5, 16, 1000, 4, dtype, 1)
    near = 0
    for T in (0.0, 0.3, 0.7, 1.0, 2.5):
        for off in (0, 1, 17, 123456789):
            near += _check(vlog, alen, nodes, T, seed=42, offset=off)
    assert near == 0


def test_sample_next_matches_oracle_full_vocab():
    """Verify-row shape of the 13B workload: B = 8, N = 64, V = 32000, bf16;
    and a 128K vocabulary row."""
    vlog, alen, nodes = _inputs(8, 64, 32000, 5, torch.bfloat16, 2)
    for off in (0, 9):
        assert _check(vlog, alen, nodes, 0.7, seed=2024, offset=off) == 0
    vlog, alen, nodes = _inputs(2, 8, 128256, 5, torch.bfloat16, 3)
    assert _check(vlog, alen, nodes, 0.7, seed=7, offset=1) == 0


def test_sample_next_draws_fresh_noise_per_offset_and_is_deterministic():
    vlog, alen, nodes = _inputs(4, 16, 2000, 4, torch.bfloat16, 4)
    v, a, n = vlog.cuda(), alen.cuda(), nodes.cuda()
    a1 = api.medusa_sample_next(v, a, n, 1.0, 5, 0)
    a2 = api.medusa_sample_next(v, a, n, 1.0, 5, 0)
    assert torch.equal(a1, a2)
    draws = torch.stack([api.medusa_sample_next(v, a, n, 1.0, 5, off) for off in range(8)])
    assert (draws != draws[0]).any()          # different offsets, different draws


def test_sample_next_invalid_path_gives_minus_one():
    vlog, alen, nodes = _inputs(3, 8, 500, 3, torch.bfloat16, 5)
    alen[1] = 7            # outside [0, K]
    nodes[2, int(alen[2])] = 99   # node outside [0, N)
    got = api.medusa_sample_next(vlog.cuda(), alen.cuda(), nodes.cuda(), 0.5, 1, 1).cpu()
    assert got[1] == -1 and got[2] == -1 and got[0] >= 0


def test_device_offset_adds_to_the_host_offset():
    vlog, alen, nodes = _inputs(4, 16, 3000, 4, torch.bfloat16, 6)
    v, a, n = vlog.cuda(), alen.cuda(), nodes.cuda()
    dev_off = torch.tensor([5], dtype=torch.int64, device="cuda")
    for host in (0, 3):
        want = api.medusa_sample_next(v, a, n, 0.8, 9, host + 5)
        got = api.medusa_sample_next(v, a, n, 0.8, 9, host, offset_dev=dev_off)
        assert torch.equal(got, want)
