"""Host side of the vocabulary-sharded heads on CPU: the shard ranges, and two
gloo ranks that all-gather their candidate buffers ([values; ids] planes)
whose merge, with each shard's ids shifted by its first row, must give the
top-s of the whole row (merged here by the oracle; the merge kernel itself is
checked against the oracle on the GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from medusa_head_speculative_02_b200.sharded import gather_candidates, shard_offsets, vocab_shard


@pytest.mark.parametrize("V", [1, 127, 128, 129, 1000, 32000, 128256, 152064])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
def test_vocab_shards_tile_the_vocabulary(V, G):
    ranges = [vocab_shard(V, G, r) for r in range(G)]
    assert ranges[0][0] == 0 and ranges[-1][1] == V
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0                      # contiguous, disjoint
    for v0, v1 in ranges:
        assert v0 <= v1
        assert v0 % 128 == 0                 # every shard starts on a tile
    sizes = [v1 - v0 for v0, v1 in ranges]
    # whole tiles spread as evenly as they go; only the last shard is ragged
    assert max(sizes[:-1] or [0]) - min(sizes[:-1] or [0]) <= 128
    assert shard_offsets(V, G) == [r[0] for r in ranges]


@pytest.mark.parametrize("V,G,r", [(0, 1, 0), (10, 0, 0), (10, 2, 2), (10, 2, -1)])
def test_vocab_shard_rejects_bad_requests(V, G, r):
    with pytest.raises(ValueError):
        vocab_shard(V, G, r)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


R, V, S = 6, 1000, 5


def _logits():
    # coarse values so that ties straddle shard boundaries
    g = np.random.default_rng(7)
    return np.round(g.standard_normal((R, V)) * 4) / 4


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import medusa_oracle as O
        x = _logits()
        v0, v1 = vocab_shard(V, world, rank)
        li = O.topk(x[:, v0:v1], S)                       # ids local to the slice
        lv = np.take_along_axis(x[:, v0:v1], li, 1).astype(np.float32)
        local = torch.empty(2, R, S, dtype=torch.int32)
        local[0] = torch.from_numpy(lv).view(torch.int32)
        local[1] = torch.from_numpy(li.astype(np.int32))
        out = gather_candidates(local)
        q.put((rank, out.numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_gather_and_merge_give_the_global_topk():
    from oracle import medusa_oracle as O
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    np.testing.assert_array_equal(got[0], got[1])        # every rank holds the same lists
    cand = got[0]
    assert cand.shape == (world, 2, R, S)
    vals = cand[:, 0].view(np.float32)
    off = np.array(shard_offsets(V, world), dtype=np.int64)[:, None, None]
    idxs = cand[:, 1].astype(np.int64) + off
    mi, mv = O.topk_merge(vals, idxs, S)
    x = _logits()
    ref = O.topk(x, S)
    np.testing.assert_array_equal(mi, ref)
    np.testing.assert_array_equal(mv, np.take_along_axis(x, ref, 1))


B2, D2, V2, K2, S2 = 3, 16, 300, 2, 4


def _head_weights():
    g = torch.Generator().manual_seed(11)
    h = torch.randn(B2, D2, generator=g)
    W1 = torch.randn(K2, D2, D2, generator=g) * 0.2
    b1 = torch.randn(K2, D2, generator=g) * 0.2
    W2 = torch.randn(K2, V2, D2, generator=g) * 0.2
    return h, W1, b1, W2


def _call_worker(rank, world, port, q):
    """One rank of ShardedHeads.__call__ with the oracle standing in for the
    two kernels (this rank's top-s of its W2 rows; the merge of the gathered
    planes): the orchestration (shard bounds, planes, all-gather, offsets)
    runs as in production."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import medusa_oracle as O
        from medusa_head_speculative_02_b200.sharded import ShardedHeads, shard_w2

        def local_fn(h, W1, b1, W2s, s, idx, val):
            lg = O.heads_forward(h, W1, b1, W2s)                     # [B][K][Vr]
            ids = O.topk(lg, s)
            idx.copy_(torch.from_numpy(ids.astype(np.int32)))
            val.copy_(torch.from_numpy(np.take_along_axis(lg, ids, 2).astype(np.float32)))

        def merge_fn(gathered, s, v0, out_idx, out_val):
            g = gathered.numpy()
            vals = g[:, 0].view(np.float32)
            ids = g[:, 1].astype(np.int64) + v0.numpy().astype(np.int64)[:, None, None]
            mi, mv = O.topk_merge(vals, ids, s)
            out_idx.copy_(torch.from_numpy(mi.astype(np.int32)))
            out_val.copy_(torch.from_numpy(mv.astype(np.float32)))

        h, W1, b1, W2 = _head_weights()
        sh = ShardedHeads(W1, b1, shard_w2(W2, world, rank), V2, B2, S2, local_fn=local_fn,
                          merge_fn=merge_fn)
        oi, ov = sh(h)
        q.put((rank, oi.numpy().copy(), ov.numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_heads_call_gives_the_global_topk():
    from oracle import medusa_oracle as O
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_call_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {r: (i, v) for r, i, v in (q.get(timeout=120) for _ in range(world))}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    np.testing.assert_array_equal(got[0][0], got[1][0])
    h, W1, b1, W2 = _head_weights()
    lg = O.heads_forward(h, W1, b1, W2)
    ref = O.topk(lg, S2)
    np.testing.assert_array_equal(got[0][0], ref)
    np.testing.assert_allclose(got[0][1], np.take_along_axis(lg, ref, 2), rtol=1e-6)
