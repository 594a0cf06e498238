"""Medusa heads with the vocabulary split across the ranks of a process group.

Each head's second projection W2 [K][V][d] is cut by vocabulary rows into G
contiguous shards, one per rank.  Every rank runs the whole first projection
(K d x d weights, small next to the K V x d of the second) and the second over
its own rows only, keeps the s best ids of its slice for every (b, k), and a
single all-gather of those candidate lists lets every rank merge them into the
s best of the whole vocabulary (Medusa paper digest, section
"ツリーアテンションによる並列検証": each head contributes its s most likely
tokens).  The s best of a row are among the union of the s best of its
slices, so the merged ids are those of a top-s over the full row, ties to the
lower id included.  The weight bytes each rank streams, which bound the heads
at small batch, drop by G; what crosses the links is B * K * s * 8 bytes per
rank.

Layout of one rank's candidates: an int32 buffer [2][B*K][s], plane 0 the
fp32 values' bits and plane 1 the ids local to the slice.  The heads kernel
writes both planes in place, the all-gather stacks the G buffers into
[G][2][B*K][s] and the merge kernel reads that in place, shifting shard g's
ids by its first vocabulary row.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def vocab_shard(V: int, G: int, r: int, align: int = 128) -> tuple[int, int]:
    """Rows [v0, v1) of the vocabulary that rank r of G holds.  Boundaries
    fall on multiples of `align` (the heads kernel's vocabulary tile) so the
    shards tile evenly; the last shard ends at V."""
    if G < 1 or not 0 <= r < G or V < 1 or align < 1:
        raise ValueError(f"bad shard request V={V} G={G} r={r} align={align}")
    units = -(-V // align)

    def bound(g):
        return min(V, (g * units // G) * align)

    return bound(r), bound(r + 1)


def shard_offsets(V: int, G: int, align: int = 128) -> list[int]:
    """First vocabulary row of every shard."""
    return [vocab_shard(V, G, g, align)[0] for g in range(G)]


def shard_w2(W2: torch.Tensor, G: int, r: int, align: int = 128) -> torch.Tensor:
    """Rank r's rows of W2 [K][V][d], as a contiguous [K][v1 - v0][d] tensor."""
    v0, v1 = vocab_shard(W2.shape[1], G, r, align)
    return W2[:, v0:v1].contiguous()


def gather_candidates(local: torch.Tensor, group=None, out: torch.Tensor | None = None):
    """All-gather every rank's candidate buffer local [2][R][s] int32 into
    [G][2][R][s] (rank order).  One collective per call."""
    G = dist.get_world_size(group)
    if local.dtype != torch.int32 or local.dim() != 3 or local.shape[0] != 2:
        raise ValueError("local must be an int32 [2][R][s] buffer")
    if not local.is_contiguous():
        raise ValueError("local must be contiguous")
    if out is None:
        out = torch.empty((G,) + tuple(local.shape), dtype=torch.int32, device=local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, local, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), local, group=group)
    return out


class ShardedHeads:
    """Per-rank state of the vocabulary-sharded heads for fixed (B, K, s, V):
    the W2 slice, the candidate and gather buffers, the shard offsets on the
    device and the heads workspace, all allocated once.

    `local_fn(h, W1, b1, W2_shard, s, idx, val)` fills this rank's top-s of
    its slice and `merge_fn(gathered, s, v0, out_idx, out_val)` merges the
    gathered planes; both default to the library calls
    (medusa_heads_forward, medusa_topk_merge_planes)."""

    def __init__(self, W1, b1, W2_shard, V: int, B: int, s: int, group=None, align: int = 128,
                 local_fn=None, merge_fn=None):
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.V, self.B, self.s, self.align = V, B, s, align
        self.v0, self.v1 = vocab_shard(V, self.G, self.rank, align)
        K, Vr = W2_shard.shape[0], W2_shard.shape[1]
        if Vr != self.v1 - self.v0:
            raise ValueError(f"W2 shard has {Vr} rows, rank {self.rank} holds {self.v1 - self.v0}")
        if s > Vr:
            raise ValueError(f"s={s} exceeds the {Vr} rows of rank {self.rank}'s shard")
        self.W1, self.b1, self.W2 = W1, b1, W2_shard
        self.K = K
        self.local_fn = local_fn or self._library_local
        self.merge_fn = merge_fn or self._library_merge
        dev = W2_shard.device
        R = B * K
        self.local = torch.empty(2, R, s, dtype=torch.int32, device=dev)
        self.gathered = torch.empty(self.G, 2, R, s, dtype=torch.int32, device=dev)
        self.v0_dev = torch.tensor(shard_offsets(V, self.G, align), dtype=torch.int32, device=dev)
        self.ws = (torch.empty(max(256, api.heads_workspace_size(B, W1.shape[1], Vr, K, s,
                                                                 W1.dtype)),
                               dtype=torch.uint8, device=dev) if local_fn is None else None)
        self.out = (torch.empty(B, K, s, dtype=torch.int32, device=dev),
                    torch.empty(B, K, s, dtype=torch.float32, device=dev))

    def _library_local(self, h, W1, b1, W2, s, idx, val):
        api.medusa_heads_forward(h, W1, b1, W2, s=s, want_logits=False, out=(None, idx, val),
                                 ws=self.ws)

    @staticmethod
    def _library_merge(gathered, s, v0, out_idx, out_val):
        api.medusa_topk_merge_planes(gathered, s, v0, out=(out_idx, out_val))

    def local_topk(self, h):
        """This rank's s best ids (local to its slice) and values per (b, k),
        written into the candidate buffer's two planes."""
        B, K, s = self.B, self.K, self.s
        val = self.local[0].view(torch.float32).view(B, K, s)
        idx = self.local[1].view(B, K, s)
        self.local_fn(h, self.W1, self.b1, self.W2, s, idx, val)
        return self.local

    def __call__(self, h, out=None):
        """topk_idx [B][K][s] int32 (ids of the whole vocabulary) and
        topk_val [B][K][s] fp32, the same on every rank (into `out` when
        given)."""
        self.local_topk(h)
        gather_candidates(self.local, self.group, out=self.gathered)
        R = self.B * self.K
        oi, ov = self.out if out is None else out
        self.merge_fn(self.gathered, self.s, self.v0_dev, oi.view(R, self.s), ov.view(R, self.s))
        return oi, ov
