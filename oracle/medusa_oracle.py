"""Plain, slow, obviously-correct fp64 CPU oracle of one Medusa verify step.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py``; never by the product.
It shares no code with the CUDA library: no kernels, headers, helpers or
table generators.  Inputs arrive as torch tensors or numpy arrays in their
storage dtype (fp32 or bf16) and are converted exactly to fp64.

Sources (page title, then section):
  [MD] "論文解説: Medusa — 複数デコーディングヘッドによるLLM推論高速化フレームワーク"
       - "Medusa Headのアーキテクチャ": H_i(h) = Linear(SiLU(Linear(h)) + h),
         d->d then d->V; head i predicts the token i steps further ahead.
       - "ツリーアテンションによる並列検証": top-s per head, Cartesian product
         of the candidates pruned into a tree; Mask_ij = 1 iff j is an
         ancestor of i.
       - "候補選択：Typical Acceptance": accept x iff
         p(x) > min(eps, delta * exp(-H(p))), eps = 0.09, delta = 0.6;
         greedy (temperature 0) verification is an argmax comparison.
  [EX] "メドゥーサ デコーディング ヘッド" - "ディープダイブ": the tree is verified
       in one pass and the longest matching prefix is accepted.
  [FR] "Medusa" (glossaire) - "Attention en arbre": each node sees only its
       ancestors; the longest path whose tokens are all valid is accepted.
  [ZH] "Medusa：基于多Token预测的LLM推理加速" - "3.3 贪婪vs采样验证": greedy
       verification takes the argmax; sampling verification draws the token
       from softmax(logits / temperature).
  Workload definition (tree scoring rule prod 0.5^r_i * 0.8^depth, sizes,
  tolerances) comes from the five workload configurations of this project.

Readings taken where the pages leave a step open (each is marked READING
below): ranks are 0-based; N counts the root; ties in the tree score break
by (depth asc, tuple lexicographic asc); the ancestor mask includes the node
itself; kv-head of query head h is h // (Hq/Hkv); temperature divides the
logits before both p and H; strict '>' in the typical test; the deepest
accepted node wins, ties to the lowest node index; next token = argmax of
the last accepted node's row; tree positions are prefix_len + depth; with
one temperature per head, the candidates of depth D are verified at the
temperature of head D; the
sampled next token is drawn from the last accepted node's row by Gumbel-max
with SplitMix64 noise keyed by (seed, call offset, sequence, vocab index);
candidate lists of vocabulary shards merge in the top-s order of the whole
row (value desc, global id asc), so a merge of per-shard top-s lists equals
the top-s of the unsplit row; the layers of a multi-layer verification
share the tree, the prefix lengths and the accepted path.

Parity: every function here is pinned by tests/test_oracle_pins.py against
closed forms, library routines or brute force (see each docstring).
"""
from __future__ import annotations

import itertools
from fractions import Fraction

import numpy as np

__all__ = [
    "f64", "tree_score", "tree_plan", "silu", "heads_forward", "topk_row",
    "topk", "build_tree", "tree_attention", "row_argmax", "accept_greedy",
    "typical_row_stats", "typical_threshold", "accept_typical", "kv_compact",
    "ancestors_or_self", "heads_hidden", "heads_logits", "splitmix64",
    "uniform01", "gumbel32", "sample_next", "temperature_by_depth", "topk_merge",
    "tree_attention_layers", "kv_compact_layers",
]


def f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor (fp32/bf16/int) or array to numpy fp64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _rows(x, idx) -> np.ndarray:
    """fp64 copy of rows ``idx`` of a 2-D torch tensor or array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return f64(x[torch.as_tensor(np.asarray(idx), dtype=torch.long)])
    except ImportError:  # pragma: no cover
        pass
    return f64(np.asarray(x)[np.asarray(idx)])


def _i64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").long().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


# ---------------------------------------------------------------------------
# Tree plan.  [MD] "ツリーアテンションによる並列検証": the s candidates of each
# of the K heads form a Cartesian product of paths that is pruned to a tree.
# Pruning rule: keep the N rank tuples (r_1..r_D), 0 <= D <= K, with the
# largest score prod_i 0.5^{r_i} * 0.8^D.
# ---------------------------------------------------------------------------
def tree_score(t) -> Fraction:
    """Exact score 0.8^D * prod 0.5^{r_i} of a rank tuple (READING: 0-based ranks)."""
    return Fraction(4, 5) ** len(t) * Fraction(1, 2) ** sum(t)


def tree_plan(K: int, s: int, N: int) -> dict:
    """Select the N best rank tuples and lay them out as a tree.

    READINGS: N includes the root (the empty tuple, score 1); ties in score
    break by (depth asc, tuple lexicographic asc); node order is
    (depth asc, tuple lexicographic asc) so node 0 is the root and every
    parent precedes its children.
    Returns parent[N] (-1 for the root), depth[N], rank[N] (last rank, -1
    for the root), rank_path[N][K] (-1 padded), anc_mask[N][ceil(N/32)]
    (bit j of node i set iff j is i or an ancestor of i) and the tuples.
    """
    tuples = [()]
    for D in range(1, K + 1):
        tuples.extend(itertools.product(range(s), repeat=D))
    if not 1 <= N <= len(tuples):
        raise ValueError(f"N={N} outside [1, {len(tuples)}]")
    ranked = sorted(tuples, key=lambda t: (-tree_score(t), len(t), t))
    nodes = sorted(ranked[:N], key=lambda t: (len(t), t))
    index = {t: i for i, t in enumerate(nodes)}
    parent = np.array([-1] + [index[t[:-1]] for t in nodes[1:]], dtype=np.int64)
    depth = np.array([len(t) for t in nodes], dtype=np.int64)
    rank = np.array([t[-1] if t else -1 for t in nodes], dtype=np.int64)
    rank_path = np.full((N, K), -1, dtype=np.int64)
    for i, t in enumerate(nodes):
        rank_path[i, :len(t)] = t
    words = (N + 31) // 32
    anc_mask = np.zeros((N, words), dtype=np.uint32)
    for i, t in enumerate(nodes):
        for D in range(len(t) + 1):          # every prefix of t, t itself included
            j = index[t[:D]]
            anc_mask[i, j // 32] |= np.uint32(1 << (j % 32))
    return dict(K=K, s=s, N=N, parent=parent, depth=depth, rank=rank,
                rank_path=rank_path, anc_mask=anc_mask, tuples=nodes)


def ancestors_or_self(plan: dict, i: int) -> list[int]:
    """Node indices on the root-to-i path, root first (walks the parent array)."""
    path = []
    while i >= 0:
        path.append(int(i))
        i = int(plan["parent"][i])
    return path[::-1]


# ---------------------------------------------------------------------------
# Heads.  [MD] "Medusa Headのアーキテクチャ":
#   logits_k = W2_k (SiLU(W1_k h + b1_k) + h),   SiLU(x) = x * sigma(x).
# READING: b1 present (NULL means zero); W2 has no bias.
# ---------------------------------------------------------------------------
def silu(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return x * (1.0 / (1.0 + np.exp(-x)))


def heads_forward(h, W1, b1, W2, heads=None, vocab=None) -> np.ndarray:
    """fp64 head logits [B][len(heads)][len(vocab)].

    h [B][d]; W1 [K][d][d] (row = output feature); b1 [K][d] or None;
    W2 [K][V][d] (row = vocab entry).  ``heads``/``vocab`` restrict the
    output (used to sample full-size problems); default all.
    """
    hh = f64(h)
    K = W1.shape[0]
    V = W2.shape[1]
    heads = list(range(K)) if heads is None else list(heads)
    vocab = np.arange(V) if vocab is None else np.asarray(vocab)
    out = np.zeros((hh.shape[0], len(heads), len(vocab)))
    for j, k in enumerate(heads):
        out[:, j, :] = heads_logits(heads_hidden(hh, W1, b1, k), W2, k, vocab)
    return out


def heads_hidden(h, W1, b1, k: int, rows=None) -> np.ndarray:
    """u = SiLU(W1_k h + b1_k) + h for head k ([B][d], or [B][len(rows)])."""
    hh = f64(h)
    rows = np.arange(W1.shape[1]) if rows is None else np.asarray(rows)
    a = hh @ _rows(W1[k], rows).T
    if b1 is not None:
        a = a + f64(b1[k])[rows][None, :]
    return silu(a) + hh[:, rows]


def heads_logits(u, W2, k: int, vocab=None) -> np.ndarray:
    """logits = W2_k u for head k ([B][V], or [B][len(vocab)])."""
    vocab = np.arange(W2.shape[1]) if vocab is None else np.asarray(vocab)
    return f64(u) @ _rows(W2[k], vocab).T


# ---------------------------------------------------------------------------
# Top-s.  [MD] "ツリーアテンションによる並列検証": the s best tokens per head.
# Order: value descending, ties to the lower index.
# ---------------------------------------------------------------------------
def topk_row(row, s: int) -> np.ndarray:
    row = f64(row)
    order = np.lexsort((np.arange(row.shape[0]), -row))
    return order[:s].astype(np.int64)


def topk(logits, s: int) -> np.ndarray:
    """Top-s indices along the last axis of ``logits`` (any leading shape)."""
    x = f64(logits)
    lead = x.shape[:-1]
    flat = x.reshape(-1, x.shape[-1])
    out = np.stack([topk_row(r, s) for r in flat]) if flat.shape[0] else \
        np.zeros((0, s), dtype=np.int64)
    return out.reshape(*lead, s)


# ---------------------------------------------------------------------------
# Tree expansion: node with rank tuple (r_1..r_D) carries the token of rank
# r_D of head D (head D predicts D+1 steps ahead; the root carries the token
# just produced by the base model).  READING: tree_pos = prefix_len + depth.
# ---------------------------------------------------------------------------
def topk_merge(vals, idxs, s: int):
    """Top-s of candidate lists: vals, idxs [G][R][c] (index < 0 = empty
    slot); per row r, the s best of all G * c candidates by value descending,
    ties to the lower index.  Returns (idx [R][s], val [R][s]) with -1 / NaN
    where fewer than s candidates exist."""
    v = f64(vals)
    ix = _i64(idxs)
    G, R, c = ix.shape
    out_i = np.full((R, s), -1, dtype=np.int64)
    out_v = np.full((R, s), np.nan)
    for r in range(R):
        cand = [(v[g, r, j], ix[g, r, j]) for g in range(G) for j in range(c) if ix[g, r, j] >= 0]
        cand.sort(key=lambda t: (-t[0], t[1]))
        for j, (val, i) in enumerate(cand[:s]):
            out_i[r, j], out_v[r, j] = i, val
    return out_i, out_v


def build_tree(plan: dict, root_tok, topk_idx, prefix_len):
    root = _i64(root_tok)
    tk = _i64(topk_idx)
    L = _i64(prefix_len)
    B, N = root.shape[0], plan["N"]
    tok = np.zeros((B, N), dtype=np.int64)
    pos = np.zeros((B, N), dtype=np.int64)
    for b in range(B):
        for n in range(N):
            D = int(plan["depth"][n])
            tok[b, n] = root[b] if D == 0 else tk[b, D - 1, plan["rank_path"][n, D - 1]]
            pos[b, n] = L[b] + D
    return tok, pos


# ---------------------------------------------------------------------------
# Tree attention.  [MD] Mask_ij = 1 iff j is an ancestor of i; READING: the
# node itself is visible too (a chain tree then equals causal attention).
# Node i of sequence b attends to prefix slots 0..L_b-1 and tree slots
# L_b + j for every j in ancestors_or_self(i).
# ---------------------------------------------------------------------------
def tree_attention(q, k_cache, v_cache, prefix_len, plan, scale, rows=None):
    """fp64 attention output.

    q [B][N][Hq][dh]; k_cache, v_cache [B][Lcap][Hkv][dh]; tree K/V of node j
    at slot L_b + j.  With ``rows`` = iterable of (b, i, h) only those rows are
    computed and an array [len(rows)][dh] is returned; otherwise [B][N][Hq][dh].
    """
    B, N, Hq, dh = q.shape
    Hkv = k_cache.shape[2]
    G = Hq // Hkv
    L = _i64(prefix_len)

    def one(b, i, h):
        kvh = h // G
        Lb = int(L[b])
        slots = list(range(Lb)) + [Lb + j for j in ancestors_or_self(plan, i)]
        Kb = f64(k_cache[b, slots, kvh, :])
        Vb = f64(v_cache[b, slots, kvh, :])
        qv = f64(q[b, i, h, :])
        sc = scale * (Kb @ qv)
        w = np.exp(sc - sc.max())
        return (w @ Vb) / w.sum()

    if rows is not None:
        return np.stack([one(b, i, h) for (b, i, h) in rows])
    out = np.zeros((B, N, Hq, dh))
    for b in range(B):
        for i in range(N):
            for h in range(Hq):
                out[b, i, h] = one(b, i, h)
    return out


# ---------------------------------------------------------------------------
# Acceptance.
# ---------------------------------------------------------------------------
def row_argmax(row) -> int:
    """argmax with the lowest index on ties (np.argmax returns the first)."""
    return int(np.argmax(f64(row)))


def _pick_path(plan: dict, accepted: np.ndarray, K: int):
    """Deepest accepted node (ties: lowest index) and its root-first path."""
    best = 0
    for n in range(plan["N"]):
        if accepted[n] and plan["depth"][n] > plan["depth"][best]:
            best = n
    path = ancestors_or_self(plan, best)
    nodes = np.full(K + 1, -1, dtype=np.int64)
    nodes[:len(path)] = path
    return best, int(plan["depth"][best]), nodes


def accept_greedy(vlogits, tree_tok, plan: dict):
    """Greedy verification ([MD] Typical Acceptance section, temperature 0).

    Node n != 0 is accepted iff its parent is accepted and the argmax of the
    parent's verify row equals tok[n]; the deepest accepted node wins
    ([EX], [FR]).  Returns accept_len [B], accept_nodes [B][K+1], next_tok [B].
    """
    tok = _i64(tree_tok)
    B, N = tok.shape
    K = plan["K"]
    alen = np.zeros(B, dtype=np.int64)
    anodes = np.full((B, K + 1), -1, dtype=np.int64)
    nxt = np.zeros(B, dtype=np.int64)
    for b in range(B):
        amax = [row_argmax(vlogits[b, n]) for n in range(N)]
        acc = np.zeros(N, dtype=bool)
        acc[0] = True
        for n in range(1, N):
            p = int(plan["parent"][n])
            acc[n] = acc[p] and amax[p] == tok[b, n]
        best, alen[b], anodes[b] = _pick_path(plan, acc, K)
        nxt[b] = amax[best]
    return alen, anodes, nxt


def typical_row_stats(row, temperature: float):
    """p = softmax(row / T) and its entropy H = -sum p ln p (natural log)."""
    z = f64(row) / temperature
    e = np.exp(z - z.max())
    p = e / e.sum()
    nz = p > 0
    H = -np.sum(p[nz] * np.log(p[nz]))
    return p, H


def typical_threshold(H: float, eps: float, delta: float) -> float:
    """[MD] Typical Acceptance: threshold min(eps, delta * exp(-H))."""
    return min(eps, delta * np.exp(-H))


def temperature_by_depth(temperature, K: int) -> list:
    """T[D] for the candidates of depth D = 1..K (index 0 unused).  A scalar
    applies to every depth.  READING of the per-head temperatures ([ZH]
    "4.2 温度调优", one temperature per Medusa head): head D proposes the
    nodes of depth D, and those are verified on their parent's row at T[D]."""
    if np.ndim(temperature) == 0:
        return [float(temperature)] * (K + 1)
    t = [float(x) for x in temperature]
    if len(t) != K:
        raise ValueError("one temperature per head")
    return [t[0]] + t


def accept_typical(vlogits, tree_tok, plan: dict, temperature,
                   eps: float = 0.09, delta: float = 0.6):
    """Typical acceptance ([MD] "候補選択：Typical Acceptance").

    Node n != 0 is accepted iff its parent is accepted and
    p_parent(tok[n]) > min(eps, delta * exp(-H(p_parent))) with p = softmax of
    the parent's verify row at the temperature of n's depth (a scalar, or one
    per head: ``temperature_by_depth``).  Also returns, per (b, n), the
    relative margin |p - thr| / thr of each node's own decision (used by the
    tests to flag decisions too close to call in any finite precision).
    """
    tok = _i64(tree_tok)
    B, N = tok.shape
    K = plan["K"]
    T = temperature_by_depth(temperature, K)
    alen = np.zeros(B, dtype=np.int64)
    anodes = np.full((B, K + 1), -1, dtype=np.int64)
    nxt = np.zeros(B, dtype=np.int64)
    margin = np.full((B, N), np.inf)
    for b in range(B):
        # every child of a row has the same depth: one temperature per row
        stats = [typical_row_stats(vlogits[b, n], T[min(int(plan["depth"][n]) + 1, K)])
                 for n in range(N)]
        acc = np.zeros(N, dtype=bool)
        acc[0] = True
        for n in range(1, N):
            par = int(plan["parent"][n])
            p, H = stats[par]
            thr = typical_threshold(H, eps, delta)
            px = p[tok[b, n]]
            margin[b, n] = abs(px - thr) / thr
            acc[n] = acc[par] and px > thr
        best, alen[b], anodes[b] = _pick_path(plan, acc, K)
        nxt[b] = row_argmax(vlogits[b, best])
    return alen, anodes, nxt, margin


# ---------------------------------------------------------------------------
# KV compaction: the accepted path's K/V move to contiguous slots after the
# root (slot L_b); tree slot of path node j -> slot L_b + j.
# ---------------------------------------------------------------------------
def kv_compact(k_cache, v_cache, prefix_len, accept_len, accept_nodes):
    """Returns (new_k, new_v, new_len) as numpy copies in the input dtype's
    exact fp64 image; slots L_b+1..L_b+a take old slots L_b+accept_nodes[j]."""
    k_old, v_old = f64(k_cache), f64(v_cache)
    k_new, v_new = k_old.copy(), v_old.copy()
    L, A, nodes = _i64(prefix_len), _i64(accept_len), _i64(accept_nodes)
    new_len = np.zeros_like(L)
    for b in range(L.shape[0]):
        for j in range(1, int(A[b]) + 1):
            k_new[b, L[b] + j] = k_old[b, L[b] + nodes[b, j]]
            v_new[b, L[b] + j] = v_old[b, L[b] + nodes[b, j]]
        new_len[b] = L[b] + 1 + A[b]
    return k_new, v_new, new_len


# ---------------------------------------------------------------------------
# Several layers.  [MD] "ツリーアテンションによる並列検証": the whole candidate
# tree is verified in one forward pass of the base model, i.e. every layer
# runs the masked attention over its own cache with the same tree and prefix
# lengths, and after acceptance every layer's cache keeps the accepted path.
# READING: the layers share the tree, the prefix lengths and the accepted
# path; each has its own queries and K/V cache.
# ---------------------------------------------------------------------------
def tree_attention_layers(q, k_caches, v_caches, prefix_len, plan, scale, rows=None):
    """q [layers][B][N][Hq][dh]; k_caches, v_caches [layers][B][Lcap][Hkv][dh].
    Layer l's output is tree_attention over layer l's queries and cache;
    returns [layers][...] (the shape tree_attention gives for ``rows``)."""
    return np.stack([tree_attention(q[l], k_caches[l], v_caches[l], prefix_len, plan, scale,
                                    rows=rows) for l in range(q.shape[0])])


def kv_compact_layers(k_caches, v_caches, prefix_len, accept_len, accept_nodes):
    """The accepted path compacted in every layer's cache ([layers][B][Lcap]
    [Hkv][dh]); returns (new_k, new_v, new_len), new_len being the same for
    every layer."""
    ks, vs, new_len = [], [], None
    for l in range(k_caches.shape[0]):
        k, v, new_len = kv_compact(k_caches[l], v_caches[l], prefix_len, accept_len,
                                   accept_nodes)
        ks.append(k)
        vs.append(v)
    return np.stack(ks), np.stack(vs), new_len


# ---------------------------------------------------------------------------
# Sampled next token.  [ZH] "3.3 贪婪vs采样验证": with temperature 0 the token
# is the argmax, otherwise a draw from softmax(logits / temperature).
# READING (the pages fix no generator): the draw is Gumbel-max, i.e. the
# argmax of logits / T + G_v with G_v = -log(-log(U_v)) i.i.d. standard
# Gumbel, which is distributed exactly as softmax(logits / T) (Gumbel 1954;
# the "Gumbel-max trick"); U_v comes from the counter-based SplitMix64
# generator (Steele, Lea & Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014) at counter index ((offset * B) + b) * V + v,
# as (top 23 bits + 1/2) * 2^-23.
# The decision is taken in fp32, the precision of the kernel.
# ---------------------------------------------------------------------------
_GAMMA = np.uint64(0x9E3779B97F4A7C15)


def splitmix64(seed: int, idx) -> np.ndarray:
    """Output number idx (0-based) of SplitMix64 started at state ``seed``:
    the state after idx + 1 steps is seed + (idx + 1) * gamma (mod 2^64),
    then the published finaliser (xor-shift 30, multiply, xor-shift 27,
    multiply, xor-shift 31)."""
    with np.errstate(over="ignore"):
        x = np.uint64(seed) + (np.asarray(idx, dtype=np.uint64) + np.uint64(1)) * _GAMMA
        z = (x ^ (x >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def uniform01(seed: int, idx) -> np.ndarray:
    """fp32 uniforms in (0, 1): the top 23 bits t of the SplitMix64 output,
    (t + 1/2) * 2^-23.  Every step is exact in fp32 (t + 1/2 < 2^23 needs 24
    significant bits), so u lies in [2^-24, 1 - 2^-24]: never 0 or 1."""
    top = (splitmix64(seed, idx) >> np.uint64(41)).astype(np.float32)
    return ((top + np.float32(0.5)) * np.float32(2.0 ** -23)).astype(np.float32)


def gumbel32(u: np.ndarray) -> np.ndarray:
    """Standard Gumbel noise -log(-log(u)) in fp32."""
    u = np.asarray(u, dtype=np.float32)
    return (-np.log(-np.log(u))).astype(np.float32)


def sample_next(vlogits, accept_len, accept_nodes, temperature: float, seed: int,
                offset: int):
    """Next token of every sequence drawn from the row of its last accepted
    node n_a = accept_nodes[b][accept_len[b]].  temperature == 0: argmax
    (lowest index on ties).  Otherwise argmax_v of z_v = fl(fl(l_v * (1/T)) +
    G_v) in fp32 (ties: lowest index).  Returns (next_tok [B], gap [B]) where
    gap is the fp32 distance between the best and second-best z (inf for the
    argmax), so that a test can tell decisions too close to call."""
    A = _i64(accept_len)
    nodes = _i64(accept_nodes)
    B = A.shape[0]
    V = vlogits.shape[-1]
    nxt = np.zeros(B, dtype=np.int64)
    gap = np.full(B, np.inf)
    inv_t = np.float32(1.0) / np.float32(temperature) if temperature > 0 else None
    for b in range(B):
        n_a = int(nodes[b, int(A[b])])
        row = f64(vlogits[b, n_a]).astype(np.float32)   # exact: fp32 / bf16 inputs
        if inv_t is None:
            nxt[b] = int(np.argmax(row))
            continue
        idx = (np.uint64(offset) * np.uint64(B) + np.uint64(b)) * np.uint64(V) + \
            np.arange(V, dtype=np.uint64)
        z = (row * inv_t).astype(np.float32) + gumbel32(uniform01(seed, idx))
        z = z.astype(np.float32)
        nxt[b] = int(np.argmax(z))
        srt = np.sort(z)
        gap[b] = float(srt[-1]) - float(srt[-2])
    return nxt, gap
