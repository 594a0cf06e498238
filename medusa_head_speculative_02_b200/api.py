"""Thin PyTorch binding of the libmedusa C ABI (same names as include/medusa.h).

Argument marshalling only: tensors are checked for device, dtype and
contiguity, outputs and scratch are allocated with torch on the tensors'
device, and the raw pointers plus the current CUDA stream go to the C call.
Every step of the computation runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib as L

_DT = {torch.float32: L.F32, torch.bfloat16: L.BF16}


def _dt(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)") from None


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _stream(dev) -> C.c_void_p:
    return C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ws(nbytes: int, dev) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=dev)


def version() -> str:
    return L.lib().medusa_version().decode()


def device_status(clear: bool = True) -> int:
    st = C.c_int(0)
    L.check(L.lib().medusa_device_status(C.byref(st), int(clear)), "medusa_device_status")
    return st.value


def selftest_wait_timeout(limit_ms: int, device=None) -> None:
    """Launch the library's bounded-wait self-test on the current stream: one
    thread waits for a barrier phase that nothing completes, gives up after
    limit_ms, raises the device status word and returns."""
    L.check(L.lib().medusa_selftest_wait_timeout(int(limit_ms), _stream(device)),
            "medusa_selftest_wait_timeout")


def tree_plan_host(K: int, s: int, N: int):
    """Host-only tree plan: (parent[N], depth[N], rank_path[N][K], anc_mask[N][W]) tensors."""
    W = (N + 31) // 32
    parent = torch.empty(N, dtype=torch.int32)
    depth = torch.empty(N, dtype=torch.int32)
    rank_path = torch.empty(N, K, dtype=torch.int32)
    anc = torch.empty(N, W, dtype=torch.int32)
    L.check(L.lib().medusa_tree_plan_host(K, s, N, _ptr(parent), _ptr(depth), _ptr(rank_path),
                                          _ptr(anc)), "medusa_tree_plan_host")
    return parent, depth, rank_path, anc


class Tree:
    """Owns a medusa_tree_t (plan uploaded to the current CUDA device)."""

    def __init__(self, K: int, s: int, N: int):
        h = C.c_void_p()
        L.check(L.lib().medusa_tree_create(K, s, N, C.byref(h)), "medusa_tree_create")
        self.handle, self.K, self.s, self.N = h, K, s, N

    def info(self):
        K, s, N = C.c_int(), C.c_int(), C.c_int()
        L.check(L.lib().medusa_tree_info(self.handle, C.byref(K), C.byref(s), C.byref(N),
                                         None, None, None, None), "medusa_tree_info")
        n, k = N.value, K.value
        parent = torch.empty(n, dtype=torch.int32)
        depth = torch.empty(n, dtype=torch.int32)
        rank_path = torch.empty(n, k, dtype=torch.int32)
        anc = torch.empty(n, (n + 31) // 32, dtype=torch.int32)
        L.check(L.lib().medusa_tree_info(self.handle, None, None, None, _ptr(parent), _ptr(depth),
                                         _ptr(rank_path), _ptr(anc)), "medusa_tree_info")
        return parent, depth, rank_path, anc

    def close(self):
        if self.handle:
            L.lib().medusa_tree_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def heads_workspace_size(B, d, V, K, s, dtype: torch.dtype) -> int:
    return int(L.lib().medusa_heads_workspace_size(B, d, V, K, s, _DT[dtype]))


def medusa_heads_forward(h, W1, b1, W2, s: int = 0, want_logits: bool = True,
                         want_topk: bool = True, out=None, ws=None):
    """Returns (logits [B][K][V] fp32 or None, topk_idx [B][K][s] int32 or None,
    topk_val [B][K][s] fp32 or None)."""
    B, d = h.shape
    K, V = W2.shape[0], W2.shape[1]
    dt = h.dtype
    _need(h, "h", dt)
    _need(W1, "W1", dt, (K, d, d))
    if b1 is not None:
        _need(b1, "b1", dt, (K, d))
    _need(W2, "W2", dt, (K, V, d))
    dev = h.device
    if out is not None:
        logits, idx, val = out
    else:
        logits = torch.empty(B, K, V, dtype=torch.float32, device=dev) if want_logits else None
        idx = torch.empty(B, K, s, dtype=torch.int32, device=dev) if want_topk else None
        val = torch.empty(B, K, s, dtype=torch.float32, device=dev) if want_topk else None
    need = heads_workspace_size(B, d, V, K, s if want_topk else 1, dt)
    if ws is None or ws.numel() < need:
        ws = _ws(need, dev)
    L.check(L.lib().medusa_heads_forward(_ptr(h), _ptr(W1), _ptr(b1), _ptr(W2), B, d, V, K, _dt(h),
                                         _ptr(logits), s if idx is not None else 0, _ptr(idx),
                                         _ptr(val), _ptr(ws), ws.numel(), _stream(dev)),
            "medusa_heads_forward")
    return logits, idx, val


def medusa_topk(logits, s: int):
    R, V = logits.reshape(-1, logits.shape[-1]).shape
    _need(logits, "logits")
    idx = torch.empty(*logits.shape[:-1], s, dtype=torch.int32, device=logits.device)
    val = torch.empty(*logits.shape[:-1], s, dtype=torch.float32, device=logits.device)
    L.check(L.lib().medusa_topk(_ptr(logits), _dt(logits), R, V, s, _ptr(idx), _ptr(val),
                                _stream(logits.device)), "medusa_topk")
    return idx, val


def _merge(val_ptr, idx_ptr, gs, G, R, c, s, v0, out, dev):
    if v0 is not None:
        _need(v0, "v0", torch.int32, (G,))
    oi, ov = out if out is not None else (
        torch.empty(R, s, dtype=torch.int32, device=dev),
        torch.empty(R, s, dtype=torch.float32, device=dev))
    L.check(L.lib().medusa_topk_merge(val_ptr, idx_ptr, gs, _ptr(v0), G, R, c, s, _ptr(oi),
                                      _ptr(ov), _stream(dev)), "medusa_topk_merge")
    return oi, ov


def medusa_topk_merge(vals, idxs, s: int, v0=None, out=None):
    """Top-s of G candidate lists per row: vals float32 / idxs int32
    [G][R][c] (index < 0 = empty), shard g's indices offset by v0[g]
    (int32 device tensor [G] or None).  Returns (idx [R][s], val [R][s])."""
    G, R, c = idxs.shape
    _need(vals, "vals", torch.float32, (G, R, c))
    _need(idxs, "idxs", torch.int32, (G, R, c))
    return _merge(_ptr(vals), _ptr(idxs), R * c, G, R, c, s, v0, out, idxs.device)


def medusa_topk_merge_planes(cand, s: int, v0=None, out=None):
    """As medusa_topk_merge on one int32 buffer cand [G][2][R][c]: plane 0
    holds the fp32 values' bits, plane 1 the ids (the layout an all-gather
    of each shard's [values; ids] buffer produces), read in place."""
    G, two, R, c = cand.shape
    _need(cand, "cand", torch.int32, (G, 2, R, c))
    base = cand.data_ptr()
    return _merge(base, base + 4 * R * c, 2 * R * c, G, R, c, s, v0, out, cand.device)


def medusa_build_tree(tree: Tree, root_tok, topk_idx, prefix_len, out=None):
    B = root_tok.shape[0]
    _need(root_tok, "root_tok", torch.int32, (B,))
    _need(topk_idx, "topk_idx", torch.int32, (B, tree.K, tree.s))
    _need(prefix_len, "prefix_len", torch.int32, (B,))
    dev = root_tok.device
    tok, pos = out if out is not None else (
        torch.empty(B, tree.N, dtype=torch.int32, device=dev),
        torch.empty(B, tree.N, dtype=torch.int32, device=dev))
    L.check(L.lib().medusa_build_tree(tree.handle, _ptr(root_tok), _ptr(topk_idx), _ptr(prefix_len),
                                      B, _ptr(tok), _ptr(pos), _stream(dev)), "medusa_build_tree")
    return tok, pos


def attention_workspace_size(tree: Tree, B, Hq, Hkv, dh, Lcap) -> int:
    return int(L.lib().medusa_tree_attention_workspace_size(tree.handle, B, Hq, Hkv, dh, Lcap))


def attention_chunks(tree: Tree, B, Hq, Hkv, dh, Lcap, dtype: torch.dtype) -> int:
    n = int(L.lib().medusa_tree_attention_chunks(tree.handle, B, Hq, Hkv, dh, Lcap, _DT[dtype]))
    if n < 1:
        L.check(n, "medusa_tree_attention_chunks")
    return n


def attention_tiles_per_cta(tree: Tree, B, Hq, Hkv, dh, Lcap, dtype: torch.dtype) -> int:
    """128-row query tiles one attention CTA takes (1 or 2)."""
    n = int(L.lib().medusa_tree_attention_tiles_per_cta(tree.handle, B, Hq, Hkv, dh, Lcap,
                                                         _DT[dtype]))
    if n < 1:
        L.check(n, "medusa_tree_attention_tiles_per_cta")
    return n


def attention_launches(tree: Tree, B, Hq, Hkv, dh, Lcap, dtype: torch.dtype) -> int:
    """Kernels one medusa_tree_attention call launches on the current device."""
    n = int(L.lib().medusa_tree_attention_launches(tree.handle, B, Hq, Hkv, dh, Lcap, _DT[dtype]))
    if n < 0:
        L.check(n, "medusa_tree_attention_launches")
    return n


def medusa_tree_attention(q, k_cache, v_cache, prefix_len, tree: Tree, scale: float, out=None,
                          ws=None):
    B, N, Hq, dh = q.shape
    Lcap, Hkv = k_cache.shape[1], k_cache.shape[2]
    dt = q.dtype
    _need(q, "q", dt)
    _need(k_cache, "k_cache", dt, (B, Lcap, Hkv, dh))
    _need(v_cache, "v_cache", dt, (B, Lcap, Hkv, dh))
    _need(prefix_len, "prefix_len", torch.int32, (B,))
    if N != tree.N:
        raise ValueError(f"q has {N} nodes, tree has {tree.N}")
    out = torch.empty_like(q) if out is None else out
    need = attention_workspace_size(tree, B, Hq, Hkv, dh, Lcap)
    if ws is None or ws.numel() < need:
        ws = _ws(need, q.device)
    L.check(L.lib().medusa_tree_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(prefix_len),
                                          tree.handle, B, Hq, Hkv, dh, Lcap, float(scale), _dt(q),
                                          _ptr(out), _ptr(ws), ws.numel(), _stream(q.device)),
            "medusa_tree_attention")
    return out


def accept_workspace_size(tree: Tree, B, V) -> int:
    return int(L.lib().medusa_accept_workspace_size(tree.handle, B, V))


def _accept_outputs(B, K, dev):
    return (torch.empty(B, dtype=torch.int32, device=dev),
            torch.empty(B, K + 1, dtype=torch.int32, device=dev),
            torch.empty(B, dtype=torch.int32, device=dev))


def medusa_accept_greedy(vlogits, tree_tok, tree: Tree, out=None, ws=None):
    B, N, V = vlogits.shape
    _need(vlogits, "vlogits")
    _need(tree_tok, "tree_tok", torch.int32, (B, N))
    alen, anodes, nxt = out if out is not None else _accept_outputs(B, tree.K, vlogits.device)
    need = accept_workspace_size(tree, B, V)
    if ws is None or ws.numel() < need:
        ws = _ws(need, vlogits.device)
    L.check(L.lib().medusa_accept_greedy(_ptr(vlogits), _dt(vlogits), _ptr(tree_tok), tree.handle,
                                         B, V, _ptr(alen), _ptr(anodes), _ptr(nxt), _ptr(ws),
                                         ws.numel(), _stream(vlogits.device)),
            "medusa_accept_greedy")
    return alen, anodes, nxt


def medusa_accept_typical(vlogits, tree_tok, tree: Tree, temperature: float, eps: float = 0.09,
                          delta: float = 0.6, out=None, ws=None):
    B, N, V = vlogits.shape
    _need(vlogits, "vlogits")
    _need(tree_tok, "tree_tok", torch.int32, (B, N))
    alen, anodes, nxt = out if out is not None else _accept_outputs(B, tree.K, vlogits.device)
    need = accept_workspace_size(tree, B, V)
    if ws is None or ws.numel() < need:
        ws = _ws(need, vlogits.device)
    L.check(L.lib().medusa_accept_typical(_ptr(vlogits), _dt(vlogits), _ptr(tree_tok), tree.handle,
                                          B, V, float(temperature), float(eps), float(delta),
                                          _ptr(alen), _ptr(anodes), _ptr(nxt), _ptr(ws),
                                          ws.numel(), _stream(vlogits.device)),
            "medusa_accept_typical")
    return alen, anodes, nxt


def medusa_accept_greedy_typical(vlogits, tree_tok, tree: Tree, temperature: float,
                                 eps: float = 0.09, delta: float = 0.6, out_greedy=None,
                                 out_typical=None, ws=None):
    """Greedy and typical acceptance of the same verify logits from one pass
    over them; returns ((accept_len, accept_nodes, next_tok) greedy,
    (accept_len, accept_nodes, next_tok) typical)."""
    B, N, V = vlogits.shape
    _need(vlogits, "vlogits")
    _need(tree_tok, "tree_tok", torch.int32, (B, N))
    g = out_greedy if out_greedy is not None else _accept_outputs(B, tree.K, vlogits.device)
    t = out_typical if out_typical is not None else _accept_outputs(B, tree.K, vlogits.device)
    need = accept_workspace_size(tree, B, V)
    if ws is None or ws.numel() < need:
        ws = _ws(need, vlogits.device)
    L.check(L.lib().medusa_accept_greedy_typical(
        _ptr(vlogits), _dt(vlogits), _ptr(tree_tok), tree.handle, B, V, float(temperature),
        float(eps), float(delta), _ptr(g[0]), _ptr(g[1]), _ptr(g[2]), _ptr(t[0]), _ptr(t[1]),
        _ptr(t[2]), _ptr(ws), ws.numel(), _stream(vlogits.device)), "medusa_accept_greedy_typical")
    return g, t


def medusa_accept_typical_per_head(vlogits, tree_tok, tree: Tree, temperatures, eps: float = 0.09,
                                   delta: float = 0.6, out=None, ws=None):
    """Typical acceptance with one temperature per head (the candidates of
    depth D are verified at temperatures[D-1])."""
    B, N, V = vlogits.shape
    _need(vlogits, "vlogits")
    _need(tree_tok, "tree_tok", torch.int32, (B, N))
    temps = [float(t) for t in temperatures]
    if len(temps) != tree.K:
        raise ValueError(f"{len(temps)} temperatures for {tree.K} heads")
    arr = (C.c_float * tree.K)(*temps)
    alen, anodes, nxt = out if out is not None else _accept_outputs(B, tree.K, vlogits.device)
    need = accept_workspace_size(tree, B, V)
    if ws is None or ws.numel() < need:
        ws = _ws(need, vlogits.device)
    L.check(L.lib().medusa_accept_typical_per_head(
        _ptr(vlogits), _dt(vlogits), _ptr(tree_tok), tree.handle, B, V, arr, float(eps),
        float(delta), _ptr(alen), _ptr(anodes), _ptr(nxt), _ptr(ws), ws.numel(),
        _stream(vlogits.device)), "medusa_accept_typical_per_head")
    return alen, anodes, nxt


def medusa_sample_next(vlogits, accept_len, accept_nodes, temperature: float, seed: int,
                       offset: int, out=None, offset_dev=None):
    """Next token of every sequence drawn from softmax(row / temperature) of its
    last accepted node's verify row (Gumbel-max over counter-based noise;
    temperature 0 = argmax).  offset_dev: optional one-element int64 device
    tensor added to ``offset`` when the kernel runs."""
    B, N, V = vlogits.shape
    _need(vlogits, "vlogits")
    K = accept_nodes.shape[1] - 1
    _need(accept_len, "accept_len", torch.int32, (B,))
    _need(accept_nodes, "accept_nodes", torch.int32, (B, K + 1))
    out = torch.empty(B, dtype=torch.int32, device=vlogits.device) if out is None else out
    L.check(L.lib().medusa_sample_next(_ptr(vlogits), _dt(vlogits), _ptr(accept_len),
                                       _ptr(accept_nodes), B, N, V, K, float(temperature),
                                       int(seed) & ((1 << 64) - 1), int(offset) & ((1 << 64) - 1),
                                       _ptr(offset_dev), _ptr(out), _stream(vlogits.device)),
            "medusa_sample_next")
    return out


def medusa_kv_compact_layers(k_caches, v_caches, prefix_len, accept_len, accept_nodes, K: int,
                             new_len=None):
    """Compaction of the accepted path in every layer's cache: k_caches,
    v_caches [layers][B][Lcap][Hkv][dh] (contiguous, so the layer stride is
    one layer's cache); returns new_len [B]."""
    nl, B, Lcap, Hkv, dh = k_caches.shape
    _need(k_caches, "k_caches")
    _need(v_caches, "v_caches", k_caches.dtype, k_caches.shape)
    _need(prefix_len, "prefix_len", torch.int32, (B,))
    _need(accept_len, "accept_len", torch.int32, (B,))
    _need(accept_nodes, "accept_nodes", torch.int32, (B, K + 1))
    new_len = torch.empty(B, dtype=torch.int32, device=k_caches.device) if new_len is None \
        else new_len
    L.check(L.lib().medusa_kv_compact_layers(_ptr(k_caches), _ptr(v_caches), nl,
                                             B * Lcap * Hkv * dh, _ptr(prefix_len),
                                             _ptr(accept_len), _ptr(accept_nodes), B, Hkv, dh,
                                             Lcap, K, _dt(k_caches), _ptr(new_len),
                                             _stream(k_caches.device)),
            "medusa_kv_compact_layers")
    return new_len


def medusa_kv_compact(k_cache, v_cache, prefix_len, accept_len, accept_nodes, K: int,
                      new_len=None):
    B, Lcap, Hkv, dh = k_cache.shape
    _need(k_cache, "k_cache")
    _need(v_cache, "v_cache", k_cache.dtype, k_cache.shape)
    _need(prefix_len, "prefix_len", torch.int32, (B,))
    _need(accept_len, "accept_len", torch.int32, (B,))
    _need(accept_nodes, "accept_nodes", torch.int32, (B, K + 1))
    new_len = torch.empty(B, dtype=torch.int32, device=k_cache.device) if new_len is None else new_len
    L.check(L.lib().medusa_kv_compact(_ptr(k_cache), _ptr(v_cache), _ptr(prefix_len),
                                      _ptr(accept_len), _ptr(accept_nodes), B, Hkv, dh, Lcap, K,
                                      _dt(k_cache), _ptr(new_len), _stream(k_cache.device)),
            "medusa_kv_compact")
    return new_len
