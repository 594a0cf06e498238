"""One Medusa verify step through the public API, with preallocated buffers.

A step is: heads (+ fused top-s) -> tree expansion -> tree attention ->
acceptance (greedy, typical or both) -> KV compaction, all on the current
CUDA stream.  ``HostIO`` adds the per-step host<->device traffic of a real
decoder (hidden state, tree queries, tree K/V, verify logits and token ids
in; acceptance results out) for end-to-end timing.
"""
from __future__ import annotations

import math

import torch

from . import api, kernel_bench
from .synthetic import MedusaConfig, gen_inputs, plant_verify_logits

# kernels this library launches per call
# (heads: stage-1 GEMM, SiLU epilogue, stage-2 GEMM, top-s merge; attention:
# one or two, asked of the library, see launches_per_step)
LAUNCHES = {"heads": 4, "build_tree": 1, "accept": 2, "kv_compact": 1}


class VerifyStep:
    def __init__(self, cfg: MedusaConfig, device="cuda", seed: int = 0):
        self.cfg = cfg
        self.dev = torch.device(device)
        self.x = gen_inputs(cfg, self.dev, seed)
        self.tree = api.Tree(cfg.K, cfg.s, cfg.N)
        B, K, s, N = cfg.B, cfg.K, cfg.s, cfg.N
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.topk_idx = torch.empty(B, K, s, **i32)
        self.topk_val = torch.empty(B, K, s, dtype=torch.float32, device=self.dev)
        self.tree_tok = torch.empty(B, N, **i32)
        self.tree_pos = torch.empty(B, N, **i32)
        self.attn_out = torch.empty_like(self.x["q"])
        self.accept_len = torch.empty(B, **i32)
        self.accept_nodes = torch.empty(B, K + 1, **i32)
        self.next_tok = torch.empty(B, **i32)
        self.accept_len2 = torch.empty(B, **i32)
        self.accept_nodes2 = torch.empty(B, K + 1, **i32)
        self.next_tok2 = torch.empty(B, **i32)
        self.new_len = torch.empty(B, **i32)
        self.ws_heads = torch.empty(api.heads_workspace_size(B, cfg.d, cfg.V, K, s, cfg.torch_dtype),
                                    dtype=torch.uint8, device=self.dev)
        self.ws_attn = torch.empty(max(256, api.attention_workspace_size(self.tree, B, cfg.Hq,
                                                                         cfg.Hkv, cfg.dh, cfg.Lcap)),
                                   dtype=torch.uint8, device=self.dev)
        self.ws_acc = torch.empty(max(256, api.accept_workspace_size(self.tree, B, cfg.V)),
                                  dtype=torch.uint8, device=self.dev)
        self.scale = 1.0 / math.sqrt(cfg.dh)
        # verify logits are planted along the tree this step's heads produce
        self.heads()
        self.build_tree()
        torch.cuda.synchronize(self.dev)
        parent = self.tree.info()[0]
        self.vlogits = plant_verify_logits(cfg, parent, self.tree_tok.cpu(), self.dev, seed)

    # individual calls --------------------------------------------------------
    def heads(self):
        x = self.x
        api.medusa_heads_forward(x["h"], x["W1"], x["b1"], x["W2"], s=self.cfg.s,
                                 want_logits=False,
                                 out=(None, self.topk_idx, self.topk_val), ws=self.ws_heads)

    def build_tree(self):
        api.medusa_build_tree(self.tree, self.x["root_tok"], self.topk_idx, self.x["prefix_len"],
                              out=(self.tree_tok, self.tree_pos))

    def attention(self):
        x = self.x
        api.medusa_tree_attention(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], self.tree,
                                  self.scale, out=self.attn_out, ws=self.ws_attn)

    def accept(self):
        cfg = self.cfg
        if cfg.accept == "both":  # one pass over the verify logits serves both rules
            api.medusa_accept_greedy_typical(
                self.vlogits, self.tree_tok, self.tree, cfg.temperature, cfg.eps, cfg.delta,
                out_greedy=(self.accept_len, self.accept_nodes, self.next_tok),
                out_typical=(self.accept_len2, self.accept_nodes2, self.next_tok2), ws=self.ws_acc)
            return
        if cfg.accept in ("greedy", "both"):
            api.medusa_accept_greedy(self.vlogits, self.tree_tok, self.tree,
                                     out=(self.accept_len, self.accept_nodes, self.next_tok),
                                     ws=self.ws_acc)
        if cfg.accept in ("typical", "both"):
            out = (self.accept_len, self.accept_nodes, self.next_tok) if cfg.accept == "typical" \
                else (self.accept_len2, self.accept_nodes2, self.next_tok2)
            api.medusa_accept_typical(self.vlogits, self.tree_tok, self.tree, cfg.temperature,
                                      cfg.eps, cfg.delta, out=out, ws=self.ws_acc)

    def compact(self):
        x = self.x
        api.medusa_kv_compact(x["k_cache"], x["v_cache"], x["prefix_len"], self.accept_len,
                              self.accept_nodes, self.cfg.K, new_len=self.new_len)

    def run(self):
        self.heads()
        self.build_tree()
        self.attention()
        self.accept()
        self.compact()

    def launches_per_step(self) -> int:
        c = self.cfg
        # both rules: one row reduction and two walks
        acc = LAUNCHES["accept"] + 1 if c.accept == "both" else LAUNCHES["accept"]
        attn = api.attention_launches(self.tree, c.B, c.Hq, c.Hkv, c.dh, c.Lcap, c.torch_dtype)
        return (LAUNCHES["heads"] + LAUNCHES["build_tree"] + attn + acc + LAUNCHES["kv_compact"])

    # algorithmic work ---------------------------------------------------------
    def heads_bytes(self) -> int:
        return kernel_bench.heads_bytes(self.cfg)

    def attention_flops(self) -> int:
        """Tensor-core work of the attention call: S = Q K^T and O = P V over
        every key of a sequence's prefix and tree slots, per query row."""
        return kernel_bench.attention_flops(self.cfg, int(self.x["prefix_len"].sum().item()))

    def attention_bytes(self) -> int:
        """K/V actually read (prefix + tree slots) + Q + O."""
        return kernel_bench.attention_bytes(self.cfg, int(self.x["prefix_len"].sum().item()))


class MultiLayerStep:
    """A verify step through `layers` attention layers: heads (+ top-s), tree
    expansion, one tree-attention call per layer on that layer's queries and
    cache (the tree, prefix lengths and workspace shared), acceptance, and
    one compaction of the accepted path over every layer's cache.  The
    per-layer queries and caches are synthetic (no base model): layer l
    draws them from its own seed."""

    def __init__(self, cfg: MedusaConfig, layers: int, device="cuda", seed: int = 0):
        from .synthetic import gen_attention_inputs
        self.st = VerifyStep(cfg, device, seed)
        self.layers = layers
        c = cfg
        dev = self.st.dev
        self.q = torch.empty(layers, c.B, c.N, c.Hq, c.dh, dtype=c.torch_dtype, device=dev)
        self.k = torch.empty(layers, c.B, c.Lcap, c.Hkv, c.dh, dtype=c.torch_dtype, device=dev)
        self.v = torch.empty_like(self.k)
        for l in range(layers):
            xl = gen_attention_inputs(c, dev, seed * 1000 + l)
            self.q[l].copy_(xl["q"])
            self.k[l].copy_(xl["k_cache"])
            self.v[l].copy_(xl["v_cache"])
            del xl
        self.out = torch.empty_like(self.q)

    def attention(self):
        st = self.st
        for l in range(self.layers):
            api.medusa_tree_attention(self.q[l], self.k[l], self.v[l], st.x["prefix_len"],
                                      st.tree, st.scale, out=self.out[l], ws=st.ws_attn)

    def compact(self):
        st = self.st
        api.medusa_kv_compact_layers(self.k, self.v, st.x["prefix_len"], st.accept_len,
                                     st.accept_nodes, st.cfg.K, new_len=st.new_len)

    def run(self):
        self.st.heads()
        self.st.build_tree()
        self.attention()
        self.st.accept()
        self.compact()

    def launches_per_step(self) -> int:
        c = self.st.cfg
        attn = api.attention_launches(self.st.tree, c.B, c.Hq, c.Hkv, c.dh, c.Lcap, c.torch_dtype)
        acc = LAUNCHES["accept"] + 1 if c.accept == "both" else LAUNCHES["accept"]
        return (LAUNCHES["heads"] + LAUNCHES["build_tree"] + self.layers * attn + acc +
                LAUNCHES["kv_compact"])


class HostIO:
    """Pinned host copies of one step's per-step inputs and outputs."""

    def __init__(self, st: VerifyStep):
        self.st = st
        c = st.cfg
        x = st.x
        pin = dict(pin_memory=True)
        self.h = x["h"].cpu().pin_memory()
        self.q = x["q"].cpu().pin_memory()
        self.vlog = st.vlogits.cpu().pin_memory()
        self.root = x["root_tok"].cpu().pin_memory()
        self.plen = x["prefix_len"].cpu().pin_memory()
        self.L = [int(v) for v in self.plen.tolist()]
        self.tree_k = torch.stack([x["k_cache"][b, self.L[b]:self.L[b] + c.N] for b in range(c.B)]).cpu().pin_memory()
        self.tree_v = torch.stack([x["v_cache"][b, self.L[b]:self.L[b] + c.N] for b in range(c.B)]).cpu().pin_memory()
        self.o_alen = torch.empty(c.B, dtype=torch.int32, **pin)
        self.o_nodes = torch.empty(c.B, c.K + 1, dtype=torch.int32, **pin)
        self.o_next = torch.empty(c.B, dtype=torch.int32, **pin)
        self.o_len = torch.empty(c.B, dtype=torch.int32, **pin)
        self.o_topk = torch.empty(c.B, c.K, c.s, dtype=torch.int32, **pin)

    def h2d_bytes(self) -> int:
        ts = [self.h, self.q, self.vlog, self.root, self.plen, self.tree_k, self.tree_v]
        return sum(t.numel() * t.element_size() for t in ts)

    def d2h_bytes(self) -> int:
        ts = [self.o_alen, self.o_nodes, self.o_next, self.o_len, self.o_topk]
        return sum(t.numel() * t.element_size() for t in ts)

    def step(self):
        st, x, c = self.st, self.st.x, self.st.cfg
        x["h"].copy_(self.h, non_blocking=True)
        x["q"].copy_(self.q, non_blocking=True)
        st.vlogits.copy_(self.vlog, non_blocking=True)
        x["root_tok"].copy_(self.root, non_blocking=True)
        x["prefix_len"].copy_(self.plen, non_blocking=True)
        for b in range(c.B):
            x["k_cache"][b, self.L[b]:self.L[b] + c.N].copy_(self.tree_k[b], non_blocking=True)
            x["v_cache"][b, self.L[b]:self.L[b] + c.N].copy_(self.tree_v[b], non_blocking=True)
        st.run()
        self.o_alen.copy_(st.accept_len, non_blocking=True)
        self.o_nodes.copy_(st.accept_nodes, non_blocking=True)
        self.o_next.copy_(st.next_tok, non_blocking=True)
        self.o_len.copy_(st.new_len, non_blocking=True)
        self.o_topk.copy_(st.topk_idx, non_blocking=True)


class PipelinedHostIO(HostIO):
    """HostIO with the host->device copies of the next step overlapped with
    the current step's kernels, and with few copies per step.

    The per-step inputs that do not live in the KV cache (hidden state, tree
    queries, verify logits, root tokens, prefix lengths) are packed into one
    pinned host buffer and copied with one copy into one of two device
    buffers, whose views the step reads: a copy stream fills the buffer of
    step k+1 while step k runs on the compute stream, once the step that last
    used that buffer has finished.  The tree K/V slots of step k go through
    the copy stream too, ahead of that, as soon as step k-1 (whose attention
    and compaction use the same cache) has finished.  The step writes its
    results into views of one device buffer, read back with one copy.
    """

    _KEYS = ("h", "q", "root_tok", "prefix_len")

    @staticmethod
    def _pack(specs, align=256):
        offs, total = [], 0
        for _, t in specs:
            total = (total + align - 1) // align * align
            offs.append(total)
            total += t.numel() * t.element_size()
        return offs, total

    def __init__(self, st: VerifyStep):
        super().__init__(st)
        c, dev = st.cfg, st.dev
        ins = [("h", self.h), ("q", self.q), ("vlog", self.vlog), ("root_tok", self.root),
               ("prefix_len", self.plen)]
        offs, total = self._pack(ins)
        self.host_in = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        self.dev_in = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]

        def view(buf, off, t):
            n = t.numel() * t.element_size()
            return buf[off:off + n].view(t.dtype).view(t.shape)

        for (name, t), off in zip(ins, offs):
            view(self.host_in, off, t).copy_(t)
        self.sets = [{name: view(buf, off, t) for (name, t), off in zip(ins, offs)}
                     for buf in self.dev_in]
        # results: views of one int32 device buffer, read back with one copy
        outs = [("accept_len", self.o_alen), ("accept_nodes", self.o_nodes),
                ("next_tok", self.o_next), ("new_len", self.o_len), ("topk_idx", self.o_topk)]
        n_out = sum(t.numel() for _, t in outs)
        self.dev_out = torch.empty(n_out, dtype=torch.int32, device=dev)
        self.host_out = torch.empty(n_out, dtype=torch.int32, pin_memory=True)
        o = 0
        for name, t in outs:
            setattr(st, name, self.dev_out[o:o + t.numel()].view(t.shape))
            setattr(self, {"accept_len": "o_alen", "accept_nodes": "o_nodes", "next_tok": "o_next",
                           "new_len": "o_len", "topk_idx": "o_topk"}[name],
                    self.host_out[o:o + t.numel()].view(t.shape))
            o += t.numel()
        self.copy_stream = torch.cuda.Stream(dev)
        self.ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.free = [torch.cuda.Event(), torch.cuda.Event()]
        self.kv_ready = torch.cuda.Event()

    def h2d_bytes(self) -> int:
        return self.host_in.numel() + sum(t.numel() * t.element_size()
                                          for t in (self.tree_k, self.tree_v))

    def _copy_inputs(self, j: int, wait_free: bool) -> None:
        with torch.cuda.stream(self.copy_stream):
            if wait_free:   # the step that used buffer j earlier in this run has finished
                self.copy_stream.wait_event(self.free[j])
            self.dev_in[j].copy_(self.host_in, non_blocking=True)
            self.ready[j].record(self.copy_stream)

    def run(self, n: int) -> None:
        """n steps; the inputs of step k+1 are copied while step k computes.
        All host->device copies go through the copy stream, in the order they
        are needed: once step k-1 has finished, the tree K/V slots of step k
        (which step k-1's attention and compaction used), then the packed
        inputs of step k+1, which overlap step k's kernels.  Every event a
        run waits on is recorded within the same run, so a run can also be
        captured into a CUDA graph (``capture``)."""
        st, c = self.st, self.st.cfg
        cs = torch.cuda.current_stream(st.dev)
        if n <= 0:
            return
        self.copy_stream.wait_stream(cs)   # no copy starts before the work already queued
        self._copy_inputs(0, wait_free=False)
        for k in range(n):
            j = k & 1
            with torch.cuda.stream(self.copy_stream):
                if k >= 1:   # step k-1 has released the cache slots
                    self.copy_stream.wait_event(self.free[j ^ 1])
                for b in range(c.B):
                    st.x["k_cache"][b, self.L[b]:self.L[b] + c.N].copy_(self.tree_k[b],
                                                                        non_blocking=True)
                    st.x["v_cache"][b, self.L[b]:self.L[b] + c.N].copy_(self.tree_v[b],
                                                                        non_blocking=True)
                self.kv_ready.record(self.copy_stream)
            if k + 1 < n:
                self._copy_inputs(j ^ 1, wait_free=k >= 1)
            cs.wait_event(self.ready[j])
            cs.wait_event(self.kv_ready)
            cur = self.sets[j]
            for key in self._KEYS:
                st.x[key] = cur[key]
            st.vlogits = cur["vlog"]
            st.run()
            self.free[j].record(cs)
            self.host_out.copy_(self.dev_out, non_blocking=True)

    def capture(self, steps_per_graph: int = 8) -> None:
        """Capture ``steps_per_graph`` pipelined steps (host copies included:
        the graph's copy nodes read the pinned host buffers at every replay)
        into a CUDA graph; ``replay()`` then runs them with one launch."""
        dev = self.st.dev
        self.run(2)   # library set-up (first-call attributes, tensor maps) outside the capture
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.run(steps_per_graph)
        torch.cuda.synchronize(dev)
        self.steps_per_graph = steps_per_graph

    def replay(self) -> None:
        self.graph.replay()
