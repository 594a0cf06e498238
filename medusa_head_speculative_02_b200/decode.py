"""Multi-step speculative decoding over the verify step.

Medusa paper digest ("論文解説: Medusa") and the explainer's decoding loop:
every step drafts a tree from the heads, verifies it, keeps the accepted
path and continues from there.  Here each step runs the whole chain
(heads + top-s, tree expansion, tree attention, acceptance, KV compaction)
through the public API; the next token of a step becomes the root of the
next step's tree and its new lengths the next prefix lengths, so every
sequence's cache grows by 1 + accept_len per step.  One step can be captured
into a CUDA graph and replayed: the chain then runs without host work
between steps.  With a sampling temperature the next token is drawn from the
last accepted node's row ("3.3 贪婪vs采样验证" of the page "Medusa：基于多Token
预测的LLM推理加速") with a device-side draw counter as the noise offset, so
every replay of a captured step draws fresh noise.
"""
from __future__ import annotations

import torch

from . import api
from .step import VerifyStep
from .synthetic import MedusaConfig


class DecodeLoop:
    """Chained verify steps on one stream, eager or replayed from a CUDA graph.

    ``max_steps`` sizes the cache headroom: each step appends at most K + 1
    slots per sequence, so L_b + N <= Lcap holds for that many steps.
    """

    def __init__(self, cfg: MedusaConfig, device="cuda", seed: int = 0, max_steps: int = 64,
                 sample_temperature=None, sample_seed: int = 0):
        self.cfg = cfg.scaled(headroom=cfg.headroom + max_steps * (cfg.K + 1))
        self.max_steps = int(max_steps)
        self.st = VerifyStep(self.cfg, device, seed)
        x = self.st.x
        self._init = {k: x[k].clone() for k in ("prefix_len", "root_tok", "k_cache", "v_cache")}
        self.sample_temperature = sample_temperature
        self.sample_seed = int(sample_seed)
        self.draws = torch.zeros(1, dtype=torch.int64, device=self.st.dev)  # noise offset
        self.steps_done = 0
        self.graph = None

    def reset(self) -> None:
        """Back to the state before the first step (prefix lengths, roots,
        cache, draw counter)."""
        for k, v in self._init.items():
            self.st.x[k].copy_(v)
        self.draws.zero_()
        self.steps_done = 0

    def _advance(self) -> None:
        st = self.st
        st.run()
        if self.sample_temperature is not None:
            api.medusa_sample_next(st.vlogits, st.accept_len, st.accept_nodes,
                                   self.sample_temperature, self.sample_seed, 0,
                                   out=st.next_tok, offset_dev=self.draws)
            self.draws.add_(1)
        st.x["prefix_len"].copy_(st.new_len)
        st.x["root_tok"].copy_(st.next_tok)

    def step(self) -> None:
        if self.steps_done >= self.max_steps:
            raise RuntimeError(f"cache headroom covers {self.max_steps} steps")
        if self.graph is not None:
            self.graph.replay()
        else:
            self._advance()
        self.steps_done += 1

    def capture(self) -> None:
        """Capture one step into a CUDA graph.  One eager step runs first on a
        side stream (library set-up outside the capture), then the state is
        reset; later ``step()`` calls replay the graph."""
        dev = self.st.dev
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._advance()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        self.reset()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._advance()
        torch.cuda.synchronize(dev)
        self.graph = g
