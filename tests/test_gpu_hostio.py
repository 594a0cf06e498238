"""The pipelined end-to-end path (next step's inputs copied on a second
stream while the current step computes) gives the same results as the
sequential host-buffer path, step for step."""
import pytest
import torch

from medusa_head_speculative_02_b200.step import HostIO, PipelinedHostIO, VerifyStep
from medusa_head_speculative_02_b200.synthetic import MedusaConfig

pytestmark = pytest.mark.gpu

CFG = MedusaConfig("hostio_small", "bf16", B=3, d=512, V=1000, K=4, s=3, N=16, Hq=4, Hkv=2,
                   dh=128, L_lo=100, L_hi=300)


def test_pipelined_host_io_equals_sequential():
    st = VerifyStep(CFG, "cuda", seed=3)
    seq = HostIO(st)
    seq.step()
    torch.cuda.synchronize()
    want = [t.clone() for t in (seq.o_alen, seq.o_nodes, seq.o_next, seq.o_len, seq.o_topk)]
    attn = st.attn_out.clone()
    st2 = VerifyStep(CFG, "cuda", seed=3)
    pio = PipelinedHostIO(st2)
    for n in (1, 2, 5):
        pio.run(n)
        torch.cuda.synchronize()
        got = (pio.o_alen, pio.o_nodes, pio.o_next, pio.o_len, pio.o_topk)
        for a, b in zip(got, want):
            assert torch.equal(a, b)
        assert torch.equal(st2.attn_out, attn)


def test_captured_host_io_equals_sequential():
    st = VerifyStep(CFG, "cuda", seed=4)
    seq = HostIO(st)
    seq.step()
    torch.cuda.synchronize()
    want = [t.clone() for t in (seq.o_alen, seq.o_nodes, seq.o_next, seq.o_len, seq.o_topk)]
    st2 = VerifyStep(CFG, "cuda", seed=4)
    pio = PipelinedHostIO(st2)
    pio.capture(4)
    # scribble over the device copies of the inputs: a replay must copy them again
    for t in (st2.x["h"], st2.x["q"], st2.vlogits):
        t.zero_()
    for s_ in pio.sets:
        for t in s_.values():
            t.zero_()
    pio.replay()
    torch.cuda.synchronize()
    got = (pio.o_alen, pio.o_nodes, pio.o_next, pio.o_len, pio.o_topk)
    for a, b in zip(got, want):
        assert torch.equal(a, b)
