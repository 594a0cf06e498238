"""CPU tests of the C ABI: the library loads, exports every symbol that
include/medusa.h declares, its host tree plan matches the oracle bit for bit,
and argument validation rejects bad calls before touching the GPU."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from oracle import medusa_oracle as O
from medusa_head_speculative_02_b200 import _lib as L
from medusa_head_speculative_02_b200.api import tree_plan_host
from medusa_head_speculative_02_b200.synthetic import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "medusa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(medusa_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = L.lib()
    names = _declared_symbols()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.SIGNATURES)


def test_version_string():
    assert b"sm_100a" in L.lib().medusa_version()


def test_debug_library_exports_every_declared_symbol():
    """libmedusa_debug.so (MEDUSA_DEBUG index checks) has the same ABI."""
    path = os.path.join(os.path.dirname(L.LIB_PATH), "libmedusa_debug.so")
    dbg = C.CDLL(path)
    for n in _declared_symbols():
        assert hasattr(dbg, n), n
    dbg.medusa_version.restype = C.c_char_p
    assert b"MEDUSA_DEBUG" in dbg.medusa_version()


@pytest.mark.parametrize("name", list(CONFIGS))
def test_host_tree_plan_matches_oracle(name):
    cfg = CONFIGS[name]
    ref = O.tree_plan(cfg.K, cfg.s, cfg.N)
    parent, depth, rank_path, anc = tree_plan_host(cfg.K, cfg.s, cfg.N)
    assert (parent.numpy() == ref["parent"]).all()
    assert (depth.numpy() == ref["depth"]).all()
    assert (rank_path.numpy() == ref["rank_path"]).all()
    assert (anc.numpy().view(np.uint32) == ref["anc_mask"]).all()


@pytest.mark.parametrize("K,s,N", [(1, 1, 1), (1, 5, 6), (2, 2, 5), (3, 4, 30), (5, 3, 200),
                                   (8, 2, 256), (3, 16, 256), (4, 7, 97), (2, 16, 256)])
def test_host_tree_plan_matches_oracle_various(K, s, N):
    ref = O.tree_plan(K, s, N)
    parent, depth, rank_path, anc = tree_plan_host(K, s, N)
    assert (parent.numpy() == ref["parent"]).all()
    assert (depth.numpy() == ref["depth"]).all()
    assert (rank_path.numpy() == ref["rank_path"]).all()
    assert (anc.numpy().view(np.uint32) == ref["anc_mask"]).all()


def test_tree_plan_rejects_bad_sizes():
    lib = L.lib()
    assert lib.medusa_tree_plan_host(0, 3, 4, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.medusa_tree_plan_host(2, 2, 8, None, None, None, None) == L.ERR_INVALID_ARG  # > 7 tuples
    assert lib.medusa_tree_plan_host(2, 2, 7, None, None, None, None) == L.OK
    assert lib.medusa_tree_plan_host(9, 2, 8, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.medusa_tree_plan_host(3, 17, 8, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.medusa_tree_plan_host(5, 3, 257, None, None, None, None) == L.ERR_INVALID_ARG
    assert b"N" in lib.medusa_last_error()


def test_validation_before_any_launch():
    lib = L.lib()
    p = C.c_void_p(256)
    # bad dtype, d not a multiple of 8, nothing requested, B too large, unaligned
    assert lib.medusa_heads_forward(p, p, None, p, 1, 64, 10, 2, 7, p, 1, p, None, p, 1 << 20,
                                    None) == L.ERR_INVALID_ARG
    assert lib.medusa_heads_forward(p, p, None, p, 1, 60, 10, 2, L.BF16, p, 1, p, None, p,
                                    1 << 20, None) == L.ERR_UNSUPPORTED
    assert lib.medusa_heads_forward(p, p, None, p, 1, 64, 10, 2, L.BF16, None, 1, None, None, p,
                                    1 << 20, None) == L.ERR_INVALID_ARG
    # bf16 batches beyond MEDUSA_MAX_HEADS_B (4096); fp32 beyond 16
    assert lib.medusa_heads_forward(p, p, None, p, 4097, 64, 10, 2, L.BF16, p, 1, p, None, p,
                                    1 << 20, None) == L.ERR_UNSUPPORTED
    assert lib.medusa_heads_forward(p, p, None, p, 17, 64, 10, 2, L.F32, p, 1, p, None, p,
                                    1 << 20, None) == L.ERR_UNSUPPORTED
    assert lib.medusa_heads_forward(C.c_void_p(258), p, None, p, 1, 64, 10, 2, L.BF16, p, 1, p,
                                    None, p, 1 << 20, None) == L.ERR_INVALID_ARG
    assert lib.medusa_heads_forward(p, p, None, p, 1, 64, 10, 2, L.BF16, p, 11, p, None, p,
                                    1 << 20, None) == L.ERR_INVALID_ARG      # s > V
    assert lib.medusa_topk(p, L.BF16, 4, 10, 0, p, None, None) == L.ERR_INVALID_ARG
    # both acceptance rules in one pass: greedy outputs missing, or shared with typical's
    q, r = C.c_void_p(512), C.c_void_p(768)
    assert lib.medusa_accept_greedy_typical(p, L.BF16, p, p, 2, 10, 0.7, 0.09, 0.6, None, q, r,
                                            p, q, r, p, 1 << 20, None) == L.ERR_INVALID_ARG
    assert lib.medusa_accept_greedy_typical(p, L.BF16, p, p, 2, 10, 0.7, 0.09, 0.6, p, q, r,
                                            p, q, r, p, 1 << 20, None) == L.ERR_INVALID_ARG
    assert b"overlap" in lib.medusa_last_error()
    assert lib.medusa_topk(p, L.BF16, 4, 10, 17, p, None, None) == L.ERR_INVALID_ARG
    # calls taking a tree reject a NULL plan
    assert lib.medusa_build_tree(None, p, p, p, 1, p, p, None) == L.ERR_INVALID_ARG
    assert lib.medusa_tree_attention(p, p, p, p, None, 1, 4, 4, 128, 64, 0.1, L.BF16, p, p, 1,
                                     None) == L.ERR_INVALID_ARG
    assert lib.medusa_accept_greedy(p, L.BF16, p, None, 1, 10, p, p, p, p, 1, None) == \
        L.ERR_INVALID_ARG
    assert lib.medusa_kv_compact(p, p, p, p, p, 1, 4, 128, 64, 9, L.BF16, p, None) == \
        L.ERR_INVALID_ARG
    assert lib.medusa_kv_compact(p, p, p, p, p, 1, 1, 1, 64, 4, L.BF16, p, None) == \
        L.ERR_UNSUPPORTED
    st = C.c_int()
    assert lib.medusa_device_status(None, 0) == L.ERR_INVALID_ARG
    assert lib.medusa_heads_workspace_size(0, 64, 10, 2, 1, L.BF16) == 0


def test_shard_merge_and_attention_plan_queries_validate_first():
    """The shard merge and the attention plan queries reject bad arguments
    before any CUDA call."""
    lib = L.lib()
    p = C.c_void_p(256)
    # G < 1, c < 1, s out of range, shard stride below R * c, NULL outputs
    assert lib.medusa_topk_merge(p, p, 40, None, 0, 4, 10, 10, p, p, None) == L.ERR_INVALID_ARG
    assert lib.medusa_topk_merge(p, p, 40, None, 2, 4, 0, 10, p, p, None) == L.ERR_INVALID_ARG
    assert lib.medusa_topk_merge(p, p, 40, None, 2, 4, 10, 0, p, p, None) == L.ERR_INVALID_ARG
    assert lib.medusa_topk_merge(p, p, 40, None, 2, 4, 10, 17, p, p, None) == L.ERR_INVALID_ARG
    assert lib.medusa_topk_merge(p, p, 39, None, 2, 4, 10, 10, p, p, None) == L.ERR_INVALID_ARG
    assert lib.medusa_topk_merge(p, p, 40, None, 2, 4, 10, 10, None, p, None) == \
        L.ERR_INVALID_ARG
    assert lib.medusa_topk_merge(None, p, 40, None, 2, 4, 10, 10, p, p, None) == \
        L.ERR_INVALID_ARG
    # no rows: nothing to do, accepted without touching the pointers
    assert lib.medusa_topk_merge(None, None, 0, None, 2, 0, 10, 10, None, None, None) == L.OK
    # plan queries reject a NULL tree (the other checks need a tree, whose
    # plan lives on the device)
    for fn in (lib.medusa_tree_attention_chunks, lib.medusa_tree_attention_launches,
               lib.medusa_tree_attention_tiles_per_cta):
        assert fn(None, 1, 4, 4, 128, 4096, L.BF16) == L.ERR_INVALID_ARG
