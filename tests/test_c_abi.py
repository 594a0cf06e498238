"""CPU: the library is a C ABI.  A plain C program (tests/c_abi_client.c),
compiled with gcc against include/medusa.h and linked to libmedusa.so,
computes the tree plan through medusa_tree_plan_host; its output must equal
the oracle's plan ([MD] "ツリーアテンションによる並列検証": the top-N rank tuples
by 0.8^D 0.5^(sum of ranks)), and a bad request must come back as
MEDUSA_ERR_INVALID_ARG with a message."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import medusa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "medusa_head_speculative_02_b200")


@pytest.fixture(scope="module")
def client(tmp_path_factory):
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    if not os.path.exists(os.path.join(PKG, "libmedusa.so")):
        pytest.fail("libmedusa.so is missing: build with `python -m medusa_head_speculative_02_b200.build`")
    exe = str(tmp_path_factory.mktemp("c_abi") / "client")
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_client.c"), "-o", exe, "-L", PKG, "-lmedusa",
           "-Wl,-rpath," + PKG]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def _run(exe, K, s, N):
    r = subprocess.run([exe, str(K), str(s), str(N)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    return r.stdout.splitlines()


@pytest.mark.parametrize("K,s,N", [(4, 3, 16), (5, 10, 64), (5, 8, 128), (5, 3, 256)])
def test_c_client_tree_plan_equals_the_oracle(client, K, s, N):
    out = _run(client, K, s, N)
    assert out[0].startswith("version medusa-b200") and out[1] == "status 0"
    rows = np.array([[int(v) for v in line.split()] for line in out[2:]], dtype=np.int64)
    ref = O.tree_plan(K, s, N)
    assert rows.shape == (N, 2 + K + 1)
    assert (rows[:, 0] == ref["parent"]).all()
    assert (rows[:, 1] == ref["depth"]).all()
    assert (rows[:, 2:2 + K] == ref["rank_path"]).all()
    assert (rows[:, 2 + K].astype(np.uint32) == np.asarray(ref["anc_mask"])[:, 0]).all()


def test_c_client_bad_request_reports_invalid_arg(client):
    out = _run(client, 2, 2, 8)   # only 1 + 2 + 4 = 7 rank tuples
    assert out[1] == "status -1" and out[2].startswith("error ")
