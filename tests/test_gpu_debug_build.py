"""The debug build of the library (libqsa_b200_debug.so, compiled with -DQSA_DEBUG) on the GPU.

A child process with QSA_DEBUG=1 loads the debug library, runs every kernel family on small seeded
cases (tests/debug_cases.py) and checks that no device-side bounds check fired (status word) and
that the canary guard after every buffer the binding allocated is intact.  Its results must equal
the release library's on the same inputs bit for bit: the checks skip nothing in a correct run.
"""
import os
import subprocess
import sys

import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import build as B
from hybrid_sparse_attention_qsa_b200 import qsa as Q
from tests import debug_cases

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_runs_clean_with_intact_canaries_and_equals_release(tmp_path):
    if Q.DEBUG:
        pytest.skip("compares the debug library with the release one: run without QSA_DEBUG")
    B.build(debug=True)
    out = tmp_path / "debug.pt"
    env = dict(os.environ, QSA_DEBUG="1")
    p = subprocess.run([sys.executable, "-m", "tests.debug_cases", str(out)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    got = torch.load(out)
    assert got["lib"].endswith("libqsa_b200_debug.so")
    assert got["canaries_checked"] >= 20
    ref = debug_cases.run_cases("cuda:0")
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert sorted(got["results"]) == sorted(ref)
    for name, t in ref.items():
        assert torch.equal(got["results"][name], t), name
