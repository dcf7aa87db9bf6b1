"""A C program that uses the library through include/qsa.h alone (tests/c_caller/prefill_host.c):
it builds with gcc against the header and the in-tree libqsa_b200.so, its host-side calls work
without a GPU, and on the GPU its qsa_prefill_host output equals the Python binding's prefill of
the same inputs bit for bit."""
import os
import subprocess

import numpy as np
import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    lib = B.build()
    libdir = os.path.dirname(lib)
    out = str(tmp_path_factory.mktemp("c_caller") / "prefill_host")
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I",
           os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_caller", "prefill_host.c"), "-o", out,
           "-L", libdir, "-lqsa_b200", "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def test_c_caller_host_side_calls(exe):
    p = subprocess.run([exe, "check"], capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "check ok" in p.stdout


@pytest.mark.gpu
def test_c_caller_prefill_equals_the_binding(exe, tmp_path):
    T = 6000
    p = subprocess.run([exe, "run", str(tmp_path), str(T), "12345"], capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stdout + p.stderr
    from hybrid_sparse_attention_qsa_b200 import qsa as Q

    def load(name, shape):
        a = np.fromfile(tmp_path / f"{name}.bin", dtype=np.uint16).reshape(shape)
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to("cuda:0")

    x = dict(q=load("q", (1, T, 16, 128)), k=load("k", (1, T, 2, 128)), v=load("v", (1, T, 2, 128)),
             qi=load("qi", (1, T, 4, 64)), ki=load("ki", (1, T, 64)))
    got = load("out", (1, T, 16, 128))
    ref = Q.prefill(x["q"], x["k"], x["v"], x["qi"], x["ki"], topk=512)
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == Q.QSA_OK
    assert torch.equal(got, ref["out"])
