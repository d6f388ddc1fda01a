"""The product has no CPU path: the binding refuses host tensors before any work, and neither
the package nor the library reaches the oracle (which is test infrastructure). No GPU is used."""
import os
import re
import subprocess
import sys

import pytest
import torch

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import build as lqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fractional_bit_weight_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    lqbuild.build()


def _layer(K=256, N=128, d=2, D=5, batch=1):
    L = lq.lifted_bits(K, d, D)
    return dict(x=torch.randn(batch, K, dtype=torch.bfloat16),
                packed=torch.zeros(N, lq.row_stride_bytes(K, d, D) // 4, dtype=torch.int32),
                M=torch.randn(d, D), s=torch.ones(N, dtype=torch.float16),
                b=torch.ones(N, L, dtype=torch.int8), K=K, N=N, d=d, D=D, batch=batch)


def test_operator_refuses_host_tensors():
    t = _layer()
    with pytest.raises(TypeError, match="CUDA tensor"):
        lq.gemm(t["x"], t["packed"], t["M"], t["s"], t["d"], t["D"])
    with pytest.raises(TypeError, match="CUDA tensor"):
        lq.gemm(t["x"], t["packed"], t["M"], t["s"], t["d"], t["D"], route=lq.ROUTE_GEMV_BULK)


def test_steps_refuse_host_tensors():
    t = _layer()
    with pytest.raises(TypeError, match="CUDA tensor"):
        lq.pack(t["b"], t["K"], t["d"], t["D"])
    with pytest.raises(TypeError, match="CUDA tensor"):
        lq.unpack(t["packed"], t["K"], t["d"], t["D"])
    with pytest.raises(TypeError, match="CUDA tensor"):
        lq.whiten(t["x"])
    with pytest.raises(TypeError, match="CUDA tensor"):
        lq.lift(t["x"], t["M"], t["d"], t["D"])


def test_package_does_not_import_the_oracle():
    code = ("import sys, fractional_bit_weight_b200 as lq; lq.lib(); "
            "assert not any(m == 'oracle' or m.startswith('oracle.') for m in sys.modules)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_product_sources_do_not_reference_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle|#\s*include\s*[<\"].*oracle)", re.M)
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not pat.search(text), os.path.join(dirpath, f)
    text = open(os.path.join(ROOT, "include", "liblq.h"), encoding="utf-8").read()
    assert not pat.search(text)
