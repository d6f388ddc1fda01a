"""Helpers shared by the GPU parity tests: move synthetic layers to the device and compare
results with the oracle's."""
import os

import numpy as np
import torch

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import synth

# Tolerance on y for the decode operator (fp32 accumulation over bf16/fp16 inputs):
# relative L2 error <= 2e-3 and max-abs error <= 1e-2 x RMS of the reference.
REL_L2 = 2e-3
MAX_ABS_OVER_RMS = 1e-2


def _raw_to_torch(raw, dtype):
    if dtype == synth.BF16:
        return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16).copy()).view(
            torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(raw))


def to_torch_x(layer):
    return _raw_to_torch(layer.x_raw, layer.x_dtype)


def to_torch_s(layer):
    return _raw_to_torch(layer.s_raw, layer.s_dtype)


def device_layer(layer, dev="cuda"):
    """Device tensors of a layer; the codes are packed on the device by lq_pack."""
    b = torch.from_numpy(layer.b).to(dev)
    packed = lq.pack(b, layer.K, layer.d, layer.D)
    del b
    return dict(
        x=to_torch_x(layer).to(dev),
        s=to_torch_s(layer).to(dev),
        M=torch.from_numpy(layer.M).to(dev),
        sign=torch.from_numpy(layer.sign).to(dev),
        packed=packed,
    )


def run_gemm(layer, dl, workspace=None, route=None):
    return lq.gemm(dl["x"], dl["packed"], dl["M"], dl["s"], layer.d, layer.D, sign=dl["sign"],
                   block=layer.block, workspace=workspace, route=route)


def oracle_rows(orc, layer, rows, tokens=None, nthreads=None):
    """Oracle outputs for a subset of rows (and tokens): [len(tokens)][len(rows)] fp64."""
    x = layer.x if tokens is None else layer.x[tokens]
    if nthreads is None:
        nthreads = max(1, len(os.sched_getaffinity(0)))
    p = orc.pack(layer.b[rows], layer.K, layer.d, layer.D)
    return orc.forward(x, p, layer.M, layer.s[rows], layer.d, layer.D, sign=layer.sign,
                       block=layer.block, nthreads=nthreads)


def errors(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = y - ref
    rms = np.sqrt(np.mean(ref * ref))
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    mx = np.abs(err).max() / rms
    return rel, mx


# every comparison made by assert_close in this session: (what, rel-L2, max-abs/RMS), printed in
# the terminal summary (tests/conftest.py)
OBSERVED = []
# other figures a test reports (one line each), printed in the same summary
NOTES = []


def assert_close(y, ref, what=""):
    rel, mx = errors(y, ref)
    OBSERVED.append((what, rel, mx))
    assert np.isfinite(y).all(), what
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_OVER_RMS, f"{what}: max-abs/RMS {mx:.3e} > {MAX_ABS_OVER_RMS}"
    return rel, mx
