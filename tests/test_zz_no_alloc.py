"""lq_gemm_noalloc: the decode GEMV for callers that cannot allocate device memory.

Such callers (a plugin or serving backend whose device memory belongs to a host framework, or
code that runs where allocating is not allowed) cannot pass lq_gemm a workspace; this entry
point keeps its scratch in a fixed device array owned by the library. The test calls it through
the C ABI and compares it with the fp64 oracle, and with lq_gemm on the same inputs, twice in a
row (the second call finds the scratch as the first call left it). It runs last so that a failure here does not hide the
other GPU tests, and passes both on its own and after them.
"""
import ctypes

import numpy as np
import pytest
import torch

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import synth
from gpu_helpers import assert_close, device_layer, oracle_rows

pytestmark = pytest.mark.gpu


def _call_noalloc(layer, dl, y):
    desc = lq.WhitenDesc(dl["sign"].data_ptr(), None, layer.block)
    return lq.lib().lq_gemm_noalloc(
        ctypes.c_void_p(dl["x"].data_ptr()), lq._DTYPES[dl["x"].dtype], layer.batch,
        ctypes.byref(desc), ctypes.c_void_p(dl["packed"].data_ptr()),
        ctypes.c_void_p(dl["M"].data_ptr()), ctypes.c_void_p(dl["s"].data_ptr()),
        lq._DTYPES[dl["s"].dtype], layer.d, layer.D, layer.K, layer.N,
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("K,N,d,D,batch", [(4096, 4096, 10, 24, 1), (8192, 3000, 3, 8, 3),
                                           (28672, 1024, 10, 24, 2), (256, 128, 2, 5, 1)])
def test_noalloc_matches_oracle_and_gemm_twice(orc, K, N, d, D, batch):
    layer = synth.make_layer("noalloc", 11, K + N + batch, K, N, d, D, batch)
    dl = device_layer(layer)
    ref = oracle_rows(orc, layer, np.arange(N))
    y_gemm = lq.gemm(dl["x"], dl["packed"], dl["M"], dl["s"], d, D, sign=dl["sign"],
                     block=layer.block).cpu().numpy()
    what = f"K={K} N={N} d={d} D={D} batch={batch}"
    for _ in range(2):
        y = torch.full((batch, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call_noalloc(layer, dl, y) == lq.LQ_OK, lq.lib().lq_last_error().decode()
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert_close(got, ref, f"noalloc vs oracle, {what}")
        assert_close(got, y_gemm, f"noalloc vs lq_gemm, {what}")


def test_noalloc_rejects_what_does_not_fit():
    fake = ctypes.c_void_p(0x10000)     # never dereferenced: the call is rejected first
    # 1 token of a 2^24-input row: ~3900 K-slices, whose fragments and partials need far more
    # than the library's scratch
    rc = lq.lib().lq_gemm_noalloc(fake, lq.LQ_BF16, 1, None, fake, fake, fake, lq.LQ_F16, 10, 24,
                                  1 << 24, 1024, fake, None)
    assert rc == lq.LQ_EINVAL
    assert "scratch" in lq.lib().lq_last_error().decode()
    # 8 tokens of a 2^20-input row: no GEMV plan (the fragments of a slice wide enough for the
    # rows to fit the partial slots outgrow shared memory)
    rc = lq.lib().lq_gemm_noalloc(fake, lq.LQ_BF16, 8, None, fake, fake, fake, lq.LQ_F16, 10, 24,
                                  1 << 20, 1024, fake, None)
    assert rc in (lq.LQ_EINVAL, lq.LQ_EUNSUPPORTED)
    rc = lq.lib().lq_gemm_noalloc(fake, lq.LQ_BF16, 9, None, fake, fake, fake, lq.LQ_F16, 10, 24,
                                  4096, 4096, fake, None)
    assert rc == lq.LQ_EINVAL
