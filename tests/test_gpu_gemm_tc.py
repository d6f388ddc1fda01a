"""Parity of lq_gemm's two tensor-core routes (large batches) with the fp64 oracle: the lifted
GEMM over fp16 z and the +-1 codes, and the dequantise-once GEMM over fp16 T(x) and fp16
W = blockwise M b. Each test runs on both routes (lq_gemm_on_route).

Shapes span several 128-token x 256-row tiles with ragged tails in tokens, rows and the
contraction length; one shape gives every CTA several tiles (both accumulators and the whole
shared-memory ring are reused); inputs of very different magnitudes check the per-token
power-of-two scale of the fp16 activations.
"""
import numpy as np
import pytest
import torch

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import synth
from gpu_helpers import assert_close, device_layer, errors, oracle_rows, run_gemm, REL_L2

pytestmark = pytest.mark.gpu

ROUTES = [lq.ROUTE_GEMM_TC, lq.ROUTE_GEMM_DQ]

TC = [
    # (K, N, d, D, batch, block, x_dtype, s_dtype)
    (512, 600, 10, 24, 200, 256, synth.BF16, synth.F16),    # 3x2 tiles, ragged L, N, batch
    (256, 256, 2, 5, 64, 256, synth.F32, synth.F32),        # one partial token tile
    (300, 130, 3, 8, 129, 0, synth.F16, synth.BF16),        # identity T; N % 4 != 0
    (1024, 1000, 1, 2, 128, 1024, synth.BF16, synth.F16),   # 2 bits, whole-K Hadamard
    (8192, 300, 10, 24, 100, 256, synth.BF16, synth.F16),   # 308 stages per tile
    (96, 513, 16, 32, 300, 32, synth.BF16, synth.F16),      # D = 32: one word per group
    (4096, 260, 10, 25, 65, 4096, synth.BF16, synth.F32),
]


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("K,N,d,D,batch,block,xdt,sdt", TC)
def test_tc_gemm_all_outputs(orc, K, N, d, D, batch, block, xdt, sdt, route):
    layer = synth.make_layer("tc", 11, K + N + batch, K, N, d, D, batch, block=block, x_dtype=xdt,
                             s_dtype=sdt)
    dl = device_layer(layer)
    ws = lq.new_workspace(batch, K, N, d, D, block=block, route=route)
    y = run_gemm(layer, dl, ws, route=route).cpu().numpy()
    assert lq.device_status(ws) == (lq.LQ_OK, 0)
    ref = oracle_rows(orc, layer, np.arange(N))
    what = f"route {route}: K={K} N={N} d={d} D={D} batch={batch}"
    rel, mx = assert_close(y, ref, what)
    print(f"{what}: rel_l2={rel:.2e} max_abs/rms={mx:.2e}")


@pytest.mark.parametrize("route", ROUTES)
def test_tc_gemm_many_tiles_per_cta(orc, route):
    """157 x 2 tiles: more than one tile per CTA on any GPU with up to 157 SMs."""
    K, N, d, D, batch = 64, 40000, 4, 12, 256
    layer = synth.make_layer("tc_many", 12, 0, K, N, d, D, batch, block=64)
    dl = device_layer(layer)
    y = run_gemm(layer, dl, route=route).cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, N, 37), np.arange(N - 300, N)]))
    ref = oracle_rows(orc, layer, rows)
    assert_close(y[:, rows], ref, "many tiles per CTA")


@pytest.mark.parametrize("route", ROUTES)
def test_tc_gemm_per_token_scale(orc, route):
    """Tokens scaled by 1e-20 .. 1e20: each token's outputs keep their own relative accuracy."""
    K, N, d, D, batch = 512, 384, 10, 24, 96
    layer = synth.make_layer("tc_scale", 13, 0, K, N, d, D, batch, block=256, x_dtype=synth.F32,
                             s_dtype=synth.F32)
    f = (10.0 ** np.linspace(-20, 20, batch)).astype(np.float32)
    layer.x_raw = (layer.x_raw * f[:, None]).astype(np.float32)
    layer.x = layer.x_raw.astype(np.float64)
    dl = device_layer(layer)
    y = run_gemm(layer, dl, route=route).cpu().numpy()
    ref = oracle_rows(orc, layer, np.arange(N))
    for t in range(batch):
        rel, mx = errors(y[t], ref[t])
        assert rel <= REL_L2 and np.isfinite(y[t]).all(), (t, f[t], rel)


@pytest.mark.parametrize("route", ROUTES)
def test_tc_gemm_zero_input(route):
    K, N, d, D, batch = 256, 256, 2, 5, 64
    layer = synth.make_layer("tc_zero", 14, 0, K, N, d, D, batch, block=256)
    dl = device_layer(layer)
    dl["x"].zero_()
    y = run_gemm(layer, dl, route=route)
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("route", ROUTES)
def test_tc_gemm_repeat_is_deterministic(route):
    K, N, d, D, batch = 2048, 700, 10, 24, 160
    layer = synth.make_layer("tc_rep", 15, 0, K, N, d, D, batch)
    dl = device_layer(layer)
    ws = lq.new_workspace(batch, K, N, d, D, block=layer.block, route=route)
    y1 = run_gemm(layer, dl, ws, route=route).clone()
    y2 = run_gemm(layer, dl, ws, route=route).clone()
    assert torch.equal(y1, y2)
    assert lq.device_status(ws) == (lq.LQ_OK, 0)


@pytest.mark.parametrize("route", ROUTES)
def test_prefill_workload_on_both_routes(orc, route):
    """The 2048-token prefill layer (8192 -> 28672, (10, 24)) on each route: all 28672 rows of
    a seeded sample of 24 tokens against the oracle."""
    spec = synth.workload_specs(5)[0]
    layer = synth.build(spec)
    dl = device_layer(layer)
    ws = lq.new_workspace(layer.batch, layer.K, layer.N, layer.d, layer.D, block=layer.block,
                          route=route)
    y = run_gemm(layer, dl, ws, route=route)
    assert lq.device_status(ws) == (lq.LQ_OK, 0)
    toks = np.sort(np.random.Generator(np.random.PCG64(55)).choice(layer.batch, 24, replace=False))
    got = y[torch.from_numpy(toks).cuda()].cpu().numpy()
    del y, ws, dl
    torch.cuda.empty_cache()
    ref = oracle_rows(orc, layer, np.arange(layer.N), toks)
    rel, mx = assert_close(got, ref, f"prefill route {route}")
    print(f"prefill route {route}: {got.size} outputs, rel_l2={rel:.2e} max_abs/rms={mx:.2e}")
