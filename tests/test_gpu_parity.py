"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on seeded synthetic inputs.

Bit packing must match byte for byte; whitening and lift are fp32 computations of exact
inputs; the decode operator must meet relative L2 <= 2e-3 and max-abs <= 1e-2 x RMS.
"""
import numpy as np
import pytest
import torch

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import synth
from gpu_helpers import assert_close, device_layer, errors, oracle_rows, run_gemm, to_torch_x

pytestmark = pytest.mark.gpu


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ---------------------------------------------------------------- packing (bit-exact)

@pytest.mark.parametrize("N,K,d,D", [(1, 1, 1, 1), (3, 7, 3, 5), (17, 256, 2, 5),
                                     (5, 4096, 10, 24), (9, 100, 10, 25), (33, 8192, 1, 2),
                                     (4, 8192, 3, 8), (2, 28672, 10, 24), (7, 96, 16, 32)])
def test_pack_bytes_match_oracle(orc, N, K, d, D):
    G = -(-K // d)
    b = synth.random_signs(_rng(N * 1000 + K), (N, G * D))
    packed = lq.pack(torch.from_numpy(b).cuda(), K, d, D)
    got = packed.cpu().numpy().view(np.uint8).reshape(N, -1)
    expect = orc.pack(b, K, d, D)
    assert got.shape == expect.shape
    assert np.array_equal(got, expect)
    back = lq.unpack(packed, K, d, D).cpu().numpy()
    assert np.array_equal(back, b)


def test_pack_exhaustive_codewords(orc):
    for d, D in [(1, 2), (2, 4), (2, 5), (3, 8)]:
        G = 5
        C = np.array([[(-1 if (c >> j) & 1 else 1) for j in range(D)] for c in range(1 << D)],
                     np.int8)
        b = np.tile(C, (1, G))
        packed = lq.pack(torch.from_numpy(b).cuda(), G * d, d, D)
        got = packed.cpu().numpy().view(np.uint8).reshape(1 << D, -1)
        assert np.array_equal(got, orc.pack(b, G * d, d, D))


# ---------------------------------------------------------------- whitening and lift

def _x(rng, batch, K, dtype):
    raw, exact = synth.round_to(rng.standard_normal((batch, K)).astype(np.float32), dtype)
    t = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16) if dtype == synth.BF16 \
        else torch.from_numpy(raw)
    return t.cuda(), exact


@pytest.mark.parametrize("block,K,dtype", [(0, 300, synth.F32), (1, 64, synth.F16),
                                           (2, 64, synth.BF16), (256, 4096, synth.BF16),
                                           (4096, 8192, synth.F32), (16, 48, synth.F32)])
def test_whiten_matches_oracle(orc, block, K, dtype):
    rng = _rng(block + K)
    x, xe = _x(rng, 3, K, dtype)
    sign = synth.random_signs(rng, (K,))
    cs = rng.uniform(0.5, 2.0, K).astype(np.float32)
    got = lq.whiten(x, sign=torch.from_numpy(sign).cuda(), chan_scale=torch.from_numpy(cs).cuda(),
                    block=block).cpu().numpy()
    ref = orc.whiten(xe, sign=sign, chan_scale=cs, block=block) if block else xe
    rel, mx = errors(got, ref)
    assert rel < 1e-6 and mx < 1e-5, (rel, mx)


@pytest.mark.parametrize("K,d,D,block,batch", [(256, 2, 5, 256, 1), (4096, 10, 24, 256, 2),
                                               (1000, 3, 8, 8, 3), (37, 10, 25, 0, 1),
                                               (8192, 4, 12, 4096, 1), (512, 16, 32, 1, 2)])
def test_lift_matches_oracle(orc, K, d, D, block, batch):
    rng = _rng(K + d)
    x, xe = _x(rng, batch, K, synth.BF16)
    sign = synth.random_signs(rng, (K,))
    M = (rng.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    got = lq.lift(x, torch.from_numpy(M).cuda(), d, D, sign=torch.from_numpy(sign).cuda(),
                  block=block).cpu().numpy()
    ref = orc.lift(xe, M, d, D, sign=sign, block=block)
    rel, mx = errors(got, ref)
    assert rel < 1e-6 and mx < 1e-5, (rel, mx)


# ---------------------------------------------------------------- decode operator, all rows

SMALL = [
    # (K, N, d, D, batch, block, x_dtype, s_dtype): several tiles, ragged tails
    (256, 128, 2, 5, 1, 256, synth.F32, synth.F32),
    (1000, 67, 10, 24, 1, 8, synth.BF16, synth.F16),
    (4096, 300, 10, 24, 3, 256, synth.BF16, synth.F16),
    (2048, 129, 3, 8, 5, 256, synth.F16, synth.BF16),
    (777, 65, 1, 2, 2, 1, synth.F32, synth.F32),
    (512, 200, 4, 12, 9, 0, synth.BF16, synth.F16),
    (8192, 70, 10, 25, 17, 256, synth.BF16, synth.F16),
    (1536, 64, 16, 32, 63, 512, synth.BF16, synth.F16),
    (96, 1, 2, 4, 1, 32, synth.F32, synth.F32),
    (4096, 513, 10, 24, 8, 4096, synth.BF16, synth.F16),
    (8192, 300, 10, 24, 2, 4096, synth.BF16, synth.F16),
    (4096, 100, 10, 24, 3, 1024, synth.F16, synth.F32),
]


def test_small_shapes_reach_every_route():
    """The small shapes run every automatic route; the staged GEMV (chosen for one or two
    tokens on layers of >= 32 MB of codes, and where the register-streamed GEMV cannot take the
    batch in one launch) and the dequantise-once GEMM are also run on their own routes
    (test_gemm_small_on_staged_route, test_gpu_gemm_tc.py)."""
    routes = {lq.gemm_route(b, K, N, d, D, blk) for K, N, d, D, b, blk, _, _ in SMALL}
    assert routes >= {lq.ROUTE_GEMV_I8, lq.ROUTE_GEMM_TC, lq.ROUTE_GEMV_GROUPS}, routes
    staged = [s for s in SMALL
              if lq.lib().lq_gemm_route_workspace_bytes(s[4], s[0], s[1], s[2], s[3], s[5],
                                                        lq.ROUTE_GEMV_BULK) > 0]
    assert len(staged) >= 6, staged


@pytest.mark.parametrize("K,N,d,D,batch,block,xdt,sdt", SMALL)
def test_gemm_small_all_rows(orc, K, N, d, D, batch, block, xdt, sdt):
    layer = synth.make_layer("small", 99, K + N, K, N, d, D, batch, block=block, x_dtype=xdt,
                             s_dtype=sdt)
    dl = device_layer(layer)
    y = run_gemm(layer, dl).cpu().numpy()
    ref = oracle_rows(orc, layer, np.arange(N))
    route = lq.gemm_route(batch, K, N, d, D, block)
    assert_close(y, ref, f"K={K} N={N} d={d} D={D} batch={batch} route={route}")


@pytest.mark.parametrize("K,N,d,D,batch,block,xdt,sdt", SMALL)
def test_gemm_small_on_staged_route(orc, K, N, d, D, batch, block, xdt, sdt):
    """The staged int8 GEMV (lq_gemm_on_route), all outputs, twice on one workspace."""
    if lq.lib().lq_gemm_route_workspace_bytes(batch, K, N, d, D, block, lq.ROUTE_GEMV_BULK) == 0:
        pytest.skip("the staged GEMV's plan does not fit this shape")
    layer = synth.make_layer("small", 99, K + N, K, N, d, D, batch, block=block, x_dtype=xdt,
                             s_dtype=sdt)
    dl = device_layer(layer)
    ws = lq.new_workspace(batch, K, N, d, D, block=block, route=lq.ROUTE_GEMV_BULK)
    ref = oracle_rows(orc, layer, np.arange(N))
    for _ in range(2):
        y = run_gemm(layer, dl, ws, route=lq.ROUTE_GEMV_BULK).cpu().numpy()
        assert_close(y, ref, f"staged K={K} N={N} d={d} D={D} batch={batch}")
    assert lq.device_status(ws) == (lq.LQ_OK, 0)


def test_staged_route_two_tokens_full_size(orc):
    """Two tokens on the Llama-3-70B gate/up shape (8192 -> 28672, d=10, D=24, block 256, bf16
    x, f16 s) take the staged GEMV by default: all 28672 x 2 outputs against the oracle."""
    K, N, d, D, batch = 8192, 28672, 10, 24, 2
    assert lq.gemm_route(batch, K, N, d, D, 256) == lq.ROUTE_GEMV_BULK
    layer = synth.make_layer("gateup2", 12, 0, K, N, d, D, batch, block=256, x_dtype=synth.BF16,
                             s_dtype=synth.F16)
    dl = device_layer(layer)
    y = run_gemm(layer, dl).cpu().numpy()
    ref = oracle_rows(orc, layer, np.arange(N))
    assert_close(y, ref, "staged GEMV, 2 tokens, 8192 x 28672")


def test_gemm_identity_special_case(orc):
    """d = D and M = I: a plain +-1 matrix-vector product of the whitened input."""
    layer = synth.make_layer("eye", 5, 0, 1024, 96, 4, 4, 2, block=256)
    layer.M = np.eye(4, dtype=np.float32)
    dl = device_layer(layer)
    y = run_gemm(layer, dl).cpu().numpy()
    xt = orc.whiten(layer.x, sign=layer.sign, block=256)
    ref = (xt @ layer.b.T.astype(np.float64)) * layer.s
    assert_close(y, ref, "M = I")


def test_gemm_repeat_is_deterministic(orc):
    layer = synth.make_layer("rep", 6, 0, 8192, 1000, 10, 24, 4)
    dl = device_layer(layer)
    ws = lq.new_workspace(4, 8192, 1000, 10, 24)
    y1 = run_gemm(layer, dl, ws).clone()
    y2 = run_gemm(layer, dl, ws).clone()
    assert torch.equal(y1, y2)
    assert lq.device_status(ws) == (lq.LQ_OK, 0)


def test_gemm_rejects_bad_arguments():
    layer = synth.make_layer("bad", 7, 0, 256, 16, 2, 5, 1)
    dl = device_layer(layer)
    with pytest.raises(lq.LQError):
        lq.gemm(dl["x"], dl["packed"], dl["M"], dl["s"], 2, 5, sign=dl["sign"], block=3)
    with pytest.raises(lq.LQError):
        lq.gemm(dl["x"], dl["packed"], dl["M"], dl["s"], 2, 5, sign=dl["sign"], block=256,
                workspace=torch.zeros(64, dtype=torch.uint8, device="cuda"))


# ---------------------------------------------------------------- the five workloads

def _sample_rows(N, n, seed):
    r = _rng(seed).choice(N, size=min(n, N), replace=False)
    return np.unique(np.concatenate([r, [0, N - 1]]))


def _check_workload(orc, cfg, max_rows=None, max_tokens=48):
    """Every output of every layer of a workload against the oracle, except on the 2048-token
    prefill, where the oracle's cost calls for a sample of rows and tokens (max_rows x
    max_tokens, chosen by a seeded draw plus the first and last row)."""
    specs = synth.workload_specs(cfg)
    cache = {}
    for spec in specs:
        name, seed, li, K, N, d, D, batch, kw = spec
        layer = synth.build(spec)
        key = (seed, li)
        if key not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            cache[key] = device_layer(layer)
        dl = dict(cache[key])
        dl["x"] = to_torch_x(layer).cuda()
        y = run_gemm(layer, dl).cpu().numpy()
        rows = np.arange(N) if max_rows is None or N <= max_rows else \
            _sample_rows(N, max_rows, cfg * 7 + li)
        toks = None if batch <= max_tokens else np.sort(_rng(cfg).choice(batch, max_tokens,
                                                                          replace=False))
        ref = oracle_rows(orc, layer, rows, toks)
        got = y[:, rows] if toks is None else y[toks][:, rows]
        route = lq.gemm_route(batch, K, N, d, D, layer.block)
        rel, mx = assert_close(got, ref, f"{name} route={route}")
        print(f"{name}: {got.size} outputs, rel_l2={rel:.2e} max_abs/rms={mx:.2e}")
    cache.clear()
    torch.cuda.empty_cache()


def test_workload_tiny_all_outputs(orc):
    _check_workload(orc, 1)


def test_workload_llama2_7b_qproj(orc):
    _check_workload(orc, 2)


def test_workload_llama3_70b_mlp(orc):
    _check_workload(orc, 3)


def test_workload_bitwidth_sweep(orc):
    _check_workload(orc, 4)


def test_workload_prefill(orc):
    _check_workload(orc, 5, max_rows=512)
