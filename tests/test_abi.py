"""liblq.so loads, exports every entry point that include/liblq.h declares, and its host-side
logic (sizes, argument checks) agrees with the oracle. No GPU is used: every call below
returns before any CUDA work."""
import ctypes
import os
import re

import pytest

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import build as lqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "liblq.h")


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^LQ_API\s+[^(]*?\b(lq_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def L():
    lqbuild.build()
    return lq.lib()


def test_header_declares_entry_points():
    names = declared()
    for required in ("lq_pack", "lq_whiten", "lq_gemm"):
        assert required in names
    assert set(names) == set(lq.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {lq.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (lq_\w+)", out))
    assert set(declared()) <= exported
    assert exported <= set(declared()), exported - set(declared())


def test_sizes_match_oracle(L, orc):
    assert lq.abi_version() == 1
    for K, d, D in [(256, 2, 5), (4096, 10, 24), (28672, 10, 24), (8192, 3, 8), (7, 3, 5),
                    (1, 1, 1), (8192, 16, 32), (100, 10, 25)]:
        assert lq.lifted_bits(K, d, D) == orc.lifted_bits(K, d, D)
        assert lq.row_stride_bytes(K, d, D) == orc.row_bytes(K, d, D)
    for K, d, D in [(0, 1, 1), (10, 0, 1), (10, 5, 4), (10, 8, 33)]:
        assert lq.lifted_bits(K, d, D) == -1
        assert lq.row_stride_bytes(K, d, D) == -1


def test_workspace_bytes(L):
    assert lq.gemm_workspace_bytes(1, 4096, 4096, 10, 24) > 0
    assert lq.gemm_workspace_bytes(1, 4096, 4096, 10, 24) % 256 == 0
    assert lq.gemm_workspace_bytes(0, 4096, 4096, 10, 24) == 0
    assert lq.gemm_workspace_bytes(1, 4096, 0, 10, 24) == 0
    assert lq.gemm_workspace_bytes(1, 4096, 4096, 10, 33) == 0


def _r256(n):
    return -(-n // 256) * 256


def test_encode_arguments_without_gpu(L):
    fake = ctypes.c_void_p(0x10000)     # never dereferenced: every call below returns first
    S = None
    assert L.lq_encode(None, 4, 16, fake, 2, 5, 1, fake, None, S) == lq.LQ_EINVAL
    assert L.lq_encode(fake, 4, 16, fake, 2, 5, 7, fake, None, S) == lq.LQ_EINVAL    # mode
    assert "mode" in L.lq_last_error().decode()
    assert L.lq_encode(fake, 4, 16, fake, 5, 4, 1, fake, None, S) == lq.LQ_EINVAL    # D < d
    assert L.lq_encode(fake, -1, 16, fake, 2, 5, 1, fake, None, S) == lq.LQ_EINVAL
    assert L.lq_encode(ctypes.c_void_p(0x10002), 4, 16, fake, 2, 5, 1, fake, None, S) == \
        lq.LQ_EINVAL                                                                  # w align
    assert L.lq_encode(fake, 4, 64, fake, 17, 20, 1, fake, None, S) == lq.LQ_EUNSUPPORTED
    assert L.lq_encode(fake, 4, 64, fake, 2, 25, 0, fake, None, S) == lq.LQ_EUNSUPPORTED
    assert L.lq_encode(fake, 4, 64, fake, 2, 27, 1, fake, None, S) == lq.LQ_EUNSUPPORTED
    assert L.lq_encode(fake, 0, 64, fake, 2, 5, 1, fake, None, S) == lq.LQ_OK        # no work


def test_wait_timeout_check_arguments_without_gpu(L):
    assert L.lq_check_wait_timeout(None, 20, None) == lq.LQ_EINVAL
    assert "workspace" in L.lq_last_error().decode()
    assert L.lq_check_wait_timeout(ctypes.c_void_p(256), 0, None) == lq.LQ_EINVAL
    assert "limit_ms" in L.lq_last_error().decode()


def test_gemm_launches(L):
    assert lq.gemm_launches(1, 4096, 4096, 10, 24, 256) == 2        # two-kernel int8 GEMV
    assert lq.gemm_launches(2, 8192, 300, 10, 24, 4096) == 2        # two-kernel int8 GEMV
    assert lq.gemm_launches(2048, 8192, 28672, 10, 24, 256) == 3    # W, xt, dense GEMM
    assert lq.gemm_launches(64, 8192, 28672, 10, 24, 256) == 2      # lifted tcgen05 GEMM
    n16 = lq.gemm_launches(16, 28672, 8192, 10, 24, 256)            # token groups
    assert n16 >= 4 and n16 % 2 == 0
    assert lq.gemm_launches(0, 4096, 4096, 10, 24, 256) == 0
    assert lq.gemm_launches(1, 4096, 4096, 10, 24, 3) == 0


@pytest.mark.parametrize("K,N,max_single", [(4096, 4096, 8), (8192, 8192, 8), (8192, 28672, 4),
                                            (28672, 8192, 4), (256, 128, 8), (40, 64, 8)])
def test_small_batches_run_as_one_gemv(L, K, N, max_single):
    """Up to 4 tokens on the Llama-3-70B MLP shapes, up to 8 on 4096- and 8192-wide layers, the
    batch runs as one int8 GEMV (prep + contraction: register-streamed or TMA-staged) instead of
    token groups."""
    for b in range(1, max_single + 1):
        route = lq.gemm_route(b, K, N, 10, 24, 256)
        assert route in (lq.ROUTE_GEMV_BULK, lq.ROUTE_GEMV_I8), (b, route)
        assert lq.gemm_launches(b, K, N, 10, 24, 256) == 2


@pytest.mark.parametrize("batch,K,N,d,D", [(64, 8192, 28672, 10, 24), (2048, 8192, 28672, 10, 24),
                                           (200, 512, 600, 10, 24), (300, 96, 513, 16, 32)])
def test_workspace_of_tensor_core_path(L, batch, K, N, d, D):
    """batch >= 64, lifted GEMM: a 256-byte header, fp16 z [batch][L padded to 64], then batch
    fp32 scales. Dequantise-once GEMM: the header, fp16 W [N][Kw], fp16 xt [batch][Kw], batch
    fp32 scales (Kw = ceil(K/d)*d padded to 64)."""
    Lp = -(-lq.lifted_bits(K, d, D) // 64) * 64
    Kw = -(-(-(-K // d) * d) // 64) * 64
    for blk in (0, 256):
        if K % max(blk, 1):
            continue
        tc = L.lq_gemm_route_workspace_bytes(batch, K, N, d, D, blk, lq.ROUTE_GEMM_TC)
        assert tc == 256 + _r256(batch * Lp * 2 + batch * 4)
        dq = L.lq_gemm_route_workspace_bytes(batch, K, N, d, D, blk, lq.ROUTE_GEMM_DQ)
        assert dq == 256 + _r256(N * Kw * 2 + batch * Kw * 2 + batch * 4)
        route = lq.gemm_route(batch, K, N, d, D, blk)
        assert route in (lq.ROUTE_GEMM_TC, lq.ROUTE_GEMM_DQ)
        assert lq.gemm_workspace_bytes(batch, K, N, d, D) >= (tc if route == lq.ROUTE_GEMM_TC
                                                              else dq)


def _ptr(v):
    return ctypes.c_void_p(v)


def test_argument_checks_without_gpu(L):
    fake = _ptr(0x10000)       # aligned, never dereferenced: every call below is rejected
    odd = _ptr(0x10004)
    S = None
    assert L.lq_pack(None, 4, 16, 2, 4, fake, S) == lq.LQ_EINVAL
    assert L.lq_pack(fake, 4, 16, 2, 4, odd, S) == lq.LQ_EINVAL      # packed misaligned
    assert L.lq_pack(fake, -1, 16, 2, 4, fake, S) == lq.LQ_EINVAL
    assert L.lq_pack(fake, 0, 16, 2, 4, fake, S) == lq.LQ_OK         # N = 0: no work
    assert L.lq_pack(fake, 4, 16, 5, 4, fake, S) == lq.LQ_EINVAL     # D < d
    assert "D" in L.lq_last_error().decode() or "invalid" in L.lq_last_error().decode()
    assert L.lq_unpack(fake, 4, 16, 2, 40, fake, S) == lq.LQ_EINVAL  # D > 32

    bad = lq.WhitenDesc(None, None, 3)
    assert L.lq_whiten(fake, 0, 2, 12, ctypes.byref(bad), fake, S) == lq.LQ_EINVAL
    big = lq.WhitenDesc(None, None, 8192)
    assert L.lq_whiten(fake, 0, 1, 8192, ctypes.byref(big), fake, S) == lq.LQ_EUNSUPPORTED
    nodiv = lq.WhitenDesc(None, None, 256)
    assert L.lq_whiten(fake, 0, 1, 300, ctypes.byref(nodiv), fake, S) == lq.LQ_EINVAL
    assert L.lq_whiten(fake, 7, 1, 256, None, fake, S) == lq.LQ_EINVAL   # unknown dtype

    args = dict(x=fake, xdt=2, batch=1, T=None, packed=fake, M=fake, s=fake, sdt=1, d=10, D=24,
                K=4096, N=4096, y=fake, ws=fake, wsb=1 << 30)

    def gemm(**kw):
        a = dict(args, **kw)
        return L.lq_gemm(a["x"], a["xdt"], a["batch"], a["T"], a["packed"], a["M"], a["s"],
                         a["sdt"], a["d"], a["D"], a["K"], a["N"], a["y"], a["ws"], a["wsb"], S)

    assert gemm(batch=0) == lq.LQ_EINVAL
    assert gemm(N=0) == lq.LQ_EINVAL
    assert gemm(packed=None) == lq.LQ_EINVAL
    assert gemm(packed=_ptr(0x10008)) == lq.LQ_EINVAL
    assert gemm(ws=_ptr(0x10010)) == lq.LQ_EINVAL                      # not 256-aligned
    assert gemm(wsb=16) == lq.LQ_EINVAL
    assert "workspace" in L.lq_last_error().decode()
    assert gemm(T=ctypes.byref(lq.WhitenDesc(None, None, 3000))) == lq.LQ_EINVAL
    assert gemm(x=_ptr(0x10001)) == lq.LQ_EINVAL                       # bf16 x misaligned
    assert gemm(D=8) == lq.LQ_EINVAL
    code = ctypes.c_int32(0)
    assert L.lq_device_status(None, ctypes.byref(code), S) == lq.LQ_EINVAL
    for st in range(6):
        assert L.lq_status_string(st)


def test_routes_without_gpu(L):
    """The host-side route query names the kernel family each shape runs on."""
    # one or two tokens on a layer of >= 32 MB of codes: the TMA-staged GEMV; else the
    # register-streamed one up to 8 tokens
    assert lq.gemm_route(1, 8192, 28672, 10, 24, 256) == lq.ROUTE_GEMV_BULK
    assert lq.gemm_route(2, 28672, 8192, 10, 24, 256) == lq.ROUTE_GEMV_BULK
    assert lq.gemm_route(3, 8192, 28672, 10, 24, 256) == lq.ROUTE_GEMV_I8
    assert lq.gemm_route(1, 4096, 4096, 10, 24, 256) == lq.ROUTE_GEMV_I8
    assert lq.gemm_route(2048, 8192, 28672, 10, 24, 256) == lq.ROUTE_GEMM_DQ
    assert lq.gemm_route(64, 8192, 28672, 10, 24, 256) == lq.ROUTE_GEMM_TC
    assert lq.gemm_route(2, 8192, 300, 10, 24, 4096) == lq.ROUTE_GEMV_I8     # block > 256
    assert lq.gemm_route(8, 4096, 513, 10, 24, 4096) == lq.ROUTE_GEMV_GROUPS
    assert lq.gemm_route(1, 1048570, 4096, 10, 24, 0) == lq.ROUTE_NONE
    assert lq.gemm_route(0, 8192, 28672, 10, 24, 256) == -1
    assert lq.gemm_route(1, 8192, 28672, 10, 24, 3) == -1
    assert lq.gemm_launches(1, 8192, 28672, 10, 24, 256) == 2
    assert lq.gemm_launches(1, 1048570, 4096, 10, 24, 0) == 0


def test_gemm_rejects_shapes_no_plan_fits_without_gpu(L):
    fake = ctypes.c_void_p(0x10000)     # never dereferenced: the call is rejected first
    K, N = 1048570, 4096
    ws = lq.gemm_workspace_bytes(1, K, N, 10, 24)
    assert ws > 0
    rc = L.lq_gemm(fake, lq.LQ_BF16, 1, None, fake, fake, fake, lq.LQ_F16, 10, 24, K, N, fake,
                   ctypes.c_void_p(0x100000), ws, None)
    assert rc == lq.LQ_EUNSUPPORTED
    assert "no GEMV or GEMM plan" in L.lq_last_error().decode()


def test_route_workspace_without_gpu(L):
    """Every route that fits a shape reports its own workspace; a route that does not fit, 0."""
    args = (2048, 8192, 28672, 10, 24, 256)
    dq = L.lq_gemm_route_workspace_bytes(*args, lq.ROUTE_GEMM_DQ)
    tc = L.lq_gemm_route_workspace_bytes(*args, lq.ROUTE_GEMM_TC)
    assert dq >= 28672 * 8256 * 2 and 0 < tc < dq     # fp16 W is the bulk of the first
    assert L.lq_gemm_route_workspace_bytes(*args, lq.ROUTE_GEMV_BULK) == 0    # batch > 8
    assert L.lq_gemm_route_workspace_bytes(*args, lq.ROUTE_NONE) == 0
    assert L.lq_gemm_route_workspace_bytes(1, 8192, 28672, 10, 24, 256, lq.ROUTE_GEMV_I8) > 0
    fake = ctypes.c_void_p(0x10000)
    rc = L.lq_gemm_on_route(fake, lq.LQ_BF16, 1, None, fake, fake, fake, lq.LQ_F16, 10, 24, 8192,
                            28672, fake, ctypes.c_void_p(0x100000), 1 << 30, 9, None)
    assert rc == lq.LQ_EINVAL and "route" in L.lq_last_error().decode()
    rc = L.lq_gemm_on_route(fake, lq.LQ_BF16, 9, None, fake, fake, fake, lq.LQ_F16, 10, 24, 8192,
                            28672, fake, ctypes.c_void_p(0x100000), 1 << 30, lq.ROUTE_GEMV_BULK,
                            None)
    assert rc == lq.LQ_EUNSUPPORTED
