"""Python binding of liblq, the B200 LiftQuant decode library (argument marshalling only).

Every function here checks tensor placement and dtypes, then calls the extern "C"
entry point of the same name in liblq.so (declared in include/liblq.h). All
arithmetic runs in the library's CUDA kernels; torch only supplies device memory
and the current stream. There is no CPU fallback: if liblq.so has not been built,
the first call raises.
"""
import ctypes
import os

import torch

__all__ = [
    "LQError", "lib", "abi_version", "lifted_bits", "row_stride_bytes", "pack", "unpack",
    "whiten", "lift", "gemm_workspace_bytes", "gemm_launches", "gemm", "gemm_noalloc",
    "new_workspace",
    "device_status", "check_wait_timeout", "NOALLOC_SCRATCH_BYTES",
]

NOALLOC_SCRATCH_BYTES = 8 << 20   # LQ_NOALLOC_SCRATCH_BYTES

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblq.so")

LQ_OK, LQ_EINVAL, LQ_EUNSUPPORTED, LQ_ECUDA, LQ_ETIMEOUT, LQ_EDEVICE = range(6)
LQ_F32, LQ_F16, LQ_BF16 = 0, 1, 2
_DTYPES = {torch.float32: LQ_F32, torch.float16: LQ_F16, torch.bfloat16: LQ_BF16}

EXPORTS = ("lq_abi_version", "lq_lifted_bits", "lq_row_stride_bytes", "lq_pack", "lq_unpack", "lq_encode",
           "lq_whiten", "lq_lift", "lq_gemm_workspace_bytes", "lq_gemm_launches", "lq_gemm_route",
           "lq_gemm", "lq_gemm_on_route", "lq_gemm_route_workspace_bytes", "lq_gemv_staged_plan",
           "lq_codebook_workspace_bytes", "lq_codebook_round",
           "lq_gemm_noalloc", "lq_check_wait_timeout",
           "lq_device_status", "lq_status_string", "lq_last_error")


class LQError(RuntimeError):
    def __init__(self, status, where, message):
        self.status = status
        super().__init__(f"{where}: status {status}: {message}")


class WhitenDesc(ctypes.Structure):
    _fields_ = [("sign", ctypes.c_void_p), ("chan_scale", ctypes.c_void_p),
                ("block", ctypes.c_int32)]


_LIB = None


def _declare(L):
    i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    dp = ctypes.POINTER(WhitenDesc)
    sig = {
        "lq_abi_version": ([], i32),
        "lq_lifted_bits": ([i32, i32, i32], i64),
        "lq_row_stride_bytes": ([i32, i32, i32], i64),
        "lq_pack": ([vp, i32, i32, i32, i32, vp, vp], ctypes.c_int),
        "lq_encode": ([vp, i32, i32, vp, i32, i32, i32, vp, vp, vp], ctypes.c_int),
        "lq_unpack": ([vp, i32, i32, i32, i32, vp, vp], ctypes.c_int),
        "lq_whiten": ([vp, ctypes.c_int, i32, i32, dp, vp, vp], ctypes.c_int),
        "lq_lift": ([vp, ctypes.c_int, i32, i32, dp, vp, i32, i32, vp, vp], ctypes.c_int),
        "lq_gemm_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
        "lq_gemm_launches": ([i32, i32, i32, i32, i32, i32], i32),
        "lq_gemm_route": ([i32, i32, i32, i32, i32, i32], i32),
        "lq_gemm": ([vp, ctypes.c_int, i32, dp, vp, vp, vp, ctypes.c_int, i32, i32, i32, i32, vp,
                     vp, sz, vp], ctypes.c_int),
        "lq_gemm_on_route": ([vp, ctypes.c_int, i32, dp, vp, vp, vp, ctypes.c_int, i32, i32, i32,
                              i32, vp, vp, sz, i32, vp], ctypes.c_int),
        "lq_gemm_route_workspace_bytes": ([i32, i32, i32, i32, i32, i32, i32], sz),
        "lq_gemv_staged_plan": ([i32, i32, i32, i32, i32, i32, ctypes.POINTER(i64)], ctypes.c_int),
        "lq_codebook_workspace_bytes": ([ctypes.c_int64, i32, i32], sz),
        "lq_codebook_round": ([vp, ctypes.c_int64, vp, i32, i32, i32, vp, vp, vp, sz, vp],
                              ctypes.c_int),
        "lq_gemm_noalloc": ([vp, ctypes.c_int, i32, dp, vp, vp, vp, ctypes.c_int, i32, i32, i32,
                             i32, vp, vp], ctypes.c_int),
        "lq_device_status": ([vp, ctypes.POINTER(i32), vp], ctypes.c_int),
        "lq_check_wait_timeout": ([vp, i32, vp], ctypes.c_int),
        "lq_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "lq_last_error": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


def lib():
    """The loaded liblq.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m fractional_bit_weight_b200.build` (nvcc, sm_100a)")
        _LIB = _declare(ctypes.CDLL(LIB_PATH))
    return _LIB


def _check(rc, where):
    if rc != LQ_OK:
        msg = lib().lq_last_error().decode() or lib().lq_status_string(rc).decode()
        raise LQError(rc, where, msg)


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, dtypes=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return ctypes.c_void_p(t.data_ptr())


def _opt(t, name, dtypes):
    return None if t is None else _dev(t, name, dtypes)


def _whiten_desc(sign, chan_scale, block):
    if not block:
        return None
    sg = _opt(sign, "sign", (torch.int8,))
    cs = _opt(chan_scale, "chan_scale", (torch.float32,))
    return WhitenDesc(sg.value if sg is not None else None,
                      cs.value if cs is not None else None, int(block))


def _desc_ptr(desc):
    return None if desc is None else ctypes.byref(desc)


def abi_version():
    return int(lib().lq_abi_version())


def lifted_bits(K, d, D):
    return int(lib().lq_lifted_bits(K, d, D))


def row_stride_bytes(K, d, D):
    return int(lib().lq_row_stride_bytes(K, d, D))


def pack(b_pm1, K, d, D, out=None, stream=None):
    """int8 sign codes [N][ceil(K/d)*D] -> LQ_FORMAT_V1 rows as int32 [N][row_stride/4]."""
    N = b_pm1.shape[0]
    if out is None:
        out = torch.empty((N, row_stride_bytes(K, d, D) // 4), dtype=torch.int32,
                          device=b_pm1.device)
    _check(lib().lq_pack(_dev(b_pm1, "b_pm1", (torch.int8,)), N, K, d, D,
                         _dev(out, "packed", (torch.int32,)), _stream(stream)), "lq_pack")
    return out


LQ_ENCODE_EXACT, LQ_ENCODE_SEEDED = 0, 1


def encode(w, M, d, D, mode=LQ_ENCODE_SEEDED, with_err=True, stream=None):
    """Nearest-codeword codes of w [N][K] fp32 (see lq_encode): returns (b_pm1 int8
    [N][ceil(K/d)][D], err fp32 [N][ceil(K/d)] or None). Pack b_pm1.view(N, -1) with pack()."""
    N, K = w.shape
    G = -(-K // d)
    b = torch.empty((N, G, D), dtype=torch.int8, device=w.device)
    err = torch.empty((N, G), dtype=torch.float32, device=w.device) if with_err else None
    _check(lib().lq_encode(_dev(w, "w", (torch.float32,)), N, K, _dev(M, "M", (torch.float32,)),
                           d, D, int(mode), _dev(b, "b_pm1", (torch.int8,)),
                           _dev(err, "err", (torch.float32,)) if with_err else None,
                           _stream(stream)), "lq_encode")
    return b, err


def unpack(packed, K, d, D, out=None, stream=None):
    N = packed.shape[0]
    if out is None:
        out = torch.empty((N, lifted_bits(K, d, D)), dtype=torch.int8, device=packed.device)
    _check(lib().lq_unpack(_dev(packed, "packed", (torch.int32,)), N, K, d, D,
                           _dev(out, "b_pm1", (torch.int8,)), _stream(stream)), "lq_unpack")
    return out


def whiten(x, sign=None, chan_scale=None, block=0, out=None, stream=None):
    batch, K = x.shape
    if out is None:
        out = torch.empty((batch, K), dtype=torch.float32, device=x.device)
    desc = _whiten_desc(sign, chan_scale, block)
    _check(lib().lq_whiten(_dev(x, "x", _DTYPES), _DTYPES[x.dtype], batch, K, _desc_ptr(desc),
                           _dev(out, "xt", (torch.float32,)), _stream(stream)), "lq_whiten")
    return out


def lift(x, M, d, D, sign=None, chan_scale=None, block=0, out=None, stream=None):
    batch, K = x.shape
    if out is None:
        out = torch.empty((batch, lifted_bits(K, d, D)), dtype=torch.float32, device=x.device)
    desc = _whiten_desc(sign, chan_scale, block)
    _check(lib().lq_lift(_dev(x, "x", _DTYPES), _DTYPES[x.dtype], batch, K, _desc_ptr(desc),
                         _dev(M, "M", (torch.float32,)), d, D, _dev(out, "z", (torch.float32,)),
                         _stream(stream)), "lq_lift")
    return out


def gemm_workspace_bytes(batch, K, N, d, D):
    return int(lib().lq_gemm_workspace_bytes(batch, K, N, d, D))


STAGED_PLAN_FIELDS = ("ok", "S", "sc", "R", "rq", "rrem", "rows_per_stage", "wch", "NS", "nchunk",
                      "smem", "prep_smem")


def gemv_staged_plan(batch, K, N, d, D, block=0):
    """The TMA-staged GEMV's plan for a shape (host-only query), as a dict."""
    out = (ctypes.c_int64 * len(STAGED_PLAN_FIELDS))()
    _check(lib().lq_gemv_staged_plan(batch, K, N, d, D, block, out), "lq_gemv_staged_plan")
    return dict(zip(STAGED_PLAN_FIELDS, (int(v) for v in out)))


def gemm_launches(batch, K, N, d, D, block=0):
    """Kernels one lq_gemm call launches for this shape (host-only query)."""
    return int(lib().lq_gemm_launches(batch, K, N, d, D, block))


# lq_gemm_route codes (include/liblq.h)
ROUTE_GEMV_I8, ROUTE_NONE, ROUTE_GEMM_TC, ROUTE_GEMV_GROUPS, ROUTE_GEMV_BULK, ROUTE_GEMM_DQ = \
    0, 1, 2, 3, 4, 5


def gemm_route(batch, K, N, d, D, block=0):
    """Which kernels lq_gemm runs for this shape (host-only query; ROUTE_* codes)."""
    return int(lib().lq_gemm_route(batch, K, N, d, D, block))


def new_workspace(batch, K, N, d, D, device="cuda", block=0, route=None):
    """A zero-filled workspace tensor for lq_gemm (uint8, 256-byte aligned by torch); with a
    route, for lq_gemm_on_route on that route and Hadamard block."""
    if route is None:
        n = gemm_workspace_bytes(batch, K, N, d, D)
    else:
        n = int(lib().lq_gemm_route_workspace_bytes(batch, K, N, d, D, block, int(route)))
    if n == 0:
        raise ValueError("invalid sizes for lq_gemm")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gemm(x, packed, M, s, d, D, sign=None, chan_scale=None, block=0, y=None, workspace=None,
         stream=None, route=None):
    """y[t][n] = s[n] * (W[n] . T(x[t])), float32 [batch][N].

    route=None lets the library pick the kernels (lq_gemm); a ROUTE_* code runs that route
    (lq_gemm_on_route), which must fit the shape."""
    batch, K = x.shape
    N = packed.shape[0]
    if y is None:
        y = torch.empty((batch, N), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = new_workspace(batch, K, N, d, D, device=x.device, block=block, route=route)
    desc = _whiten_desc(sign, chan_scale, block)
    args = (_dev(x, "x", _DTYPES), _DTYPES[x.dtype], batch, _desc_ptr(desc),
            _dev(packed, "packed", (torch.int32,)), _dev(M, "M", (torch.float32,)),
            _dev(s, "s", _DTYPES), _DTYPES[s.dtype], d, D, K, N,
            _dev(y, "y", (torch.float32,)), _dev(workspace, "workspace"),
            workspace.numel() * workspace.element_size())
    if route is None:
        _check(lib().lq_gemm(*args, _stream(stream)), "lq_gemm")
    else:
        _check(lib().lq_gemm_on_route(*args, int(route), _stream(stream)), "lq_gemm_on_route")
    return y


def gemm_noalloc(x, packed, M, s, d, D, sign=None, chan_scale=None, block=0, y=None,
                 stream=None):
    """lq_gemm without a workspace: the library's own fixed device scratch is used (batch 1..8).

    For callers that cannot allocate device memory. The first call on a device sets it up and
    should come before any stream capture; calls that overlap on the GPU share the scratch and
    must be serialised by the caller.
    """
    batch, K = x.shape
    N = packed.shape[0]
    if y is None:
        y = torch.empty((batch, N), dtype=torch.float32, device=x.device)
    desc = _whiten_desc(sign, chan_scale, block)
    _check(lib().lq_gemm_noalloc(_dev(x, "x", _DTYPES), _DTYPES[x.dtype], batch, _desc_ptr(desc),
                                 _dev(packed, "packed", (torch.int32,)),
                                 _dev(M, "M", (torch.float32,)), _dev(s, "s", _DTYPES),
                                 _DTYPES[s.dtype], d, D, K, N, _dev(y, "y", (torch.float32,)),
                                 _stream(stream)), "lq_gemm_noalloc")
    return y


def codebook_round(w, M, d, D, mode=0, b=None, mse=None, workspace=None, stream=None):
    """One round of the codebook fit on samples w [S][d] (fp32, device): nearest codewords
    under M, then the least-squares M. M (fp32 [d][D], device) is updated in place. Returns
    (M, codes int8 [S][D], mse fp64 tensor of one element) on the device."""
    S = w.shape[0]
    if b is None:
        b = torch.empty((S, D), dtype=torch.int8, device=w.device)
    if mse is None:
        mse = torch.empty(1, dtype=torch.float64, device=w.device)
    if workspace is None:
        n = int(lib().lq_codebook_workspace_bytes(S, d, D))
        if n == 0:
            raise ValueError("invalid sizes for lq_codebook_round")
        workspace = torch.empty(n, dtype=torch.uint8, device=w.device)
    _check(lib().lq_codebook_round(_dev(w, "w", (torch.float32,)), S,
                                   _dev(M, "M", (torch.float32,)), d, D, int(mode),
                                   _dev(b, "b", (torch.int8,)), _dev(mse, "mse", (torch.float64,)),
                                   _dev(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "lq_codebook_round")
    return M, b, mse


def check_wait_timeout(workspace, limit_ms=20, stream=None):
    """Runs the device-side timeout check (see lq_check_wait_timeout); read the result with
    device_status(workspace)."""
    _check(lib().lq_check_wait_timeout(_dev(workspace, "workspace"), int(limit_ms),
                                       _stream(stream)), "lq_check_wait_timeout")


def device_status(workspace, stream=None):
    code = ctypes.c_int32(0)
    rc = lib().lq_device_status(_dev(workspace, "workspace"), ctypes.byref(code), _stream(stream))
    return int(rc), int(code.value)
