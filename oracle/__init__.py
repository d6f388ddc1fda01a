"""fp64 CPU oracle for the LiftQuant decode operator (argument marshalling only).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline may import this package. The arithmetic lives in lq_oracle.c; this
module converts numpy arrays to fp64/int8/uint8 buffers and calls it.

Functions follow "LiftQuant: Continuous Bit-Width LLM Quantization via
Dimensional Lifting and Projection" (sec. 3.1: w ~= M w_q; sec. 3 intro: the
fused operator o = diag(s) W (M T a)) and the romaanj.github.io review
("Method": T is Hadamard mixing plus scalings; decode is diag(s) W_q (T* a)).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_i8p = ctypes.POINTER(ctypes.c_int8)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_dp = ctypes.POINTER(ctypes.c_double)


def _load(path=None):
    lib = ctypes.CDLL(path or _build.build())
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    lib.orc_lifted_bits.argtypes = [i32, i32, i32]
    lib.orc_lifted_bits.restype = i64
    lib.orc_row_bytes.argtypes = [i32, i32, i32]
    lib.orc_row_bytes.restype = i64
    lib.orc_pack.argtypes = [_i8p, i64, i32, i32, i32, _u8p]
    lib.orc_pack.restype = ctypes.c_int
    lib.orc_unpack.argtypes = [_u8p, i64, i32, i32, i32, _i8p]
    lib.orc_unpack.restype = ctypes.c_int
    lib.orc_whiten.argtypes = [_dp, i64, i32, _i8p, _dp, i32, _dp]
    lib.orc_whiten.restype = ctypes.c_int
    lib.orc_lift.argtypes = [_dp, i64, i32, _i8p, _dp, i32, _dp, i32, i32, _dp]
    lib.orc_lift.restype = ctypes.c_int
    fwd = [_dp, i64, i32, i64, i32, i32, _u8p, _dp, _dp, _i8p, _dp, i32, _dp, ctypes.c_int]
    lib.orc_forward.argtypes = fwd
    lib.orc_forward.restype = ctypes.c_int
    lib.orc_forward_lifted.argtypes = fwd
    lib.orc_forward_lifted.restype = ctypes.c_int
    lib.orc_encode_bruteforce.argtypes = [_dp, _dp, i32, i32, _i8p]
    lib.orc_encode_bruteforce.restype = i64
    lib.orc_encode_seeded.argtypes = [_dp, _dp, i32, i32, _i8p, _dp]
    lib.orc_encode_seeded.restype = i64
    lib.orc_encode_rows.argtypes = [_dp, i64, i32, _dp, i32, i32, i32, _i8p, _dp, ctypes.c_int]
    lib.orc_encode_rows.restype = ctypes.c_int
    lib.orc_codebook_round.argtypes = [_dp, i64, _dp, i32, i32, i32, _i8p, ctypes.c_int]
    lib.orc_codebook_round.restype = ctypes.c_double
    lib.orc_codebook_refit.argtypes = [_dp, i64, _i8p, _dp, i32, i32]
    lib.orc_codebook_refit.restype = ctypes.c_int
    lib.orc_max_threads.argtypes = []
    lib.orc_max_threads.restype = ctypes.c_int
    return lib


def lib():
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


class Oracle:
    """The same functions bound to an explicit library file (used for mutants)."""

    def __init__(self, path):
        self._lib = _load(path)

    def __getattr__(self, name):
        fn = globals()[name]
        return lambda *a, **k: fn(*a, _lib=self._lib, **k)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, t):
    return a.ctypes.data_as(t)


def _opt_i8(a):
    if a is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int8))
    return a, _ptr(a, _i8p)


def _opt_f64(a):
    if a is None:
        return None, None
    a = _f64(a)
    return a, _ptr(a, _dp)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def lifted_bits(K, d, D, _lib=None):
    """G*D with G = ceil(K/d): stored bits per row."""
    return int((_lib or lib()).orc_lifted_bits(K, d, D))


def row_bytes(K, d, D, _lib=None):
    """Stored bytes per row: the bits rounded up to a multiple of 16 bytes."""
    return int((_lib or lib()).orc_row_bytes(K, d, D))


def pack(b, K, d, D, _lib=None):
    """b: [N][G*D] int8 of +1/-1 -> [N][row_bytes] uint8 (LQ_FORMAT_V1)."""
    L = _lib or lib()
    b = np.ascontiguousarray(np.asarray(b, dtype=np.int8))
    N = b.shape[0]
    assert b.shape[1] == lifted_bits(K, d, D, _lib=L)
    out = np.zeros((N, row_bytes(K, d, D, _lib=L)), dtype=np.uint8)
    _check(L.orc_pack(_ptr(b, _i8p), N, K, d, D, _ptr(out, _u8p)), "pack")
    return out


def unpack(packed, K, d, D, _lib=None):
    """[N][row_bytes] uint8 -> [N][G*D] int8 of +1/-1."""
    L = _lib or lib()
    p = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    N = p.shape[0]
    out = np.zeros((N, lifted_bits(K, d, D, _lib=L)), dtype=np.int8)
    _check(L.orc_unpack(_ptr(p, _u8p), N, K, d, D, _ptr(out, _i8p)), "unpack")
    return out


def whiten(x, sign=None, chan_scale=None, block=0, _lib=None):
    """x: [batch][K] -> T(x) in fp64."""
    L = _lib or lib()
    x = _f64(np.atleast_2d(x))
    batch, K = x.shape
    sg, sgp = _opt_i8(sign)
    cs, csp = _opt_f64(chan_scale)
    out = np.zeros_like(x)
    _check(L.orc_whiten(_ptr(x, _dp), batch, K, sgp, csp, block, _ptr(out, _dp)), "whiten")
    return out


def lift(x, M, d, D, sign=None, chan_scale=None, block=0, _lib=None):
    """x: [batch][K] -> z: [batch][G*D], z = blockwise M^T applied to T(x)."""
    L = _lib or lib()
    x = _f64(np.atleast_2d(x))
    batch, K = x.shape
    Mf = _f64(M).reshape(d, D)
    sg, sgp = _opt_i8(sign)
    cs, csp = _opt_f64(chan_scale)
    out = np.zeros((batch, lifted_bits(K, d, D, _lib=L)), dtype=np.float64)
    _check(L.orc_lift(_ptr(x, _dp), batch, K, sgp, csp, block, _ptr(Mf, _dp), d, D,
                      _ptr(out, _dp)), "lift")
    return out


def _forward(fn, x, packed, M, s, d, D, sign, chan_scale, block, nthreads, _lib):
    L = _lib or lib()
    x = _f64(np.atleast_2d(x))
    batch, K = x.shape
    p = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    nrows = p.shape[0]
    assert p.shape[1] == row_bytes(K, d, D, _lib=L)
    Mf = _f64(M).reshape(d, D)
    sf = _f64(s).reshape(nrows)
    sg, sgp = _opt_i8(sign)
    cs, csp = _opt_f64(chan_scale)
    y = np.zeros((batch, nrows), dtype=np.float64)
    rc = getattr(L, fn)(_ptr(x, _dp), batch, K, nrows, d, D, _ptr(p, _u8p), _ptr(Mf, _dp),
                        _ptr(sf, _dp), sgp, csp, block, _ptr(y, _dp), int(nthreads))
    _check(rc, fn)
    return y


def forward(x, packed, M, s, d, D, sign=None, chan_scale=None, block=0, nthreads=1, _lib=None):
    """y[t][n] = s[n] * (W[n] . T(x[t])) with W formed explicitly from the packed rows.

    x: [batch][K]; packed: [nrows][row_bytes] uint8 (any subset of a layer's rows);
    s: [nrows]. Returns y: [batch][nrows] fp64.
    """
    return _forward("orc_forward", x, packed, M, s, d, D, sign, chan_scale, block, nthreads,
                    _lib)


def forward_lifted(x, packed, M, s, d, D, sign=None, chan_scale=None, block=0, nthreads=1,
                   _lib=None):
    """The same operator computed as s . (b . z) with z = lift(x)."""
    return _forward("orc_forward_lifted", x, packed, M, s, d, D, sign, chan_scale, block,
                    nthreads, _lib)


def encode_bruteforce(w, M, d, D, _lib=None):
    """argmin_b ||w - M b||^2 over all 2^D sign vectors; returns (b int8[D], index)."""
    L = _lib or lib()
    wf = _f64(w).reshape(d)
    Mf = _f64(M).reshape(d, D)
    out = np.zeros(D, dtype=np.int8)
    c = L.orc_encode_bruteforce(_ptr(wf, _dp), _ptr(Mf, _dp), d, D, _ptr(out, _i8p))
    if c < 0:
        raise ValueError("oracle encode rejected its arguments")
    return out, int(c)


def encode_seeded(w, M, d, D, _lib=None):
    """Seeded search (first d coordinates solved, the other D - d enumerated); returns
    (b int8[D], index f, squared distance)."""
    L = _lib or lib()
    wf = _f64(w).reshape(d)
    Mf = _f64(M).reshape(d, D)
    out = np.zeros(D, dtype=np.int8)
    dist = ctypes.c_double(0.0)
    f = L.orc_encode_seeded(_ptr(wf, _dp), _ptr(Mf, _dp), d, D, _ptr(out, _i8p), ctypes.byref(dist))
    if f < 0:
        raise ValueError("oracle seeded encode rejected its arguments")
    return out, int(f), float(dist.value)


def encode_rows(w, M, d, D, mode, nthreads=0, _lib=None):
    """Encodes w [N][K] block by block: (b int8 [N][G][D], err float64 [N][G]).
    mode 0: exhaustive 2^D search; mode 1: seeded 2^(D-d) search."""
    L = _lib or lib()
    wf = _f64(w)
    N, K = wf.shape
    G = -(-K // d)
    Mf = _f64(M).reshape(d, D)
    b = np.zeros((N, G, D), dtype=np.int8)
    err = np.zeros((N, G), dtype=np.float64)
    rc = L.orc_encode_rows(_ptr(wf, _dp), N, K, _ptr(Mf, _dp), d, D, mode, _ptr(b, _i8p),
                           _ptr(err, _dp), nthreads)
    if rc != 0:
        raise ValueError("oracle encode_rows rejected its arguments")
    return b, err


def codebook_round(w, M, d, D, mode=0, nthreads=0, _lib=None):
    """One round of the codebook fit on samples w [S][d]: nearest codewords under M, then the
    least-squares M. Returns (M_new [d][D], codes int8 [S][D], mse per weight before the
    update)."""
    L = _lib or lib()
    wf = _f64(w).reshape(-1, d)
    Mf = _f64(M).reshape(d, D).copy()
    b = np.zeros((wf.shape[0], D), dtype=np.int8)
    mse = L.orc_codebook_round(_ptr(wf, _dp), wf.shape[0], _ptr(Mf, _dp), d, D, mode,
                               _ptr(b, _i8p), nthreads)
    if mse < 0:
        raise ValueError("oracle codebook_round rejected its arguments")
    return Mf, b, float(mse)


def codebook_refit(w, b, M, d, D, _lib=None):
    """The least-squares step of the codebook fit alone: M = (sum w b^T)(sum b b^T)^-1 for the
    samples w [S][d] and their codes b [S][D] (+-1). Returns M_new [d][D] (M gives its shape
    and is not modified)."""
    L = _lib or lib()
    wf = _f64(w).reshape(-1, d)
    bb = np.ascontiguousarray(b, dtype=np.int8).reshape(wf.shape[0], D)
    Mf = _f64(M).reshape(d, D).copy()
    if L.orc_codebook_refit(_ptr(wf, _dp), wf.shape[0], _ptr(bb, _i8p), _ptr(Mf, _dp), d, D) != 0:
        raise ValueError("oracle codebook_refit rejected its arguments (or sum b b^T is singular)")
    return Mf


def max_threads(_lib=None):
    return int((_lib or lib()).orc_max_threads())
