"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each pin takes an oracle object (the `oracle` module, or a deliberately broken
copy built by the mutation test) and raises AssertionError when the oracle
disagrees with something other than itself: values printed on the pages,
hand-derived golden fixtures, a textbook routine (scipy's Sylvester Hadamard,
numpy matmul), a closed form, or a pure-Python brute force on tiny inputs.
"""
import itertools
import math
import os

import numpy as np
import scipy.linalg

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _signs(rng, shape):
    return (1 - 2 * rng.integers(0, 2, size=shape)).astype(np.int8)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- bit-width (T1)

def pin_bitwidth_printed(orc):
    """Rate D/d for every (d, D) printed on the pages (Fig. 2; LQ-a/b names)."""
    for d, D, printed in _read_golden("bitwidths.txt"):
        d, D, printed = int(d), int(D), float(printed)
        K = 8192 * d                      # a multiple of d: no padding
        bits = orc.lifted_bits(K, d, D)
        assert bits == K // d * D, (d, D, bits)
        assert abs(bits / K - printed) < 0.005 + 1e-12, (d, D, bits / K, printed)
        assert bits * 10 == K * 10 // d * D


def pin_bitwidth_padding(orc):
    """K not a multiple of d is zero-padded to ceil(K/d) blocks; rows pad to 16 bytes."""
    for K, d, D in [(4096, 10, 24), (8192, 3, 8), (28672, 10, 24), (7, 3, 5), (1, 1, 1)]:
        G = -(-K // d)
        assert orc.lifted_bits(K, d, D) == G * D
        rb = orc.row_bytes(K, d, D)
        assert rb % 16 == 0 and rb * 8 >= G * D and (rb - 16) * 8 < G * D
    # the workloads' packed row sizes
    assert orc.row_bytes(4096, 10, 24) == 1232
    assert orc.row_bytes(8192, 10, 24) == 2464
    assert orc.row_bytes(28672, 10, 24) == 8608
    assert orc.row_bytes(256, 2, 5) == 80


def pin_memory_fit(orc):
    """Memory-fit figures of the pages: 70B at 2.4 bit fits 24 GB, 32B at 2.5 bit fits 12 GB
    (paper, abstract and sec. 1). Bits per weight come from the oracle's stored row length."""
    for params, d, D, budget in [(70e9, 10, 24, 24e9), (32e9, 2, 5, 12e9)]:
        K = 8192 * d
        bpw = orc.lifted_bits(K, d, D) / K
        assert params * bpw / 8 < budget
    # 70B: 3 bit (LQ-24/8) does not fit 24 GB, 2 bit (LQ-32/16) does (paper, sec. 1)
    K = 8192 * 8
    assert 70e9 * orc.lifted_bits(K, 8, 24) / K / 8 > 24e9
    K = 8192 * 16
    assert 70e9 * orc.lifted_bits(K, 16, 32) / K / 8 < 24e9


# ---------------------------------------------------------------- packing

def pin_pack_golden(orc):
    rows = _read_golden("pack_example.txt")
    K, d, D = (int(r[1]) for r in rows[:3])
    bs = [np.array([int(v) for v in r[1:]], np.int8) for r in rows if r[0] == "b"]
    by = [np.array([int(v, 16) for v in r[1:]], np.uint8) for r in rows if r[0] == "bytes"]
    b = np.stack(bs)
    expect = np.stack(by)
    got = orc.pack(b, K, d, D)
    assert got.shape == expect.shape, (got.shape, expect.shape)
    assert np.array_equal(got, expect), (got, expect)
    assert np.array_equal(orc.unpack(expect, K, d, D), b)
    # the same bytes read as little-endian uint32 words: bit q in word q//32, position q%32
    words = expect.view("<u4")
    for n in range(b.shape[0]):
        for q in range(b.shape[1]):
            assert ((int(words[n, q // 32]) >> (q % 32)) & 1) == (b[n, q] == -1)


def pin_pack_exhaustive(orc):
    """All 2^D codewords round-trip exactly for D <= 8, for several block counts."""
    for d, D in [(1, 2), (2, 4), (2, 5), (3, 8)]:
        for G in (1, 3, 7):
            K = G * d
            C = np.array([[(-1 if (c >> j) & 1 else 1) for j in range(D)]
                          for c in range(1 << D)], np.int8)
            b = np.tile(C, (1, G))                       # row c: codeword c in every block
            p = orc.pack(b, K, d, D)
            assert np.array_equal(orc.unpack(p, K, d, D), b)
            # codeword c occupies bits g*D .. g*D+D-1 as the binary digits of c
            for c in range(1 << D):
                val = int.from_bytes(p[c].tobytes(), "little")
                for g in range(G):
                    assert (val >> (g * D)) & ((1 << D) - 1) == c
                assert val >> (G * D) == 0                 # padding is zero


def pin_pack_random(orc):
    rng = _rng(11)
    for K, d, D in [(37, 3, 8), (100, 10, 24), (64, 4, 12), (5, 1, 2), (300, 10, 25)]:
        G = -(-K // d)
        b = _signs(rng, (9, G * D))
        p = orc.pack(b, K, d, D)
        bits = np.unpackbits(p, axis=1, bitorder="little")[:, :G * D]
        assert np.array_equal(bits.astype(np.int8), (b == -1).astype(np.int8))
        assert not np.unpackbits(p, axis=1, bitorder="little")[:, G * D:].any()
        assert np.array_equal(orc.unpack(p, K, d, D), b)


# ---------------------------------------------------------------- whitening (T4)

def pin_whiten_golden(orc):
    rows = _read_golden("whiten_example.txt")
    i = 0
    while i < len(rows):
        assert rows[i][0] == "case"
        B = int(rows[i][1])
        sign = np.array([int(v) for v in rows[i + 1][1:]], np.int8)
        x = np.array([[float(v) for v in rows[i + 2][1:]]])
        e = np.array([float(v) for v in rows[i + 3][1:]]) / math.sqrt(B)
        got = orc.whiten(x, sign=sign, block=B)[0]
        assert np.allclose(got, e, rtol=0, atol=1e-14), (got, e)
        i += 4


def pin_whiten_scipy(orc):
    """T equals the textbook Sylvester Hadamard (scipy.linalg.hadamard) on each block."""
    rng = _rng(3)
    for B, K in [(1, 5), (2, 6), (4, 8), (8, 64), (64, 128), (256, 512)]:
        x = rng.standard_normal((3, K))
        sign = _signs(rng, (K,))
        H = scipy.linalg.hadamard(B).astype(np.float64)
        expect = np.concatenate([(H @ (sign[b:b + B] * x[:, b:b + B]).T).T / math.sqrt(B)
                                 for b in range(0, K, B)], axis=1)
        got = orc.whiten(x, sign=sign, block=B)
        assert np.allclose(got, expect, rtol=0, atol=1e-12), B


def pin_whiten_orthogonal(orc):
    """T is orthogonal: norms are kept, and with sigma = +1 applying it twice is the identity."""
    rng = _rng(4)
    K, B = 1024, 256
    x = rng.standard_normal((4, K))
    sign = _signs(rng, (K,))
    t = orc.whiten(x, sign=sign, block=B)
    assert np.allclose(np.linalg.norm(t, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    tt = orc.whiten(orc.whiten(x, block=B), block=B)
    assert np.allclose(tt, x, rtol=0, atol=1e-12)
    # inverse: sigma . (H/sqrt(B)) undoes T
    back = orc.whiten(t, block=B) * sign
    assert np.allclose(back, x, rtol=0, atol=1e-12)
    # unit vectors: T(e_i)[j] = sigma_i * (-1)^popcount(i&j) / sqrt(B) inside the block
    for i in (0, 1, 5, 200):
        e = np.zeros((1, B))
        e[0, i] = 1.0
        col = orc.whiten(e, sign=sign[:B], block=B)[0]
        assert np.allclose(np.abs(col), 1 / math.sqrt(B), rtol=1e-14)
        assert col[0] * math.sqrt(B) == sign[i]
    # identity T
    assert np.array_equal(orc.whiten(x, block=0), x)


def pin_whiten_scalings(orc):
    """The 'plus scalings' part: a per-channel scale applied to x before the Hadamard."""
    rng = _rng(5)
    K, B = 512, 128
    x = rng.standard_normal((2, K))
    c = rng.uniform(0.5, 2.0, K)
    sign = _signs(rng, (K,))
    a = orc.whiten(x, sign=sign, chan_scale=c, block=B)
    b = orc.whiten(x * c, sign=sign, block=B)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- lift + forward

def _numpy_lift(xt, M, d, D):
    """blockdiag(M^T) applied to xt (numpy matmul on the [G][d] view)."""
    batch, K = xt.shape
    G = -(-K // d)
    xp = np.zeros((batch, G * d))
    xp[:, :K] = xt
    return (xp.reshape(batch, G, d) @ M).reshape(batch, G * D)


def pin_lift_matmul(orc):
    rng = _rng(6)
    for K, d, D, B in [(256, 2, 5, 256), (100, 10, 24, 4), (37, 3, 8, 0), (64, 1, 2, 64)]:
        x = rng.standard_normal((2, K))
        M = rng.standard_normal((d, D))
        sign = _signs(rng, (K,))
        z = orc.lift(x, M, d, D, sign=sign, block=B)
        xt = orc.whiten(x, sign=sign, block=B)
        if B:
            H = scipy.linalg.hadamard(B)
            xt_ref = np.concatenate([(H @ (sign[b:b + B] * x[:, b:b + B]).T).T / math.sqrt(B)
                                     for b in range(0, K, B)], axis=1)
            assert np.allclose(xt, xt_ref, atol=1e-12)
        assert np.allclose(z, _numpy_lift(xt, M, d, D), rtol=0, atol=1e-12), (K, d, D)


def _layer(rng, K, N, d, D, batch):
    G = -(-K // d)
    return dict(x=rng.standard_normal((batch, K)), M=rng.standard_normal((d, D)) / math.sqrt(D),
                b=_signs(rng, (N, G * D)), s=rng.uniform(0.5, 1.5, N),
                sign=_signs(rng, (K,)))


def pin_forward_numpy(orc):
    """y = s . (W T(x)) with W built by numpy from b and M (blockwise M b)."""
    rng = _rng(7)
    for K, N, d, D, B, batch in [(256, 33, 2, 5, 256, 2), (100, 17, 10, 24, 4, 3),
                                  (64, 8, 4, 12, 0, 1), (41, 5, 3, 8, 1, 2)]:
        L = _layer(rng, K, N, d, D, batch)
        G = -(-K // d)
        p = orc.pack(L["b"], K, d, D)
        y = orc.forward(L["x"], p, L["M"], L["s"], d, D, sign=L["sign"], block=B)
        W = (L["b"].reshape(N, G, D).astype(np.float64) @ L["M"].T).reshape(N, G * d)[:, :K]
        xt = orc.whiten(L["x"], sign=L["sign"], block=B)
        ref = (xt @ W.T) * L["s"]
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), (K, d, D)


def pin_forward_lifted_identity(orc):
    """b^T (M^T x) = (M b)^T x: the W-form and the lifted form agree in fp64."""
    rng = _rng(8)
    for K, N, d, D, B, batch in [(512, 40, 10, 24, 256, 2), (256, 64, 2, 5, 256, 1),
                                  (96, 12, 3, 8, 32, 4)]:
        L = _layer(rng, K, N, d, D, batch)
        p = orc.pack(L["b"], K, d, D)
        a = orc.forward(L["x"], p, L["M"], L["s"], d, D, sign=L["sign"], block=B)
        b = orc.forward_lifted(L["x"], p, L["M"], L["s"], d, D, sign=L["sign"], block=B)
        assert np.allclose(a, b, rtol=1e-12, atol=1e-13 * np.abs(a).max())


def pin_forward_sign_matrix(orc):
    """d = D, M = I: the operator is a plain +-1 matrix-vector product s . (B T(x))."""
    rng = _rng(9)
    for d in (1, 2, 3):
        K, N = 48, 7
        x = rng.standard_normal((2, K))
        b = _signs(rng, (N, K))
        s = rng.uniform(0.5, 1.5, N)
        sign = _signs(rng, (K,))
        p = orc.pack(b, K, d, d)
        y = orc.forward(x, p, np.eye(d), s, d, d, sign=sign, block=16)
        xt = orc.whiten(x, sign=sign, block=16)
        assert np.allclose(y, (xt @ b.T.astype(np.float64)) * s, rtol=1e-12, atol=1e-12)


def pin_forward_codeword_rows(orc):
    """Row r holding codeword r in every block: y_r = s_r (M c_r) . sum_g xt_g (closed form)."""
    rng = _rng(10)
    for d, D in [(1, 2), (2, 4), (2, 5), (3, 8)]:
        K = 30 * d
        G = K // d
        C = np.array([[(-1 if (c >> j) & 1 else 1) for j in range(D)] for c in range(1 << D)],
                     np.float64)
        b = np.tile(C, (1, G)).astype(np.int8)
        x = rng.standard_normal((2, K))
        s = rng.uniform(0.5, 1.5, 1 << D)
        M = rng.standard_normal((d, D))
        y = orc.forward(x, orc.pack(b, K, d, D), M, s, d, D)
        S = x.reshape(2, G, d).sum(axis=1)               # [batch][d], identity T
        expect = (S @ (M @ C.T)) * s                     # (M c_r) . S
        assert np.allclose(y, expect, rtol=1e-12, atol=1e-12), (d, D)


def pin_forward_bruteforce(orc):
    """Pure-Python loops on a tiny layer, every step spelled out."""
    rng = _rng(12)
    K, N, d, D, B, batch = 6, 3, 2, 5, 2, 2
    L = _layer(rng, K, N, d, D, batch)
    x, M, b, s, sign = L["x"], L["M"], L["b"], L["s"], L["sign"]
    G = 3
    xt = [[0.0] * K for _ in range(batch)]
    for t in range(batch):
        for blk in range(0, K, B):
            u0 = sign[blk] * x[t][blk]
            u1 = sign[blk + 1] * x[t][blk + 1]
            xt[t][blk] = (u0 + u1) / math.sqrt(2)
            xt[t][blk + 1] = (u0 - u1) / math.sqrt(2)
    expect = np.zeros((batch, N))
    for t in range(batch):
        for n in range(N):
            acc = 0.0
            for g in range(G):
                for i in range(d):
                    w = sum(M[i][j] * b[n][g * D + j] for j in range(D))
                    acc += w * xt[t][g * d + i]
            expect[t][n] = s[n] * acc
    y = orc.forward(x, orc.pack(b, K, d, D), M, s, d, D, sign=sign, block=B)
    assert np.allclose(y, expect, rtol=1e-13, atol=1e-13)


def pin_forward_rows_subset(orc):
    """Rows are independent: evaluating any subset of rows gives the same values."""
    rng = _rng(13)
    K, N, d, D = 200, 30, 10, 24
    L = _layer(rng, K, N, d, D, 2)
    p = orc.pack(L["b"], K, d, D)
    full = orc.forward(L["x"], p, L["M"], L["s"], d, D, sign=L["sign"], block=8)
    idx = np.array([29, 0, 7, 7, 15])
    sub = orc.forward(L["x"], p[idx], L["M"], L["s"][idx], d, D, sign=L["sign"], block=8)
    assert np.array_equal(sub, full[:, idx])
    # thread count does not change any value
    par = orc.forward(L["x"], p, L["M"], L["s"], d, D, sign=L["sign"], block=8, nthreads=4)
    assert np.array_equal(par, full)


# ---------------------------------------------------------------- encoder (Eq. 1 inner min)

def pin_encoder(orc):
    rng = _rng(14)
    for d, D in [(1, 2), (2, 4), (2, 5), (3, 8), (4, 10)]:
        M = rng.standard_normal((d, D))
        C = np.array(list(itertools.product([0, 1], repeat=D)))[:, ::-1]  # row c: bits of c
        assert np.array_equal((C * (1 << np.arange(D))).sum(axis=1), np.arange(1 << D))
        cw = 1 - 2 * C.astype(np.float64)                                  # [2^D][D]
        for _ in range(6):
            w = rng.standard_normal(d)
            dist = ((w[None, :] - cw @ M.T) ** 2).sum(axis=1)
            best = int(np.argmin(dist))
            b, c = orc.encode_bruteforce(w, M, d, D)
            assert c == best, (d, D, c, best)
            assert np.array_equal(b, cw[best].astype(np.int8))
        # a point that is itself a codeword is encoded to that codeword
        c0 = int(rng.integers(0, 1 << D))
        w0 = M @ cw[c0]
        b, c = orc.encode_bruteforce(w0, M, d, D)
        assert np.allclose(M @ b, w0, atol=1e-12)


def _all_codewords(D):
    C = np.array(list(itertools.product([0, 1], repeat=D)))[:, ::-1]     # row c: bits of c
    return 1 - 2 * C.astype(np.float64)                                   # [2^D][D], bit 1 -> -1


def pin_encoder_seeded(orc):
    """Seeded search (first d coordinates solved, the other D - d enumerated), checked against
    numpy: its distance is the distance of its code, its free part is its index, its solved part
    is the sign of numpy.linalg.solve, it never beats the exhaustive minimum, and it finds a
    planted codeword exactly."""
    rng = _rng(15)
    for d, D in [(1, 1), (3, 3), (1, 2), (2, 5), (3, 8), (4, 10), (6, 12)]:
        M = rng.standard_normal((d, D))
        cw = _all_codewords(D)
        for _ in range(5):
            w = rng.standard_normal(d)
            b, f, dist = orc.encode_seeded(w, M, d, D)
            bf = b.astype(np.float64)
            assert abs(dist - ((w - M @ bf) ** 2).sum()) <= 1e-12 * (1.0 + dist)
            assert f == sum(1 << k for k in range(D - d) if b[d + k] < 0)
            u = np.linalg.solve(M[:, :d], w - M[:, d:] @ bf[d:])
            assert np.array_equal(b[:d], np.where(u >= 0, 1, -1).astype(np.int8))
            best = ((w[None, :] - cw @ M.T) ** 2).sum(axis=1).min()
            assert dist >= best - 1e-12
            # the winner is the best of all 2^(D-d) candidates the reading defines
            cand = []
            for ff in range(1 << (D - d)):
                bF = np.array([-1.0 if (ff >> k) & 1 else 1.0 for k in range(D - d)])
                uu = np.linalg.solve(M[:, :d], w - M[:, d:] @ bF)
                bb = np.concatenate([np.where(uu >= 0, 1.0, -1.0), bF])
                cand.append(((w - M @ bb) ** 2).sum())
            assert f == int(np.argmin(cand))
        # a planted codeword is recovered (the candidate with its free part solves exactly)
        c0 = int(rng.integers(0, 1 << D))
        b, f, dist = orc.encode_seeded(M @ cw[c0], M, d, D)
        assert np.array_equal(b, cw[c0].astype(np.int8)) and dist < 1e-20
    # zero free columns: every free part ties, f = 0 wins, the rest is sign(M_S^-1 w)
    d, D = 3, 6
    M = np.concatenate([rng.standard_normal((d, d)), np.zeros((d, D - d))], axis=1)
    w = rng.standard_normal(d)
    b, f, _ = orc.encode_seeded(w, M, d, D)
    assert f == 0 and np.array_equal(b[d:], np.ones(D - d, dtype=np.int8))
    assert np.array_equal(b[:d], np.where(np.linalg.solve(M[:, :d], w) >= 0, 1, -1))


def pin_encode_rows(orc):
    """Whole-matrix encoding: K is zero-padded to a multiple of d, err is || w_blk - M b ||^2
    (numpy), the exhaustive mode is numpy's argmin over all codewords, and the thread count
    changes nothing."""
    rng = _rng(16)
    d, D, N, K = 3, 7, 5, 13                      # 13 = 4 full blocks + 1 padded block
    M = rng.standard_normal((d, D))
    w = rng.standard_normal((N, K))
    wp = np.concatenate([w, np.zeros((N, 2))], axis=1).reshape(N, 5, d)
    cw = _all_codewords(D)
    b0, e0 = orc.encode_rows(w, M, d, D, 0)
    b1, e1 = orc.encode_rows(w, M, d, D, 1)
    assert b0.shape == (N, 5, D) and e1.shape == (N, 5)
    for n in range(N):
        for g in range(5):
            dist = ((wp[n, g][None, :] - cw @ M.T) ** 2).sum(axis=1)
            assert np.array_equal(b0[n, g], cw[int(np.argmin(dist))].astype(np.int8))
            for b, e in ((b0, e0), (b1, e1)):
                assert abs(e[n, g] - ((wp[n, g] - M @ b[n, g]) ** 2).sum()) < 1e-12
            assert e1[n, g] >= e0[n, g] - 1e-12
    b2, e2 = orc.encode_rows(w, M, d, D, 1, nthreads=3)
    assert np.array_equal(b2, b1) and np.array_equal(e2, e1)


def pin_codebook_round(orc):
    """One round of the codebook fit (nearest codewords, then least-squares M), checked against
    numpy: the 1-bit scalar case in closed form (M = mean |w|), codes = numpy's argmin over all
    codewords, the straight-through gradient sum (w - M b) b^T vanishing at the new M, exact
    recovery of a codebook that generated the samples, order invariance, and a mean error that
    never rises from round to round with the exhaustive search."""
    rng = _rng(17)
    # d = D = 1: b = sign(w) (ties to +1), M_new = mean |w|
    w = rng.standard_normal((500, 1))
    M1, b1, mse = orc.codebook_round(w, np.array([[0.3]]), 1, 1)
    sg = np.where(w[:, 0] >= 0, 1, -1)
    assert np.array_equal(b1[:, 0], sg)
    assert abs(M1[0, 0] - np.abs(w).mean()) < 1e-12
    assert abs(mse - ((w[:, 0] - 0.3 * sg) ** 2).mean()) < 1e-12
    # (2, 5): codes are the exhaustive argmin; the new M zeroes the gradient
    d, D = 2, 5
    w = rng.standard_normal((300, d))
    M0 = rng.standard_normal((d, D)) * 0.5
    M1, b, mse = orc.codebook_round(w, M0, d, D)
    cw = _all_codewords(D)
    dist = ((w[:, None, :] - (cw @ M0.T)[None, :, :]) ** 2).sum(axis=2)
    assert np.array_equal(b, cw[np.argmin(dist, axis=1)].astype(np.int8))
    assert abs(mse - dist.min(axis=1).mean() / d) < 1e-12
    bf = b.astype(np.float64)
    grad = (w - bf @ M1.T).T @ bf
    assert np.abs(grad).max() < 1e-9 * len(w)
    # samples generated by a codebook are fitted exactly from that codebook
    Mt = rng.standard_normal((d, D))
    wt = _all_codewords(D) @ Mt.T
    Mr, br, mr = orc.codebook_round(wt, Mt, d, D)
    assert mr < 1e-24 and np.allclose(Mr, Mt, atol=1e-12)
    # order of the samples does not matter
    perm = rng.permutation(len(w))
    Mp, _, msep = orc.codebook_round(w[perm], M0, d, D)
    assert np.allclose(Mp, M1, atol=1e-12) and abs(msep - mse) < 1e-12
    # exhaustive rounds never raise the mean error
    M, last = M0, np.inf
    for _ in range(5):
        M, _, m = orc.codebook_round(w, M, d, D)
        assert m <= last + 1e-12
        last = m


def pin_codebook_refit(orc):
    """The least-squares step alone, against numpy's least-squares solver of min ||W - B M^T||
    (not the normal equations the oracle forms), on random codes up to D = 32; with the codes of
    a round it reproduces that round's M; a codebook whose sum b b^T is singular is rejected."""
    rng = _rng(23)
    for d, D, S in [(1, 2, 50), (2, 5, 400), (10, 24, 3000), (16, 32, 5000)]:
        w = rng.standard_normal((S, d))
        b = np.where(rng.random((S, D)) < 0.5, -1, 1).astype(np.int8)
        M = orc.codebook_refit(w, b, np.zeros((d, D)), d, D)
        ref = np.linalg.lstsq(b.astype(np.float64), w, rcond=None)[0].T
        assert np.allclose(M, ref, atol=1e-10, rtol=1e-9), (d, D)
    w = rng.standard_normal((300, 2))
    M0 = rng.standard_normal((2, 5)) * 0.5
    M1, b, _ = orc.codebook_round(w, M0, 2, 5)
    assert np.allclose(orc.codebook_refit(w, b, M0, 2, 5), M1, atol=1e-13)
    same = np.ones((40, 3), dtype=np.int8)          # every code equal: sum b b^T has rank 1
    try:
        orc.codebook_refit(rng.standard_normal((40, 2)), same, np.zeros((2, 3)), 2, 3)
        raise AssertionError("a singular sum b b^T was accepted")
    except ValueError:
        pass


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
