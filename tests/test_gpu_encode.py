"""lq_encode against the oracle's searches (exhaustive 2^D and seeded 2^(D-d)), through the
C ABI. Both sides search the same candidates; the GPU compares distances in fp32 and the oracle
in fp64, so where two candidates lie within fp32 rounding of each other the picks may differ.
The tests therefore compare what is unique: planted codewords are recovered exactly, every
GPU pick is as good as the oracle's to fp32 rounding (distances evaluated in fp64 by numpy),
nearly all picks are identical, and err is the distance of the returned code."""
import numpy as np
import pytest
import torch

import fractional_bit_weight_b200 as lq

pytestmark = pytest.mark.gpu


def _rng(seed):
    return np.random.default_rng([7, seed])


def _dist64(w, M, b, d):
    """fp64 ||w_block - M b||^2 of every block of w [N][K] (zero-padded) and codes b [N][G][D]."""
    N, K = w.shape
    G = b.shape[1]
    wp = np.zeros((N, G * d))
    wp[:, :K] = w
    blocks = wp.reshape(N, G, d)
    rec = np.einsum("ij,ngj->ngi", M.astype(np.float64), b.astype(np.float64))
    return ((blocks - rec) ** 2).sum(axis=2)


def _run(w, M, d, D, mode):
    b, err = lq.encode(torch.from_numpy(w).cuda(), torch.from_numpy(M).cuda(), d, D, mode)
    torch.cuda.synchronize()
    return b.cpu().numpy(), err.cpu().numpy()


@pytest.mark.parametrize("mode,d,D", [(0, 2, 5), (0, 3, 8), (0, 4, 12), (0, 1, 2), (0, 10, 14),
                                      (1, 2, 5), (1, 3, 8), (1, 4, 12), (1, 10, 24), (1, 3, 3),
                                      (1, 16, 32)])
def test_planted_codewords_are_recovered(mode, d, D):
    rng = _rng(d * 100 + D + mode)
    M = (rng.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    N, G = 6, 11
    b0 = np.where(rng.random((N, G, D)) < 0.5, -1, 1).astype(np.int8)
    w = np.einsum("ij,ngj->ngi", M.astype(np.float64), b0.astype(np.float64)).reshape(N, G * d)
    w = w.astype(np.float32)
    b, err = _run(w, M, d, D, mode)
    assert np.array_equal(b, b0)
    assert np.all(err < 1e-8)


@pytest.mark.parametrize("mode,d,D,N,K", [(0, 2, 5, 40, 256), (0, 3, 8, 17, 301),
                                          (0, 4, 12, 9, 100), (1, 2, 5, 40, 256),
                                          (1, 3, 8, 17, 301), (1, 4, 12, 9, 100),
                                          (1, 10, 24, 4, 160), (1, 5, 5, 8, 64)])
def test_matches_oracle(orc, mode, d, D, N, K):
    rng = _rng(d * 1000 + D * 10 + mode + K)
    M = (rng.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    w = rng.standard_normal((N, K)).astype(np.float32)
    b, err = _run(w, M, d, D, mode)
    bo, eo = orc.encode_rows(w, M, d, D, mode)
    dg = _dist64(w, M, b, d)
    # err is the distance of the returned code; the pick is as good as the oracle's
    assert np.allclose(err, dg, rtol=1e-4, atol=1e-5)
    assert np.all(dg <= eo * (1 + 1e-4) + 1e-5), np.max(dg - eo)
    same = np.all(b == bo, axis=2).mean()
    assert same >= 0.98, same
    print(f"mode={mode} d={d} D={D}: {same:.4f} of the blocks pick the oracle's code")
