"""Parity of lq_codebook_round (one round of the offline fit of M: nearest codewords, then the
least-squares M) with the fp64 oracle, through the C ABI, over several rounds.

The GPU compares candidate codewords in fp32 and the oracle in fp64, so near-ties may be
resolved differently; the checks compare what is unique: at least 98 % of the codes equal the
oracle's, no GPU code is worse than the oracle's beyond fp32 rounding, the new M equals the
oracle's least-squares fit on the GPU's own codes (to fp32 rounding), and the reported mean
error equals the mean distance of the GPU's codes.
"""
import numpy as np
import pytest
import torch

import fractional_bit_weight_b200 as lq
from gpu_helpers import NOTES

pytestmark = pytest.mark.gpu


def _dist(w, M, b):
    return ((w - b.astype(np.float64) @ M.T) ** 2).sum(axis=1)


@pytest.mark.parametrize("d,D,mode,S", [(1, 2, lq.LQ_ENCODE_EXACT, 500),
                                        (2, 5, lq.LQ_ENCODE_EXACT, 4000),
                                        (3, 8, lq.LQ_ENCODE_EXACT, 3000),
                                        (4, 12, lq.LQ_ENCODE_EXACT, 2000),
                                        (10, 24, lq.LQ_ENCODE_SEEDED, 1500),
                                        (2, 5, lq.LQ_ENCODE_SEEDED, 3000)])
def test_codebook_rounds_match_oracle(orc, d, D, mode, S):
    rng = np.random.Generator(np.random.PCG64([31, d, D, mode]))
    w = rng.standard_normal((S, d)).astype(np.float32)
    M0 = (rng.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    w64 = w.astype(np.float64)
    wg, Mg = torch.from_numpy(w).cuda(), torch.from_numpy(M0).cuda()
    last = np.inf
    mses = []
    for rnd in range(3):
        Mb = Mg.cpu().numpy().astype(np.float64)          # the M this round starts from
        _, b, mse = lq.codebook_round(wg, Mg, d, D, mode)
        bg = b.cpu().numpy()
        Mnew = Mg.cpu().numpy().astype(np.float64)
        mse_g = float(mse.cpu().numpy()[0])
        Mo, bo, mse_o = orc.codebook_round(w64, Mb, d, D, mode)
        same = (bg == bo).all(axis=1).mean()
        dg, do = _dist(w64, Mb, bg), _dist(w64, Mb, bo)
        assert same >= 0.98, (rnd, same)
        if mode == lq.LQ_ENCODE_EXACT:
            assert (dg <= do + 1e-5 * (1.0 + do)).all(), rnd
        ref = orc.codebook_refit(w64, bg, Mb, d, D)
        assert np.allclose(Mnew, ref, rtol=1e-5, atol=1e-6), (rnd, np.abs(Mnew - ref).max())
        assert abs(mse_g - dg.mean() / d) <= 1e-5 * dg.mean() / d + 1e-9, (rnd, mse_g)
        if same == 1.0:
            assert np.allclose(Mnew, Mo, rtol=1e-5, atol=1e-6)
            assert abs(mse_g - mse_o) <= 1e-5 * mse_o + 1e-9
        if mode == lq.LQ_ENCODE_EXACT:
            assert mse_g <= last * (1 + 1e-5)      # exhaustive rounds never raise the error
        last = mse_g
        mses.append(mse_g)
        print(f"d={d} D={D} mode={mode} round {rnd}: codes equal {same:.4f}, mse {mse_g:.6f}")
    NOTES.append(f"codebook fit d={d} D={D} {'seeded' if mode == lq.LQ_ENCODE_SEEDED else 'exact'} "
                 f"S={S}: per-coordinate MSE of the encodings in three fit steps (the first under the random M) " +
                 ", ".join(f"{m:.5f}" for m in mses))


def test_codebook_round_recovers_a_generating_codebook(orc):
    """Samples that are codewords of M (all 2^D of them, twice) are encoded exactly and refit
    to M itself, with zero error."""
    d, D = 3, 8
    rng = np.random.Generator(np.random.PCG64(32))
    M = rng.standard_normal((d, D)).astype(np.float32)
    cw = np.array([[(-1 if (c >> j) & 1 else 1) for j in range(D)] for c in range(1 << D)],
                  np.float32)
    w = np.tile(cw @ M.T, (2, 1)).astype(np.float32)
    Mg = torch.from_numpy(M).cuda()
    _, b, mse = lq.codebook_round(torch.from_numpy(w).cuda(), Mg, d, D, lq.LQ_ENCODE_EXACT)
    assert np.array_equal(b.cpu().numpy(), np.tile(cw, (2, 1)).astype(np.int8))
    assert float(mse.cpu().numpy()[0]) < 1e-10
    assert np.allclose(Mg.cpu().numpy(), M, rtol=1e-5, atol=1e-6)


def test_codebook_round_leaves_a_singular_fit_alone():
    """All samples on one codeword: sum b b^T is singular, M stays, the error reads -1."""
    d, D = 2, 5
    M = np.ones((d, D), np.float32)
    w = np.full((64, d), 5.0, np.float32)          # nearest codeword: all +1, for every sample
    Mg = torch.from_numpy(M).cuda()
    _, b, mse = lq.codebook_round(torch.from_numpy(w).cuda(), Mg, d, D, lq.LQ_ENCODE_EXACT)
    assert (b.cpu().numpy() == 1).all()
    assert float(mse.cpu().numpy()[0]) == -1.0
    assert np.array_equal(Mg.cpu().numpy(), M)
