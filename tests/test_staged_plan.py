"""The TMA-staged GEMV's plan (host-only query of liblq): for every shape the kernel may run on,
the CTAs' row ranges partition the output rows, the K-slices partition the 512-coordinate chunks,
every TMA box starts inside the code matrix on a 16-byte boundary, and shared memory fits an SM.
The checks restate the contraction kernel's own indexing: slice = CTA mod S, row range = CTA div S,
windows of `wch` chunks, stages of `rows_per_stage` rows fetched as 8-row boxes. No GPU is used."""
import pytest

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import build as lqbuild

SMEM_PER_BLOCK = 232448        # 227 KB opt-in dynamic shared memory per CTA on sm_100a
RESERVED = 1024                # static shared memory and alignment slack of the two kernels
SMS = 148                      # the host query assumes a B200 when no device is visible

SHAPES = [  # (tokens, K, N, d, D, Hadamard block)
    (1, 8192, 28672, 10, 24, 256), (1, 28672, 8192, 10, 24, 256), (1, 4096, 4096, 10, 24, 256),
    (2, 8192, 28672, 10, 24, 256), (1, 8192, 8192, 1, 2, 256), (1, 8192, 8192, 2, 4, 256),
    (1, 8192, 8192, 2, 5, 256), (1, 8192, 8192, 3, 8, 256), (1, 8192, 8192, 10, 25, 256),
    (1, 8192, 8192, 4, 12, 256), (4, 8192, 28672, 10, 24, 256), (4, 28672, 8192, 10, 24, 256),
    (8, 8192, 8192, 10, 24, 256), (1, 256, 128, 2, 5, 256), (2, 777, 65, 1, 2, 1),
    (3, 4096, 300, 10, 24, 256), (5, 2048, 129, 3, 8, 256), (1, 96, 1, 2, 4, 32),
    (8, 4100, 4096, 10, 24, 0), (1, 8192, 8192, 16, 32, 256), (1, 1000, 17, 7, 9, 8),
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    lqbuild.build()


def _row_bytes(K, d, D):
    L = lq.lifted_bits(K, d, D)
    return ((L + 7) // 8 + 15) // 16 * 16


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}_{}x{}_d{}D{}_h{}".format(*s))
def test_staged_plan_in_bounds(shape):
    batch, K, N, d, D, block = shape
    p = lq.gemv_staged_plan(batch, K, N, d, D, block)
    assert p["ok"] == 1, p
    L = lq.lifted_bits(K, d, D)
    row_bytes = _row_bytes(K, d, D)
    assert p["nchunk"] == (L + 511) // 512
    # shared memory: both kernels fit one SM with the static part
    assert 0 < p["smem"] and p["smem"] + RESERVED <= SMEM_PER_BLOCK
    assert 0 < p["prep_smem"] and p["prep_smem"] + RESERVED <= SMEM_PER_BLOCK
    # windows: an odd count of 64-byte chunks (a stride of 64 mod 128 bytes), at most 31
    wch, RS = p["wch"], p["rows_per_stage"]
    assert wch % 2 == 1 and 1 <= wch <= 31 and (64 * wch) % 128 == 64
    assert RS in (16, 32) and p["NS"] >= 3
    S, sc, R, rq, rrem = p["S"], p["sc"], p["R"], p["rq"], p["rrem"]
    assert 1 <= S and 1 <= R and S * R <= SMS * 16
    covered_rows, covered_chunks = [], set()
    for cta in range(S * R):
        sl, ri = cta % S, cta // S
        c0 = sl * sc
        nc = min(sc, p["nchunk"] - c0)
        ra = ri * rq + min(ri, rrem)
        rows = rq + (1 if ri < rrem else 0)
        assert nc > 0 and rows > 0
        assert ra + rows <= N and rows <= rq + 1
        if sl == 0:
            covered_rows.append((ra, rows))
        if ri == 0:
            covered_chunks.update(range(c0, c0 + nc))
        nwin = (nc + wch - 1) // wch
        for grp in range((rows + RS - 1) // RS):
            nr = min(RS, rows - grp * RS)
            nbox = (nr + 7) // 8
            assert nbox * 8 <= RS
            # the last box of the stage starts on a row of the matrix (it may run past N)
            assert ra + grp * RS + (nbox - 1) * 8 < N
            for win in range(nwin):
                xc = (c0 + win * wch) * 8           # box x in 8-byte elements
                assert (xc * 8) % 16 == 0
                assert xc * 8 < row_bytes
                items = min(wch, nc - win * wch)
                assert items > 0 and win * wch + items <= sc
    # the row ranges partition [0, N) in order; the slices partition the chunks
    start = 0
    for ra, rows in covered_rows:
        assert ra == start
        start += rows
    assert start == N
    assert covered_chunks == set(range(p["nchunk"]))


def test_staged_plan_prefers_few_slices_and_wide_windows():
    # gate/up (39 chunks) keeps one K-slice; down (135 chunks: 207 KB of fragments for one slice)
    # takes the fewest that leave room for three stages. Both fill the 148 SMs, stage 32 rows and
    # read >= 8 useful chunks per window.
    for K, N, S in ((8192, 28672, 1), (28672, 8192, 2)):
        p = lq.gemv_staged_plan(1, K, N, 10, 24, 256)
        assert p["S"] == S and p["S"] * p["R"] == SMS and p["rows_per_stage"] == 32
        nwin = (p["sc"] + p["wch"] - 1) // p["wch"]
        assert p["sc"] / nwin >= 8


def test_staged_plan_rejects_bad_arguments():
    with pytest.raises(lq.LQError):
        lq.gemv_staged_plan(0, 8192, 8192, 10, 24, 256)
    with pytest.raises(lq.LQError):
        lq.gemv_staged_plan(1, 8192, 8192, 10, 33, 256)
    with pytest.raises(lq.LQError):
        lq.gemv_staged_plan(1, 8192, 8192, 10, 24, 96)
    with pytest.raises(lq.LQError):
        lq.gemv_staged_plan(1, 8192, 0, 10, 24, 256)
    # a Hadamard block past what the prep holds has no staged plan, without an error
    assert lq.gemv_staged_plan(1, 8192, 8192, 10, 24, 512)["ok"] == 0


def test_staged_plan_row_limit_keeps_int32_sums_exact():
    # The contraction sums, per digit plane, eight products per code byte in int32: the raw byte
    # unsigned (<= 255) and signed (|.| <= 128), and bit q alone (2^q, q = 1..6), each times a B
    # digit of magnitude <= 127. The plan takes rows of up to 2^17 lifted coordinates, which must
    # keep the whole row's sum below 2^31.
    per_byte = 127 * (255 + 128 + sum(2 ** q for q in range(1, 7)))
    assert per_byte * (2 ** 17 // 8) < 2 ** 31
    # d = 1, D = 2 lifts K inputs to 2K coordinates: K = 65536 is the longest row the plan takes
    assert lq.lifted_bits(65536, 1, 2) == 2 ** 17
    assert lq.gemv_staged_plan(1, 65536, 4096, 1, 2, 256)["ok"] == 1
    assert lq.gemv_staged_plan(1, 65536 + 256, 4096, 1, 2, 256)["ok"] == 0
