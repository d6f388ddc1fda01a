"""Plant plausible mistakes in copies of the oracle and check that the pins catch each one.

Every mutant is a textual edit of oracle/lq_oracle.c (a flipped sign, a dropped term or
factor, a transposed operand, a wrong index or bit order), compiled into a temporary
directory and run against all pins in a child process. A mutant that no pin rejects
means the pins leave that part of the oracle unchecked.
"""
import json
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lq_oracle.c")

# (name, exact text in lq_oracle.c, replacement)
MUTANTS = [
    ("hadamard_or_instead_of_and", "orc_parity((uint32_t)(i & j))", "orc_parity((uint32_t)(i | j))"),
    ("hadamard_no_normalisation", "yr[b0 + i] = acc * norm;", "yr[b0 + i] = acc;"),
    ("hadamard_normalised_by_block", "1.0 / sqrt((double)block)", "1.0 / (double)block"),
    ("whiten_sign_dropped", "if (sign) v *= (double)sign[b0 + j];", ";"),
    ("whiten_sign_reversed", "if (sign) v *= (double)sign[b0 + j];",
     "if (sign) v *= (double)sign[b0 + block - 1 - j];"),
    ("whiten_scale_dropped", "if (chan_scale) v *= chan_scale[b0 + j];", ";"),
    ("lift_M_transposed", "acc += M[i * D + j] * v;", "acc += M[j * d + i] * v;"),
    ("forward_M_transposed", "acc += M[i * D + j] * (double)br[g * D + j];",
     "acc += M[j * d + i] * (double)br[g * D + j];"),
    ("forward_last_input_dropped", "for (int32_t k = 0; k < K; ++k) acc += w[k] * xt[t * K + k];",
     "for (int32_t k = 0; k + 1 < K; ++k) acc += w[k] * xt[t * K + k];"),
    ("forward_scale_dropped", "y[t * nrows + n] = s[n] * acc;\n      }\n    }\n    free(br);\n    free(w);",
     "y[t * nrows + n] = acc;\n      }\n    }\n    free(br);\n    free(w);"),
    ("lifted_sign_flipped", "acc += (double)br[q] * z[t * bits + q];",
     "acc -= (double)br[q] * z[t * bits + q];"),
    ("pack_msb_first", "orow[q / 8] |= (uint8_t)(1u << (q % 8));",
     "orow[q / 8] |= (uint8_t)(1u << (7 - q % 8));"),
    ("unpack_msb_first", "int bit = (prow[q / 8] >> (q % 8)) & 1;",
     "int bit = (prow[q / 8] >> (7 - q % 8)) & 1;"),
    ("pack_set_bit_means_plus_one", "if (br[q] == -1) {", "if (br[q] == 1) {"),
    ("unpack_set_bit_means_plus_one", "b[n * bits + q] = bit ? (int8_t)-1 : (int8_t)1;",
     "b[n * bits + q] = bit ? (int8_t)1 : (int8_t)-1;"),
    ("row_padding_8_bytes", "return (bytes + 15) / 16 * 16;", "return (bytes + 7) / 8 * 8;"),
    ("encoder_argmax", "if (best < 0 || dist < best_dist) {", "if (best < 0 || dist > best_dist) {"),
    ("seeded_argmax", "if (dist < best_dist || best < 0) {", "if (dist > best_dist || best < 0) {"),
    ("seeded_solved_sign", "b[c] = u >= 0.0 ? (int8_t)1 : (int8_t)-1;",
     "b[c] = u >= 0.0 ? (int8_t)-1 : (int8_t)1;"),
    ("seeded_free_bit_order", "b[d + k] = ((f >> k) & 1) ? (int8_t)-1 : (int8_t)1;",
     "b[d + k] = ((f >> (F - 1 - k)) & 1) ? (int8_t)-1 : (int8_t)1;"),
    ("codebook_gram_transposed", "C[j * (D + d) + k] += (double)bn[j] * (double)bn[k];",
     "C[j * (D + d) + k] += (double)bn[j] * (double)bn[j];"),
    ("codebook_cross_term_sign", "A[i * D + j] += w[n * d + i] * (double)bn[j];",
     "A[i * D + j] -= w[n * d + i] * (double)bn[j];"),
    ("encoder_codeword_sign", "r -= M[i * D + j] * (((c >> j) & 1) ? -1.0 : 1.0);",
     "r -= M[i * D + j] * (((c >> j) & 1) ? 1.0 : -1.0);"),
    ("lift_padding_reads_next_block", "double v = (k < K) ? xt[t * K + k] : 0.0;",
     "double v = (k < K) ? xt[t * K + k] : 1.0;"),
]

CHILD = r"""
import json, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle, oracle_pins
orc = oracle.Oracle({lib!r})
failed = []
for pin in oracle_pins.ALL_PINS:
    try:
        pin(orc)
    except Exception as e:
        failed.append(pin.__name__)
print("RESULT" + json.dumps(failed))
"""


def _build_mutant(tmp, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutant {name}: anchor text not found exactly once"
    path = os.path.join(tmp, name + ".c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp, name + ".so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", path, "-o", lib,
                    "-lm"], check=True)
    return lib


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build_mutant(tmp, name, old, new)
        code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), lib=lib)
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           timeout=300)
        if r.returncode != 0 and "RESULT" not in r.stdout:
            return          # the mutant crashed the pins' process: caught
        failed = json.loads(r.stdout.split("RESULT", 1)[1])
        assert failed, f"no pin rejects mutant {name}"
