"""Device-side failure reporting: a bounded wait that expires records LQ_ETIMEOUT in the
workspace status word, the host reads and clears it, and the same context and workspace keep
working. The expiry is provoked with a barrier nothing arrives on (lq_check_wait_timeout): no
fault, trap or unbounded wait is involved."""
import numpy as np
import pytest

import fractional_bit_weight_b200 as lq
from fractional_bit_weight_b200 import synth
from gpu_helpers import assert_close, device_layer, oracle_rows, run_gemm

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_recovers(orc):
    layer = synth.make_layer("timeout", 21, 0, 1024, 200, 10, 24, 2)
    dl = device_layer(layer)
    ws = lq.new_workspace(2, 1024, 200, 10, 24)
    lq.check_wait_timeout(ws, limit_ms=20)
    assert lq.device_status(ws) == (lq.LQ_ETIMEOUT, lq.LQ_ETIMEOUT)
    assert lq.device_status(ws) == (lq.LQ_OK, 0)   # read once, then cleared
    y = run_gemm(layer, dl, ws).cpu().numpy()
    assert lq.device_status(ws) == (lq.LQ_OK, 0)
    assert_close(y, oracle_rows(orc, layer, np.arange(200)), "lq_gemm after a timeout")


def test_wait_timeout_rejects_bad_arguments():
    ws = lq.new_workspace(1, 256, 16, 2, 5)
    with pytest.raises(lq.LQError):
        lq.check_wait_timeout(ws, limit_ms=0)
    with pytest.raises(lq.LQError):
        lq.check_wait_timeout(ws, limit_ms=5000)
