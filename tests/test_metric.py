"""CPU checks of the test metric used for bf16 outputs (no GPU)."""
import numpy as np

from oracle import tqp_oracle as O
from tests.gpu_util import rel_err, rel_err_bf16_out


def test_exact_bf16_rounding_has_zero_excess_error():
    y = np.random.default_rng(0).standard_t(4, size=200000)        # heavy tails
    yb = O.round_bf16(y)
    assert rel_err(yb, y) > 0.0
    assert rel_err_bf16_out(yb, y) == 0.0


def test_excess_error_sees_real_errors():
    y = np.random.default_rng(1).standard_normal(10000)
    bad = y.copy()
    bad[17] += 0.1 * np.sqrt(np.mean(y * y))
    assert rel_err_bf16_out(O.round_bf16(bad), y) > 0.09
