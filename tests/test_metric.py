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


def test_block_flop_counts_match_the_closed_forms():
    # one full-config layer: forward 996 GFLOP (router 15.4, experts 927.7, LoRA 53.2);
    # adapter-only backward: dgrad ~928 + adapter gradients ~106 GFLOP
    import bench
    import synth
    fl = bench.layer_flops(synth.FULL)
    assert abs(fl["router"] / 1e9 - 15.4) < 0.1 and abs(fl["expert"] / 1e9 - 927.7) < 0.1
    assert abs(fl["lora"] / 1e9 - 53.2) < 0.1
    bwd = bench.layer_bwd_flops(synth.FULL) / 1e9
    assert abs(bwd - (927.7 + 106.3 + 0.8)) < 0.2
    # rank 0: only the expert dgrads and the small gate/router terms remain
    import dataclasses
    r0 = dataclasses.replace(synth.FULL, r=0)
    A = r0.T * r0.k
    assert bench.layer_bwd_flops(r0) == 6.0 * A * r0.d * r0.f + 4.0 * A * r0.d
