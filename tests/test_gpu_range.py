"""GPU checks of the fp16 edges of the expert path and of the status word.

The expert contractions run on fp16 operands (dequantised int4 weights are
exact in fp16; x converts exactly within fp16's range) with fp16
intermediates. These tests drive the path to those edges and check that it
either matches the fp64 oracle or raises the documented status bit:

* x scaled by 16 stays in range and must match; x scaled by 64 overflows H in
  fp16 (the oracle's own max |H| says so) and must raise TQP_STATUS_NONFINITE;
* group scales between 2^-17 and 2^-14 (fp16 subnormals) still dequantise
  exactly and must match; scales below 2^-17 must raise TQP_STATUS_RANGE;
* a LoRA factor beyond the fp16 range raises TQP_STATUS_NONFINITE;
* the backward is computed for dy * 2^P with P chosen on the device, so
  cotangents scaled by 1e-5 or 1e3 must match the oracle like unscaled ones;
* a token that lists one expert twice raises TQP_STATUS_BAD_ID in moe_permute;
* a device-side wait that runs out (the test hook shortens every wait to 1 ns)
  raises TQP_STATUS_TIMEOUT, the call returns, and the next call on the same
  stream is correct.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O
from tests.gpu_util import dev, dev_bf16, host_bf16, near_tie_tokens, rel_err, rel_err_bf16_out

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_moe_b200 as Q

TOL = 2e-2
FP16_INF = 65520.0     # the smallest magnitude that rounds to inf in fp16
BASE = synth.LayerConfig("range", T=256, d=256, E=8, k=2, f=256, g=64, r=16)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    Q.lib()


def scaled_tokens(cfg, seed, mult):
    """bf16 tokens times a power of two (exact in bf16)."""
    x = O.bf16_to_f64(synth.make_tokens(cfg.T, cfg.d, seed)) * mult
    return synth.f32_to_bf16_bits(x.astype(np.float32))


def run_layer(cfg, raw, xb):
    y = torch.empty(cfg.T, cfg.d, dtype=torch.int16, device="cuda")
    st = Q.Status()
    Q.tqp_moe_layer_fwd(dev_bf16(xb), Q.DeviceLayer(raw), y, status=st)
    torch.cuda.synchronize()
    return host_bf16(y), st.read()


def oracle_maxima(x, L):
    _, cache = O.layer_forward(x, L, want_cache=True)
    mh = max(np.abs(v[2]["h"]).max() for v in cache["experts"].values())
    mo = max(np.abs(v[2]["o"]).max() for v in cache["experts"].values())
    return mh, mo


def check_layer(cfg, raw, xb, got):
    L = O.Layer(raw)
    x = O.bf16_to_f64(xb)
    keep = ~near_tie_tokens(O.router_logits(x, L), cfg.k, 1e-4 * max(1.0, np.abs(x).max()))
    ref = O.layer_forward(x, L)
    err = rel_err_bf16_out(got[keep], ref[keep])
    assert err <= TOL, err


def test_forward_large_x_within_fp16_matches_oracle():
    raw = synth.make_layer(BASE)
    xb = scaled_tokens(BASE, 41, 16.0)
    mh, mo = oracle_maxima(O.bf16_to_f64(xb), O.Layer(raw))
    assert mh < FP16_INF / 4 and mo < FP16_INF / 4      # clearly in range
    got, st = run_layer(BASE, raw, xb)
    assert st == 0, st
    check_layer(BASE, raw, xb, got)


def test_forward_overflowing_h_raises_nonfinite():
    raw = synth.make_layer(BASE)
    xb = scaled_tokens(BASE, 41, 64.0)
    mh, _ = oracle_maxima(O.bf16_to_f64(xb), O.Layer(raw))
    assert mh > 1.1 * FP16_INF                            # clearly beyond fp16
    _, st = run_layer(BASE, raw, xb)
    assert st & Q.STATUS_NONFINITE, st


def test_group_scales_in_fp16_subnormal_range_are_exact():
    # weights x 2^-9 put every group scale in [2^-15.3, 2^-13.4]: fp16
    # subnormals, but q * s still lands on fp16's 2^-24 grid, so dequant stays
    # exact; x x 2^9 keeps the activations at their usual size
    cfg = dataclasses.replace(BASE, w_mult=2.0 ** -9)
    raw = synth.make_layer(cfg)
    s = O.bf16_to_f64(raw["ws0"])
    assert s[s > 0].min() < 2.0 ** -14 and s[s > 0].min() >= 2.0 ** -17
    xb = scaled_tokens(cfg, 42, 2.0 ** 9)
    got, st = run_layer(cfg, raw, xb)
    assert st == 0, st
    check_layer(cfg, raw, xb, got)


def test_group_scales_below_fp16_grid_raise_range():
    cfg = dataclasses.replace(BASE, w_mult=2.0 ** -13)
    raw = synth.make_layer(cfg)
    s = O.bf16_to_f64(raw["ws0"])
    assert s[s > 0].max() < 2.0 ** -17
    _, st = run_layer(cfg, raw, scaled_tokens(cfg, 43, 2.0 ** 13))
    assert st & Q.STATUS_RANGE, st


def test_lora_factor_beyond_fp16_raises_nonfinite():
    raw = synth.make_layer(BASE)
    raw = dict(raw)
    lb = raw["lb0"].copy()
    lb[:, 0, 0] = synth.f32_to_bf16_bits(np.array([1.0e5], np.float32))[0]   # every expert's first gate row
    raw["lb0"] = lb
    _, st = run_layer(BASE, raw, synth.make_tokens(BASE.T, BASE.d, 44))
    assert st & Q.STATUS_NONFINITE, st


@pytest.mark.parametrize("dy_mult", [1e-5, 1e3], ids=["dy_1e-5", "dy_1e3"])
def test_backward_scale_of_cotangent_does_not_matter(dy_mult):
    cfg = synth.LayerConfig("bwr", T=300, d=256, E=10, k=3, f=256, g=64, r=16)
    raw = synth.make_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, 45)
    dy = (synth.make_grad(cfg.T, cfg.d, 46, "dy1") * np.float32(dy_mult)).astype(np.float32)
    DL = Q.DeviceLayer(raw)
    dx = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    dA, dB, g = DL.grads()
    st = Q.Status()
    Q.tqp_moe_layer_bwd(dev_bf16(xb), dev(dy), DL, dx, g, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0, st.read()
    x = O.bf16_to_f64(xb)
    rdx, rdA, rdB = O.layer_backward(x, dy.astype(np.float64), L)
    logits = O.router_logits(x, L)
    tie = near_tie_tokens(logits, cfg.k, 1e-4)
    srt = np.argsort(-logits[tie], axis=1, kind="stable")
    amb = set(srt[:, cfg.k - 1].tolist()) | set(srt[:, cfg.k].tolist()) if tie.any() else set()
    keep = np.array([e not in amb for e in range(cfg.E)])
    assert rel_err(dx.cpu().numpy()[~tie], rdx[~tie]) <= TOL
    for p in range(3):
        assert rel_err(dA[p].cpu().numpy()[keep], rdA[p][keep]) <= TOL, ("dA", p)
        assert rel_err(dB[p].cpu().numpy()[keep], rdB[p][keep]) <= TOL, ("dB", p)


def test_permute_token_listing_an_expert_twice_raises_bad_id():
    T, E, k = 100, 16, 3
    ids = O.topk(synth.make_logits(T, E, seed=5), k).astype(np.int32)
    ids[17, 2] = ids[17, 0]          # token 17 names its first expert again
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    st = Q.Status()
    Q.moe_permute(dev(ids), E, offsets, perm, inv, status=st)
    torch.cuda.synchronize()
    assert st.read() & Q.STATUS_BAD_ID
    # without the repeat the same call is clean
    ids[17, 2] = O.topk(synth.make_logits(T, E, seed=5), k)[17, 2]
    st.clear()
    Q.moe_permute(dev(ids), E, offsets, perm, inv, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0


def test_wait_timeout_raises_status_and_next_call_is_correct():
    cfg = synth.TINY
    raw = synth.make_layer(cfg)
    xb = synth.make_tokens(cfg.T, cfg.d, 47)
    L = Q.DeviceLayer(raw)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.int16, device="cuda")
    st = Q.Status()
    try:
        Q.tqp_debug_set_wait_limit_ns(1)          # every wait that has to spin runs out
        Q.tqp_moe_layer_fwd(dev_bf16(xb), L, y, status=st)
        torch.cuda.synchronize()
    finally:
        Q.tqp_debug_set_wait_limit_ns(0)
    assert st.read() & Q.STATUS_TIMEOUT, st.read()
    # the context is intact: the same call with the default limit is correct
    st.clear()
    y2 = torch.empty_like(y)
    Q.tqp_moe_layer_fwd(dev_bf16(xb), L, y2, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0, st.read()
    check_layer(cfg, raw, xb, host_bf16(y2))
