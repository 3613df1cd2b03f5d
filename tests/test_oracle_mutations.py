"""Plant plausible mistakes in the oracle (CPU only) and check that a pin fails.

Each case swaps one oracle function for a subtly wrong version and runs the
pin that should catch it; the pin must raise AssertionError.
"""
import numpy as np
import pytest

from oracle import tqp_oracle as O
import tests.test_oracle_pins as pins


def _drop_lora(X, P, s):
    return _orig_expert_forward(X, P, 0.0)


def _transposed_tie_break(logits, k):
    l = np.asarray(logits, dtype=np.float64)
    E = l.shape[1]
    flipped = l[:, ::-1]
    ids = _orig_topk(flipped, k)
    return (E - 1 - ids).astype(np.int32)                # ties -> higher id first


def _gate_backward_sign(x, dy, L, ids=None):
    # same as the oracle but with the softmax-gate backward term negated
    dx, dA, dB = _orig_layer_backward(x, dy, L, ids)
    xr = np.asarray(x, np.float64)
    logits = O.router_logits(xr, L)
    ids_ = O.topk(logits, L.k) if ids is None else ids
    gam = O.gates(logits, ids_)
    y, cache = O.layer_forward(xr, L, ids=ids_, want_cache=True)
    dgam = np.zeros_like(gam)
    for e, (t_idx, j_idx, fwd) in cache["experts"].items():
        dgam[t_idx, j_idx] = np.sum(np.asarray(dy)[t_idx] * fwd["o"], axis=1)
    dl = gam * (dgam - np.sum(gam * dgam, axis=1, keepdims=True))
    for j in range(ids_.shape[1]):
        dx -= 2 * dl[:, j:j + 1] * L.router_w[ids_[:, j]]
    return dx, dA, dB


def _natural_nibbles(codes):
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    words = c.view("<u4").astype(np.int64)
    K = c.shape[-1] * 2
    out = np.empty(c.shape[:-1] + (K // 8, 8), dtype=np.int64)
    for i in range(8):
        out[..., i] = (words >> (4 * i)) & 0xF
    out = np.where(out >= 8, out - 16, out)
    return out.reshape(c.shape[:-1] + (K,))


def _inverse_adds(y1, y2, F, G):
    y1 = np.asarray(y1, dtype=np.float64)
    y2 = np.asarray(y2, dtype=np.float64)
    x2 = y2 + O.layer_forward(O.round_bf16(y1), G)
    return y1 - O.layer_forward(x2, F), x2


def _skip_down_adapter_grad(X, dO, P, s, fwd):
    res = _orig_expert_backward(X, dO, P, s, fwd)
    res["dB"][2] = np.zeros_like(res["dB"][2])
    return res


def _unscaled_lora_grad(X, dO, P, s, fwd):
    res = _orig_expert_backward(X, dO, P, s, fwd)
    res["dA"][0] = res["dA"][0] / s
    return res


def _stack_grads_in_walk_order(y1, y2, dy1, dy2, blocks, round_inputs=True):
    # the per-block gradients left in the order the backward walks the blocks
    res = _orig_stack_backward(y1, y2, dy1, dy2, blocks, round_inputs)
    res["grads"] = res["grads"][::-1]
    return res


def _stack_inverse_forward_order(y1, y2, blocks, round_inputs=True):
    # undoes the blocks first to last instead of last to first
    return _orig_stack_inverse(y1, y2, blocks[::-1], round_inputs)


def _adamw_coupled_decay(p, m, v, g, lr, beta1, beta2, eps, weight_decay, t, grad_scale=1.0):
    # L2-regularised Adam (decay folded into the gradient) instead of decoupled decay
    p = np.asarray(p, dtype=np.float64)
    return _orig_adamw_step(p, m, v, np.asarray(g, dtype=np.float64) + weight_decay * p, lr, beta1, beta2, eps, 0.0,
                            t, grad_scale)


_orig_adamw_step = O.adamw_step
_orig_stack_backward = O.stack_backward
_orig_stack_inverse = O.stack_inverse
_orig_expert_forward = O.expert_forward
_orig_topk = O.topk
_orig_layer_backward = O.layer_backward
_orig_expert_backward = O.expert_backward

CASES = [
    ("expert_forward", _drop_lora, pins.test_single_expert_top1_is_dense_swiglu_ffn),
    ("topk", _transposed_tie_break, pins.test_topk_matches_brute_force_with_ties_zeros_nan),
    ("layer_backward", _gate_backward_sign, pins.test_layer_backward_finite_differences),
    ("unpack_int4", _natural_nibbles, pins.test_unpack_int4_golden_words),
    ("coupling_inverse", _inverse_adds, pins.test_coupling_inverse_reconstructs_inputs),
    ("expert_backward", _skip_down_adapter_grad, pins.test_layer_backward_finite_differences),
    ("expert_backward", _unscaled_lora_grad, pins.test_layer_backward_finite_differences),
    ("stack_backward", _stack_grads_in_walk_order, pins.test_stack_backward_finite_differences),
    ("stack_inverse", _stack_inverse_forward_order, pins.test_stack_inverse_reconstructs_inputs),
    ("adamw_step", _adamw_coupled_decay, pins.test_adamw_matches_torch_adamw_over_several_steps),
]


@pytest.mark.parametrize("name,mutant,pin", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, pin):
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()
