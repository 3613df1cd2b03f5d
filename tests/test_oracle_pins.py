"""Pins for the fp64 oracle: each check ties it to something other than itself.

CPU only. Kinds of pin: hand-derived golden fixtures (tests/golden), brute
force on tiny inputs, library reductions (torch fp64 SwiGLU FFN, math.fsum),
closed forms, invariants, and central finite differences for the backward.
A plausible mistake in the oracle (a dropped LoRA term, a wrong sign in the
softmax-gate backward, a transposed adapter, a swapped tie-break) fails at
least one of them; tests/test_oracle_mutations.py plants such mistakes to show it.
"""
import dataclasses
import math
import os

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

SMALL = synth.LayerConfig("pin", T=48, d=64, E=6, k=2, f=64, g=32, r=8)


def small_layer(cfg=SMALL, seed=0):
    raw = synth.make_layer(cfg, seed)
    return raw, O.Layer(raw)


def tokens(cfg, seed=5):
    return O.bf16_to_f64(synth.make_tokens(cfg.T, cfg.d, seed))


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-300)


# ---------------------------------------------------------------- formats


def test_unpack_int4_golden_words():
    rows = []
    for line in open(os.path.join(GOLDEN, "int4_words.txt")):
        if line.strip() and not line.startswith("#"):
            parts = line.split()
            rows.append((int(parts[0], 16), [int(v) for v in parts[1:]]))
    words = np.array([w for w, _ in rows], dtype="<u4")
    codes = words.view(np.uint8).reshape(len(rows), 4)
    got = O.unpack_int4(codes)
    assert got.tolist() == [v for _, v in rows]


def test_pack_unpack_roundtrip_all_codes():
    rng = np.random.default_rng(1)
    q = rng.integers(-8, 8, size=(7, 64))
    assert np.array_equal(O.unpack_int4(synth.pack_int4(q)), q)


def test_bf16_decode_matches_torch():
    bits = np.random.default_rng(2).integers(0, 1 << 16, size=4096).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]                      # drop inf/nan patterns
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_to_f64(bits), ref)


def test_round_bf16_matches_torch_on_fp32_values():
    x = np.random.default_rng(3).standard_normal(100000).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(x.astype(np.float64)), ref)


def test_dequant_roundtrip_bound_and_on_grid_exact():
    g = 32
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((16, 128)) / 8).astype(np.float32)
    w[3, 32:64] = 0.0                                               # an all-zero group
    codes, scales = synth.quantise_int4(w, g)
    what = O.dequant(codes, scales, g)
    s = np.repeat(O.bf16_to_f64(scales).T, g, axis=1)
    assert np.all(np.abs(what - w) <= s / 2 + 1e-12)
    assert np.all(what[3, 32:64] == 0)
    # on-grid weights (q * s with bf16 s and a group reaching |q| = 7) round-trip exactly
    q = rng.integers(-7, 8, size=(16, 128))
    q[:, ::g] = 7
    sc = O.bf16_to_f64(synth.f32_to_bf16_bits(rng.uniform(0.01, 0.1, size=(16, 128 // g)).astype(np.float32)))
    w2 = (q * np.repeat(sc, g, axis=1)).astype(np.float32)
    c2, s2 = synth.quantise_int4(w2, g)
    assert np.array_equal(O.dequant(c2, s2, g), w2.astype(np.float64))
    assert np.array_equal(O.unpack_int4(c2), q)


def test_int8_decode_golden_bytes_and_dequant_roundtrip():
    # two's-complement bytes, hand-decoded
    raw = np.array([[0x00, 0x01, 0x7F, 0x80, 0x81, 0xFF, 0xF9, 0x07]], dtype=np.uint8)
    assert O.unpack_int8(raw).tolist() == [[0, 1, 127, -128, -127, -1, -7, 7]]
    g = 64
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((16, 256)) / 8).astype(np.float32)
    w[2, 64:128] = 0.0
    codes, scales = synth.quantise_int8(w, g)
    assert codes.shape == (16, 256)
    what = O.dequant(codes, scales, g, bits=8)
    s = np.repeat(O.bf16_to_f64(scales).T, g, axis=1)
    assert np.all(np.abs(what - w) <= s / 2 + 1e-12)
    assert np.all(what[2, 64:128] == 0)
    # on-grid weights with a group reaching |q| = 127 round-trip exactly
    q = rng.integers(-127, 128, size=(16, 256))
    q[:, ::g] = 127
    sc = O.bf16_to_f64(synth.f32_to_bf16_bits(rng.uniform(1e-4, 1e-3, size=(16, 256 // g)).astype(np.float32)))
    w2 = (q * np.repeat(sc, g, axis=1)).astype(np.float32)
    c2, s2 = synth.quantise_int8(w2, g)
    assert np.array_equal(O.unpack_int8(c2), q)
    assert np.array_equal(O.dequant(c2, s2, g, bits=8), w2.astype(np.float64))


# ---------------------------------------------------------------- router, top-k, gates


def test_router_logits_exact_sum():
    raw, L = small_layer()
    x = tokens(SMALL)[:5]
    l = O.router_logits(x, L)
    for t in range(5):
        for e in range(SMALL.E):
            exact = math.fsum(float(a) * float(b) for a, b in zip(x[t], L.router_w[e]))
            assert abs(l[t, e] - exact) <= 1e-13 * max(1.0, abs(exact))


def _brute_topk(row, k):
    key = [((1 if math.isnan(v) else 0), (0.0 if math.isnan(v) else -v), e) for e, v in enumerate(row)]
    return [e for _, _, e in sorted(key)[:k]]


def test_topk_matches_brute_force_with_ties_zeros_nan():
    rng = np.random.default_rng(6)
    T, E = 300, 23
    l = np.round(rng.standard_normal((T, E)) * 2) / 2              # coarse grid: many exact ties
    l[::7, 3] = -0.0
    l[::7, 9] = 0.0
    l[::11, 5] = np.nan
    l[::13, 0] = -np.inf
    l[::17, 1] = np.inf
    for k in (1, 4, E):
        ids = O.topk(l, k)
        for t in range(T):
            assert ids[t].tolist() == _brute_topk(l[t].tolist(), k)


def test_gates_golden_closed_form():
    for line in open(os.path.join(GOLDEN, "gates_closed_form.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        k_part, rest = line.split("|")
        lp, ip, gp = rest.split(";")
        k = int(k_part)
        l = np.array([[float(v) for v in lp.split()]])
        ids = O.topk(l, k)
        assert ids[0].tolist() == [int(v) for v in ip.split()]
        gam = O.gates(l, ids)
        assert np.allclose(gam[0], [float(v) for v in gp.split()], rtol=0, atol=1e-15)


def test_gates_sum_to_one_and_non_increasing():
    l = np.random.default_rng(7).standard_normal((500, 40)) * 3
    ids = O.topk(l, 12)
    gam = O.gates(l, ids)
    assert np.max(np.abs(gam.sum(1) - 1)) <= 1e-12
    assert np.all(np.diff(gam, axis=1) <= 0)
    # equals the full softmax renormalised over the chosen experts (library softmax)
    full = torch.softmax(torch.from_numpy(l), dim=1).numpy()
    sel = np.take_along_axis(full, ids.astype(np.int64), 1)
    assert np.allclose(gam, sel / sel.sum(1, keepdims=True), rtol=1e-13, atol=0)


def test_huge_bias_selects_most_biased_experts():
    cfg = dataclasses.replace(SMALL, E=10, k=3)
    raw = synth.make_layer(cfg)
    raw["bias"] = np.array([0, 100, 0, 0, 300, 0, 0, 200, 0, 0], np.float32)
    L = O.Layer(raw)
    ids = O.topk(O.router_logits(tokens(cfg), L), 3)
    assert np.all(ids == np.array([4, 7, 1]))


# ---------------------------------------------------------------- permutation


def test_permute_invariants_and_brute_force():
    rng = np.random.default_rng(8)
    T, E, k = 200, 17, 5
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    ids[:50] = ids[0]                                              # a popular set of experts
    offsets, perm, inv = O.permute(ids, E)
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.array_equal(np.diff(offsets), np.bincount(ids.ravel(), minlength=E))
    assert sorted(inv.tolist()) == list(range(T * k))              # bijection
    brute = sorted((int(ids[t, j]), t, j) for t in range(T) for j in range(k))
    for row, (e, t, j) in enumerate(brute):
        assert perm[row] == t and inv[t * k + j] == row
        assert offsets[e] <= row < offsets[e + 1]


def test_combine_matches_layer_forward():
    raw, L = small_layer()
    x = tokens(SMALL)
    y, cache = O.layer_forward(x, L, want_cache=True)
    ids, gam = cache["ids"], cache["gates"]
    offsets, perm, inv = O.permute(ids, SMALL.E)
    o_rows = np.zeros((SMALL.A, SMALL.d))
    for e in range(SMALL.E):
        rows = np.arange(offsets[e], offsets[e + 1])
        o_rows[rows] = O.expert_forward(x[perm[rows]], L.expert(e), L.s)["o"]
    assert rel(O.combine(o_rows, gam, inv, SMALL.T, SMALL.k), y) <= 1e-13


# ---------------------------------------------------------------- layer reductions


def _torch_dense_ffn(x, P, s):
    """Dense SwiGLU FFN with LoRA, through torch fp64 library ops."""
    X = torch.from_numpy(x)
    t = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in P.items()}
    lin = torch.nn.functional.linear
    gate = lin(X, t["Wg"]) + s * (X @ t["Ag"]) @ t["Bg"]
    up = lin(X, t["Wu"]) + s * (X @ t["Au"]) @ t["Bu"]
    h = torch.nn.functional.silu(gate) * up
    return (lin(h, t["Wd"]) + s * (h @ t["Ad"]) @ t["Bd"]).numpy()


def test_single_expert_top1_is_dense_swiglu_ffn():
    cfg = dataclasses.replace(SMALL, E=1, k=1)
    raw, L = small_layer(cfg)
    x = tokens(cfg)
    y, cache = O.layer_forward(x, L, want_cache=True)
    assert np.all(cache["gates"] == 1.0)
    assert rel(y, _torch_dense_ffn(x, L.expert(0), L.s)) <= 1e-12


def _identical_experts(cfg, src=0):
    raw = synth.make_layer(cfg)
    for p in range(3):
        for key in ("wq", "ws", "la", "lb"):
            raw[f"{key}{p}"][:] = raw[f"{key}{p}"][src]
    return raw


def test_identical_experts_reduce_to_dense_ffn_for_any_routing():
    # dense -> MoE growth initialises experts from the dense weights and must
    # preserve the function ("Principle 2": "Dense to MoE: Initialize experts
    # from dense weights"): with equal experts the gates sum to one.
    cfg = dataclasses.replace(SMALL, E=7, k=3)
    raw = _identical_experts(cfg)
    x = tokens(cfg)
    L = O.Layer(raw)
    dense = _torch_dense_ffn(x, L.expert(0), L.s)
    assert rel(O.layer_forward(x, L), dense) <= 1e-12
    raw["bias"] = np.linspace(-3, 3, cfg.E).astype(np.float32)    # changes routing, not the output
    assert rel(O.layer_forward(x, O.Layer(raw)), dense) <= 1e-12


def test_zero_adapters_reduce_to_plain_int4_moe():
    raw, _ = small_layer()
    x = tokens(SMALL)
    zero_b = dict(raw)
    for p in range(3):
        zero_b[f"lb{p}"] = np.zeros_like(raw[f"lb{p}"])
    y0 = O.layer_forward(x, O.Layer(zero_b))
    # the output no longer depends on A
    other_a = dict(zero_b)
    for p in range(3):
        other_a[f"la{p}"] = synth.f32_to_bf16_bits(
            np.random.default_rng(9 + p).standard_normal(raw[f"la{p}"].shape).astype(np.float32))
    assert np.array_equal(O.layer_forward(x, O.Layer(other_a)), y0)
    # s = 0 gives the same layer
    s0 = dict(raw)
    s0["cfg"] = dataclasses.replace(SMALL, lora_scale=0.0)
    assert rel(O.layer_forward(x, O.Layer(s0)), y0) <= 1e-14
    # and every token equals the plain int4 SwiGLU experts mixed by the gates (torch)
    L0 = O.Layer(zero_b)
    logits = O.router_logits(x, L0)
    ids = O.topk(logits, SMALL.k)
    gam = O.gates(logits, ids)
    ref = np.zeros_like(x)
    for t in range(SMALL.T):
        for j in range(SMALL.k):
            P = L0.expert(int(ids[t, j]))
            ref[t] += gam[t, j] * _torch_dense_ffn(x[t:t + 1], P, 0.0)[0]
    assert rel(y0, ref) <= 1e-12


def test_token_permutation_equivariance():
    raw, L = small_layer()
    x = tokens(SMALL)
    pi = np.random.default_rng(10).permutation(SMALL.T)
    y, c = O.layer_forward(x, L, want_cache=True)
    yp, cp = O.layer_forward(x[pi], L, want_cache=True)
    assert np.array_equal(cp["ids"], c["ids"][pi])
    assert np.allclose(cp["gates"], c["gates"][pi], rtol=0, atol=1e-15)
    assert rel(yp, y[pi]) <= 1e-13


def test_output_affine_in_down_adapter_b():
    raw, L = small_layer()
    x = tokens(SMALL)
    ids = O.topk(O.router_logits(x, L), SMALL.k)
    y1 = O.layer_forward(x, L, ids=ids)
    for e in range(SMALL.E):
        L.expert(e)["Bd"] = 3.0 * L.expert(e)["Bd"]
    y3 = O.layer_forward(x, L, ids=ids)
    for e in range(SMALL.E):
        L.expert(e)["Bd"] = 0.0 * L.expert(e)["Bd"]
    y0 = O.layer_forward(x, L, ids=ids)
    assert rel(y3 - y0, 3.0 * (y1 - y0)) <= 1e-12
    assert np.sqrt(np.mean((y1 - y0) ** 2)) > 1e-6 * np.sqrt(np.mean(y0 ** 2))


# ---------------------------------------------------------------- coupling


def test_coupling_inverse_reconstructs_inputs():
    cfgF = SMALL
    cfgG = dataclasses.replace(SMALL, seed=1)
    F = O.Layer(synth.make_layer(cfgF, 0))
    G = O.Layer(synth.make_layer(cfgG, 1))
    x1 = tokens(SMALL, 2)
    x2 = tokens(SMALL, 3)
    y1, y2 = O.coupling_forward(x1, x2, F, G)
    r1, r2 = O.coupling_inverse(y1, y2, F, G)
    assert rel(r1, x1) <= 1e-12 and rel(r2, x2) <= 1e-12
    # the blocks really mix: outputs differ from inputs
    assert rel(y1, x1) > 1e-3 and rel(y2, x2) > 1e-3


# ---------------------------------------------------------------- backward


def _loss(x, dy, L):
    return float(np.sum(dy * O.layer_forward(x, L)))


def test_layer_backward_finite_differences():
    cfg = SMALL
    raw, L = small_layer(cfg)
    x = tokens(cfg)
    dy = np.random.default_rng(11).standard_normal((cfg.T, cfg.d))
    logits = O.router_logits(x, L)
    assert np.min(O.routing_gap(logits, cfg.k)) > 1e-4             # FD steps never cross a routing boundary
    dx, dA, dB = O.layer_backward(x, dy, L)
    eps = 1e-6
    rng = np.random.default_rng(12)
    names = [("Ag", "Bg"), ("Au", "Bu"), ("Ad", "Bd")]

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + eps
        lp = _loss(x, dy, L)
        arr[idx] = old - eps
        lm = _loss(x, dy, L)
        arr[idx] = old
        return (lp - lm) / (2 * eps)

    checked = 0
    for e in range(cfg.E):
        P = L.expert(e)
        for p, (an, bn) in enumerate(names):
            for _ in range(3):
                i = int(rng.integers(P[an].shape[0]))
                j = int(rng.integers(P[an].shape[1]))
                got = dA[p][e][j, i]                             # dA stored as A^T [r][in]
                ref = fd(P[an], (i, j))
                assert abs(got - ref) <= 1e-6 * max(1.0, abs(ref)), (e, an, i, j, got, ref)
                i = int(rng.integers(P[bn].shape[0]))
                j = int(rng.integers(P[bn].shape[1]))
                got = dB[p][e][j, i]                             # dB stored as B^T [out][r]
                ref = fd(P[bn], (i, j))
                assert abs(got - ref) <= 1e-6 * max(1.0, abs(ref)), (e, bn, i, j, got, ref)
                checked += 2
    for _ in range(40):
        t = int(rng.integers(cfg.T))
        i = int(rng.integers(cfg.d))
        ref = fd(x, (t, i))
        assert abs(dx[t, i] - ref) <= 1e-6 * max(1.0, abs(ref)), (t, i, dx[t, i], ref)
    assert checked > 0


def test_block_backward_reversible_equals_stored_and_finite_differences():
    cfgG = dataclasses.replace(SMALL, seed=1)
    F = O.Layer(synth.make_layer(SMALL, 0))
    G = O.Layer(synth.make_layer(cfgG, 1))
    x1 = tokens(SMALL, 2)
    x2 = tokens(SMALL, 3)
    rng = np.random.default_rng(13)
    dy1 = rng.standard_normal(x1.shape)
    dy2 = rng.standard_normal(x1.shape)
    y1, y2 = O.coupling_forward(x1, x2, F, G)
    rev = O.block_backward(y1, y2, dy1, dy2, F, G)
    sto = O.block_backward_stored(x1, x2, dy1, dy2, F, G)
    assert rel(rev["x1"], x1) <= 1e-12 and rel(rev["x2"], x2) <= 1e-12
    for key in ("dx1", "dx2"):
        assert rel(rev[key], sto[key]) <= 1e-12
    for key in ("dA_F", "dB_F", "dA_G", "dB_G"):
        for p in range(3):
            assert rel(rev[key][p], sto[key][p]) <= 1e-12


def test_block_backward_finite_differences():
    # the block gradient dz1 = dy1 + J_G^T dy2, dx2 = dy2 + J_F^T dz1 against
    # central differences of L = <dy1, y1> + <dy2, y2>; the bf16 rounding at G's
    # input is switched off so that L is smooth in x1, x2 and the adapters.
    cfgG = dataclasses.replace(SMALL, seed=1)
    F = O.Layer(synth.make_layer(SMALL, 0))
    G = O.Layer(synth.make_layer(cfgG, 1))
    x1 = tokens(SMALL, 2)
    x2 = tokens(SMALL, 3)
    rng = np.random.default_rng(14)
    dy1 = rng.standard_normal(x1.shape)
    dy2 = rng.standard_normal(x1.shape)
    y1, y2 = O.coupling_forward(x1, x2, F, G, round_g_input=False)
    assert np.min(O.routing_gap(O.router_logits(x2, F), SMALL.k)) > 1e-4
    assert np.min(O.routing_gap(O.router_logits(y1, G), SMALL.k)) > 1e-4
    res = O.block_backward(y1, y2, dy1, dy2, F, G, round_g_input=False)
    eps = 1e-6

    def loss():
        u1, u2 = O.coupling_forward(x1, x2, F, G, round_g_input=False)
        return float(np.sum(dy1 * u1) + np.sum(dy2 * u2))

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + eps
        lp = loss()
        arr[idx] = old - eps
        lm = loss()
        arr[idx] = old
        return (lp - lm) / (2 * eps)

    for _ in range(8):
        t = int(rng.integers(SMALL.T))
        i = int(rng.integers(SMALL.d))
        for arr, key in ((x1, "dx1"), (x2, "dx2")):
            ref = fd(arr, (t, i))
            assert abs(res[key][t, i] - ref) <= 1e-6 * max(1.0, abs(ref))
    for Lyr, tag in ((F, "F"), (G, "G")):
        for _ in range(4):
            e = int(rng.integers(SMALL.E))
            P = Lyr.expert(e)
            for p, (an, bn) in enumerate((("Ag", "Bg"), ("Au", "Bu"), ("Ad", "Bd"))):
                i = int(rng.integers(P[an].shape[0]))
                j = int(rng.integers(P[an].shape[1]))
                ref = fd(P[an], (i, j))
                assert abs(res[f"dA_{tag}"][p][e][j, i] - ref) <= 1e-6 * max(1.0, abs(ref))
                i = int(rng.integers(P[bn].shape[0]))
                j = int(rng.integers(P[bn].shape[1]))
                ref = fd(P[bn], (i, j))
                assert abs(res[f"dB_{tag}"][p][e][j, i] - ref) <= 1e-6 * max(1.0, abs(ref))


# ---------------------------------------------------------------- reversible stack


def _stack_blocks(L, cfg=SMALL):
    """L blocks of independent small layers (seeds 0, 1, ..., 2L-1)."""
    return [(O.Layer(synth.make_layer(dataclasses.replace(cfg, seed=2 * l), 2 * l)),
             O.Layer(synth.make_layer(dataclasses.replace(cfg, seed=2 * l + 1), 2 * l + 1))) for l in range(L)]


def test_stack_of_one_block_is_the_coupling():
    # with one block the stack is the (separately pinned) coupling and its backward
    blocks = _stack_blocks(1)
    F, G = blocks[0]
    x1, x2 = tokens(SMALL, 2), tokens(SMALL, 3)
    rng = np.random.default_rng(21)
    dy1, dy2 = rng.standard_normal(x1.shape), rng.standard_normal(x1.shape)
    s1, s2 = O.stack_forward(x1, x2, blocks)
    c1, c2 = O.coupling_forward(x1, x2, F, G)
    assert rel(s1, c1) <= 1e-14 and rel(s2, c2) <= 1e-14
    st = O.stack_backward(s1, s2, dy1, dy2, blocks)
    bl = O.block_backward(c1, c2, dy1, dy2, F, G)
    for key in ("x1", "x2", "dx1", "dx2"):
        assert rel(st[key], bl[key]) <= 1e-12, key
    for i, key in enumerate(("dA_F", "dB_F", "dA_G", "dB_G")):
        for p in range(3):
            assert rel(st["grads"][0][i][p], bl[key][p]) <= 1e-12, (key, p)


def test_stack_inverse_reconstructs_inputs():
    blocks = _stack_blocks(3)
    x1, x2 = tokens(SMALL, 2), tokens(SMALL, 3)
    y1, y2 = O.stack_forward(x1, x2, blocks)
    assert rel(y1, x1) > 1e-3                     # the stack does change the streams
    r1, r2 = O.stack_inverse(y1, y2, blocks)
    # exact up to fp64 rounding: each subtraction loses at most half an ulp of
    # the larger stream, and these small random layers let the streams grow
    bound = 8 * 3 * 2.0 ** -52 * max(np.abs(y1).max(), np.abs(y2).max())
    assert np.abs(r1 - x1).max() <= bound and np.abs(r2 - x2).max() <= bound


def test_stack_reversible_backward_equals_stored():
    blocks = _stack_blocks(3)
    x1, x2 = tokens(SMALL, 2), tokens(SMALL, 3)
    rng = np.random.default_rng(22)
    dy1, dy2 = rng.standard_normal(x1.shape), rng.standard_normal(x1.shape)
    y1, y2 = O.stack_forward(x1, x2, blocks)
    rev = O.stack_backward(y1, y2, dy1, dy2, blocks)
    sto = O.stack_backward_stored(x1, x2, dy1, dy2, blocks)
    bound = 8 * 3 * 2.0 ** -52 * max(np.abs(y1).max(), np.abs(y2).max())
    assert np.abs(rev["x1"] - x1).max() <= bound and np.abs(rev["x2"] - x2).max() <= bound
    for key in ("dx1", "dx2"):
        assert rel(rev[key], sto[key]) <= 1e-9, key
    for l in range(3):
        for i in range(4):
            for p in range(3):
                assert rel(rev["grads"][l][i][p], sto["grads"][l][i][p]) <= 1e-9, (l, i, p)


def test_stack_backward_finite_differences():
    # central differences of <dy1, y1> + <dy2, y2> through two blocks (bf16
    # roundings of the layer inputs off, so that the loss is smooth)
    blocks = _stack_blocks(2)
    x1, x2 = tokens(SMALL, 2), tokens(SMALL, 3)
    rng = np.random.default_rng(23)
    dy1, dy2 = rng.standard_normal(x1.shape), rng.standard_normal(x1.shape)
    y1, y2 = O.stack_forward(x1, x2, blocks, round_inputs=False)
    res = O.stack_backward(y1, y2, dy1, dy2, blocks, round_inputs=False)
    eps = 1e-6

    def loss():
        u1, u2 = O.stack_forward(x1, x2, blocks, round_inputs=False)
        return float(np.sum(dy1 * u1) + np.sum(dy2 * u2))

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + eps
        lp = loss()
        arr[idx] = old - eps
        lm = loss()
        arr[idx] = old
        return (lp - lm) / (2 * eps)

    for _ in range(6):
        t = int(rng.integers(SMALL.T))
        i = int(rng.integers(SMALL.d))
        for arr, key in ((x1, "dx1"), (x2, "dx2")):
            ref = fd(arr, (t, i))
            assert abs(res[key][t, i] - ref) <= 1e-6 * max(1.0, abs(ref)), (key, t, i)
    for l, (F, G) in enumerate(blocks):
        for Lyr, gi in ((F, 0), (G, 2)):
            e = int(rng.integers(SMALL.E))
            P = Lyr.expert(e)
            for p, (an, bn) in enumerate((("Ag", "Bg"), ("Au", "Bu"), ("Ad", "Bd"))):
                i = int(rng.integers(P[an].shape[0]))
                j = int(rng.integers(P[an].shape[1]))
                ref = fd(P[an], (i, j))
                assert abs(res["grads"][l][gi][p][e][j, i] - ref) <= 1e-6 * max(1.0, abs(ref)), (l, gi, p)
                i = int(rng.integers(P[bn].shape[0]))
                j = int(rng.integers(P[bn].shape[1]))
                ref = fd(P[bn], (i, j))
                assert abs(res["grads"][l][gi + 1][p][e][j, i] - ref) <= 1e-6 * max(1.0, abs(ref)), (l, gi + 1, p)


# ---------------------------------------------------------------- adapter optimizer


def test_adamw_matches_torch_adamw_over_several_steps():
    # torch.optim.AdamW implements the same update (decoupled weight decay,
    # bias-corrected moments); run both in fp64 on the same gradient sequence
    import torch
    rng = np.random.default_rng(41)
    n = 257
    p0 = rng.standard_normal(n) * 0.05
    lr, b1, b2, eps, wd = 3e-3, 0.9, 0.999, 1e-8, 0.01
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 7):
        g = rng.standard_normal(n) * (0.1 if t % 2 else 3.0)
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = O.adamw_step(p, m, v, g, lr, b1, b2, eps, wd, t)
        st = opt.state[tp]
        assert np.max(np.abs(p - tp.detach().numpy())) <= 1e-14
        assert np.max(np.abs(m - st["exp_avg"].numpy())) <= 1e-15
        assert np.max(np.abs(v - st["exp_avg_sq"].numpy())) <= 1e-15


def test_adamw_first_step_and_weight_decay_closed_forms():
    rng = np.random.default_rng(42)
    n = 64
    p0 = rng.standard_normal(n)
    g = rng.standard_normal(n)
    lr, b1, b2, eps, wd = 1e-2, 0.8, 0.95, 1e-6, 0.1
    # step 1: the bias-corrected moments are g and g^2
    p, m, v = O.adamw_step(p0, np.zeros(n), np.zeros(n), g, lr, b1, b2, eps, wd, 1)
    assert np.allclose(p, p0 - lr * (g / (np.abs(g) + eps) + wd * p0), rtol=0, atol=1e-15)
    assert np.allclose(m, (1 - b1) * g, rtol=0, atol=1e-16) and np.allclose(v, (1 - b2) * g * g, rtol=0, atol=1e-16)
    # no gradient: only the decoupled decay acts, p <- p (1 - lr wd) each step
    q, mq, vq = p0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 5):
        q, mq, vq = O.adamw_step(q, mq, vq, np.zeros(n), lr, b1, b2, eps, wd, t)
    assert np.allclose(q, p0 * (1 - lr * wd) ** 4, rtol=1e-15, atol=0)
    # grad_scale multiplies the gradient before anything else
    a = O.adamw_step(p0, np.zeros(n), np.zeros(n), g, lr, b1, b2, eps, wd, 1, grad_scale=0.5)
    b = O.adamw_step(p0, np.zeros(n), np.zeros(n), 0.5 * g, lr, b1, b2, eps, wd, 1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
