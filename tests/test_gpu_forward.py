"""GPU parity of the forward path (route, permute, router GEMM, grouped FFN,
combine, layer, reversible coupling) against the fp64 oracle.

Bars: expert ids, permutation and offsets bit-exact given the same fp32
logits; gates within 1e-6; router logits max|err|/RMS <= 1e-4 (tensor-core fp32
accumulation over up to 3*d/16 steps, see ROUTER_TOL); layer and FFN
outputs max|err|/RMS(ref) <= 2e-2 (for bf16 outputs: error beyond the half-ulp
rounding of the output format, see rel_err_bf16_out); reconstruction max|x - inv(fwd(x))|/RMS(x)
<= 5e-3. Tokens whose oracle routing gap is below a margin are "near ties":
either choice is correct there, so they are compared by validity of the chosen
set, not element by element.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O
from tests.gpu_util import (dev, dev_bf16, dev_f16, host_bf16, host_f16, near_tie_tokens, rel_err, rel_err_bf16_out,
                            stream_grid)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_moe_b200 as Q

RAGGED = synth.LayerConfig("ragged", T=300, d=256, E=10, k=3, f=192, g=64, r=16)
ONE = synth.LayerConfig("one", T=37, d=128, E=1, k=1, f=64, g=32, r=8)
ALLK = synth.LayerConfig("allk", T=50, d=128, E=4, k=4, f=128, g=128, r=0)
# group 256 (one scale row spans two 128-wide K stages of the down projection) and
# the largest rank (the gate/up rank-space contraction spans two 64-wide stages)
G256 = synth.LayerConfig("g256", T=200, d=256, E=6, k=2, f=256, g=256, r=8)
R64 = synth.LayerConfig("r64", T=150, d=256, E=5, k=2, f=256, g=64, r=64)
SMALL_CFGS = [synth.TINY, RAGGED, ONE, ALLK, G256, R64, synth.MID]
# int8 base weights (TQP Quantization: int8 or int4): codes one byte each, q * s
# rounded once to fp16; group 32 (two scale groups per 64-wide K stage), rank 0
INT8_CFGS = [synth.LayerConfig("i8", T=300, d=256, E=10, k=3, f=256, g=64, r=16, bits=8),
             synth.LayerConfig("i8g32", T=200, d=128, E=6, k=2, f=128, g=32, r=0, bits=8),
             dataclasses.replace(synth.MID, name="mid_i8", bits=8)]
TOL = 2e-2
# The router's products are exact (bf16 x times an exact 3-part bf16 split of
# the fp32 weights); its error is the tensor cores' fp32 accumulation, at most
# about 2^-23 of the running sum per K=16 step, 3*d/16 = 384 steps at d=2048.
ROUTER_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    Q.lib()


# ---------------------------------------------------------------- routing


ROUTE_SHAPES = [(64, 8, 2), (2048, 64, 8), (8192, 460, 12), (1, 5, 5), (33, 1, 1), (300, 23, 23), (129, 700, 16)]


@pytest.mark.parametrize("T,E,k", ROUTE_SHAPES)
@pytest.mark.parametrize("ties", [False, True])
def test_route_bitexact(T, E, k, ties):
    l = synth.make_logits(T, E, seed=T + E, ties=ties)
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gates = torch.empty(T, k, dtype=torch.float32, device="cuda")
    st = Q.Status()
    Q.moe_route(dev(l), k, ids, gates, st)
    ref_ids = O.topk(l, k)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    ref_g = O.gates(l, ref_ids)
    assert np.max(np.abs(gates.cpu().numpy() - ref_g)) <= 1e-6
    assert st.read() == 0


def test_route_skewed_bias_bitexact():
    bias = synth.zipf_bias(460, 1.1)
    l = synth.make_logits(16384, 460, seed=3, bias=bias)
    ids = torch.empty(16384, 12, dtype=torch.int32, device="cuda")
    gates = torch.empty(16384, 12, dtype=torch.float32, device="cuda")
    Q.moe_route(dev(l), 12, ids, gates)
    ref = O.topk(l, 12)
    assert np.array_equal(ids.cpu().numpy(), ref)
    assert np.max(np.abs(gates.cpu().numpy() - O.gates(l, ref))) <= 1e-6


def test_route_nonfinite_sets_status_and_ranks_nan_last():
    l = synth.make_logits(40, 16, seed=9)
    l[3, 5] = np.nan
    l[7, 2] = np.inf
    l[9, :] = -np.inf
    l[9, 4] = 0.5
    ids = torch.empty(40, 4, dtype=torch.int32, device="cuda")
    gates = torch.empty(40, 4, dtype=torch.float32, device="cuda")
    st = Q.Status()
    Q.moe_route(dev(l), 4, ids, gates, st)
    assert st.read() & Q.STATUS_NONFINITE
    got = ids.cpu().numpy()
    ref = O.topk(l, 4)
    assert np.array_equal(got, ref)
    assert 5 not in got[3]


def test_route_rejects_bad_arguments():
    l = torch.zeros(4, 8, device="cuda")
    ids = torch.empty(4, 2, dtype=torch.int32, device="cuda")
    gates = torch.empty(4, 2, device="cuda")
    with pytest.raises(Q.TQPError):
        Q.moe_route(l, 9, ids, gates)                 # k > E
    with pytest.raises(Q.TQPError):
        Q.moe_route(l, 0, ids, gates)


# ---------------------------------------------------------------- permutation


def _ids_for(T, E, k, seed, skew=False):
    bias = synth.zipf_bias(E, 1.1) if skew else None
    return O.topk(synth.make_logits(T, E, seed=seed, bias=bias), k)


PERM_CASES = [(64, 8, 2, False), (2048, 64, 8, False), (8192, 460, 12, False), (16384, 460, 12, True),
              (1, 3, 2, False), (31, 1, 1, False), (33, 40, 40, False), (1000, 4096, 3, True)]


@pytest.mark.parametrize("T,E,k,skew", PERM_CASES)
def test_permute_bitexact(T, E, k, skew):
    ids = _ids_for(T, E, k, seed=T * 7 + E, skew=skew)
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    st = Q.Status()
    Q.moe_permute(dev(ids), E, offsets, perm, inv, status=st)
    r_off, r_perm, r_inv = O.permute(ids, E)
    assert np.array_equal(offsets.cpu().numpy(), r_off)
    assert np.array_equal(perm.cpu().numpy(), r_perm)
    assert np.array_equal(inv.cpu().numpy(), r_inv)
    assert st.read() == 0
    if skew:
        counts = np.diff(r_off)
        assert counts.max() > 4 * counts.mean() and (counts == 0).any()


def test_permute_bad_id_sets_status():
    ids = _ids_for(64, 8, 2, seed=1)
    ids[5, 1] = 8
    ids[9, 0] = -3
    offsets = torch.empty(9, dtype=torch.int32, device="cuda")
    perm = torch.empty(128, dtype=torch.int32, device="cuda")
    inv = torch.empty(128, dtype=torch.int32, device="cuda")
    st = Q.Status()
    Q.moe_permute(dev(ids), 8, offsets, perm, inv, status=st)
    assert st.read() & Q.STATUS_BAD_ID
    assert offsets.cpu().numpy()[-1] == 126


def test_permute_empty_batch():
    offsets = torch.full((9,), 7, dtype=torch.int32, device="cuda")
    e = torch.empty(0, 2, dtype=torch.int32, device="cuda")
    Q.moe_permute(e, 8, offsets, torch.empty(0, dtype=torch.int32, device="cuda"),
                  torch.empty(0, dtype=torch.int32, device="cuda"))
    assert offsets.cpu().numpy().tolist() == [0] * 9


# ---------------------------------------------------------------- router GEMM


_LAYERS = {}


def host_layer(cfg, seed=None):
    key = (cfg, seed)
    if key not in _LAYERS:
        _LAYERS[key] = synth.make_layer(cfg, seed)
    return _LAYERS[key]


def device_layer(cfg, seed=None):
    key = ("dev", cfg, seed)
    if key not in _LAYERS:
        _LAYERS[key] = Q.DeviceLayer(host_layer(cfg, seed))
    return _LAYERS[key]


@pytest.mark.parametrize("cfg", SMALL_CFGS + [synth.FULL], ids=lambda c: c.name)
def test_router_gemm(cfg):
    raw = host_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, 11)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device="cuda")
    Q.moe_router_gemm(dev_bf16(xb), device_layer(cfg), logits)
    ref = O.router_logits(O.bf16_to_f64(xb), L)
    assert rel_err(logits.cpu().numpy(), ref) <= ROUTER_TOL


def test_router_gemm_bias():
    cfg = dataclasses.replace(RAGGED, zipf_s=1.1)
    raw = synth.make_layer(cfg)
    xb = synth.make_tokens(cfg.T, cfg.d, 12)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device="cuda")
    Q.moe_router_gemm(dev_bf16(xb), Q.DeviceLayer(raw), logits)
    ref = O.router_logits(O.bf16_to_f64(xb), O.Layer(raw))
    assert np.max(np.abs(logits.cpu().numpy() - ref)) <= ROUTER_TOL * np.sqrt(np.mean(ref ** 2))


# ---------------------------------------------------------------- grouped FFN


def _ffn_case(cfg, x64, L, ids):
    offsets, perm, inv = O.permute(ids, cfg.E)
    return offsets.astype(np.int32), perm.astype(np.int32), inv.astype(np.int32)


def _run_ffn(cfg, xb, offsets, perm):
    A = cfg.T * cfg.k
    h = torch.empty(A, cfg.f, dtype=torch.int16, device="cuda")
    o = torch.empty(A, cfg.d, dtype=torch.int16, device="cuda")
    st = Q.Status()
    Q.tqp_grouped_ffn(dev_bf16(xb), dev(offsets), dev(perm), device_layer(cfg), h, o, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    return h, o


@pytest.mark.parametrize("cfg", [synth.TINY, RAGGED, synth.MID], ids=lambda c: c.name)
def test_grouped_ffn_parts_equal_whole_call(cfg):
    """The four parts issued in order give bit-identical h and out_perm."""
    xb = synth.make_tokens(cfg.T, cfg.d, 14)
    x = O.bf16_to_f64(xb)
    L = O.Layer(host_layer(cfg))
    ids = O.topk(O.router_logits(x, L), cfg.k)
    offsets, perm, _ = _ffn_case(cfg, x, L, ids)
    h1, o1 = _run_ffn(cfg, xb, offsets, perm)
    A = cfg.T * cfg.k
    h2 = torch.empty(A, cfg.f, dtype=torch.int16, device="cuda")
    o2 = torch.empty(A, cfg.d, dtype=torch.int16, device="cuda")
    layer = device_layer(cfg)
    ws = Q.workspace(Q.lib().tqp_grouped_ffn_workspace_size(cfg.T, layer.ref()), h2.device)
    st = Q.Status()
    xd, od, pd = dev_bf16(xb), dev(offsets), dev(perm)
    for part in (Q.FFN_PREPARE, Q.FFN_GATE_UP, Q.FFN_RANK, Q.FFN_DOWN):
        Q.tqp_grouped_ffn_part(part, xd, od, pd, layer, h2, o2, ws, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    assert torch.equal(h1, h2) and torch.equal(o1, o2)


@pytest.mark.parametrize("cfg", SMALL_CFGS + INT8_CFGS, ids=lambda c: c.name)
def test_grouped_ffn_matches_oracle(cfg):
    raw = host_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, 13)
    x = O.bf16_to_f64(xb)
    ids = O.topk(O.router_logits(x, L), cfg.k)
    offsets, perm, _ = _ffn_case(cfg, x, L, ids)
    h, o = _run_ffn(cfg, xb, offsets, perm)
    hg, og = host_f16(h), host_f16(o)
    href = np.zeros_like(hg)
    oref = np.zeros_like(og)
    for e in range(cfg.E):
        rows = np.arange(offsets[e], offsets[e + 1])
        if len(rows) == 0:
            continue
        out = O.expert_forward(x[perm[rows]], L.expert(e), L.s)
        href[rows] = out["h"]
        oref[rows] = out["o"]
    assert rel_err(hg, href) <= TOL
    assert rel_err(og, oref) <= TOL


def test_grouped_ffn_skewed_and_empty_experts():
    # one expert takes most rows (several 256-row blocks, ragged tail), several get none
    cfg = synth.LayerConfig("skew", T=700, d=256, E=12, k=2, f=128, g=64, r=16)
    raw = host_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, 14)
    x = O.bf16_to_f64(xb)
    ids = np.zeros((cfg.T, 2), dtype=np.int32)
    ids[:, 0] = 3
    ids[:, 1] = np.where(np.arange(cfg.T) % 5 == 0, 7, np.where(np.arange(cfg.T) % 7 == 0, 0, 9))
    offsets, perm, _ = _ffn_case(cfg, x, L, ids)
    h, o = _run_ffn(cfg, xb, offsets, perm)
    og = host_f16(o)
    oref = np.zeros_like(og)
    for e in range(cfg.E):
        rows = np.arange(offsets[e], offsets[e + 1])
        if len(rows):
            oref[rows] = O.expert_forward(x[perm[rows]], L.expert(e), L.s)["o"]
    assert rel_err(og, oref) <= TOL


@pytest.mark.parametrize("cfg", [synth.FULL, synth.SKEWED], ids=lambda c: c.name)
def test_grouped_ffn_full_size_sampled_experts(cfg):
    """Every row of at least 16 experts at full size: the busiest, the
    least-loaded non-empty one, one whose rows span three or more of the down
    kernel's 256-row blocks (when the load has one) and random others."""
    raw = host_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, cfg.seed)
    x = O.bf16_to_f64(xb)
    ids = O.topk(O.router_logits(x, L), cfg.k)
    offsets, perm, _ = _ffn_case(cfg, x, L, ids)
    h, o = _run_ffn(cfg, xb, offsets, perm)
    hg_all, og_all = host_f16(h), host_f16(o)
    counts = np.diff(offsets)
    nz = np.nonzero(counts)[0]
    picks = [int(np.argmax(counts)), int(nz[np.argmin(counts[nz])])]
    wide = np.nonzero((counts > 512) & (counts <= 4096))[0]
    if len(wide):
        picks.append(int(wide[0]))
    rng = np.random.default_rng(1)
    picks += [int(e) for e in rng.choice(nz, 16, replace=False)]
    picks = list(dict.fromkeys(picks))
    assert len(picks) >= 16
    for e in picks:
        rows = np.arange(offsets[e], offsets[e + 1])
        out = O.expert_forward(x[perm[rows]], L.expert(e), L.s)
        assert rel_err(og_all[rows], out["o"]) <= TOL, (e, len(rows))
        assert rel_err(hg_all[rows], out["h"]) <= TOL, (e, len(rows))


# ---------------------------------------------------------------- combine


def test_combine_and_coupling_epilogue():
    cfg = RAGGED
    rng = np.random.default_rng(5)
    T, k, d = cfg.T, cfg.k, cfg.d
    ids = _ids_for(T, cfg.E, k, seed=2)
    _, _, inv = O.permute(ids, cfg.E)
    gam = O.gates(synth.make_logits(T, cfg.E, 2), ids).astype(np.float32)
    ob = rng.standard_normal((T * k, d)).astype(np.float16)
    res = rng.standard_normal((T, d)).astype(np.float32)
    y = torch.empty(T, d, dtype=torch.int16, device="cuda")
    Q.moe_combine(dev_f16(ob), dev(inv.astype(np.int32)), dev(gam), y)
    ref = O.combine(ob.astype(np.float64), gam.astype(np.float64), inv, T, k)
    # bf16 output: round-to-nearest error <= 2^-9 |ref| (2^-8 leaves room for the fp32 sum)
    assert np.all(np.abs(host_bf16(y) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
    # coupling form: y = residual - bf16(sum), fp32 out, plus a bf16 copy
    yf = torch.empty(T, d, dtype=torch.float32, device="cuda")
    yb = torch.empty(T, d, dtype=torch.int16, device="cuda")
    Q.moe_combine(dev_f16(ob), dev(inv.astype(np.int32)), dev(gam), yf, residual=dev(res), sign=-1.0, y_bf16=yb)
    m = host_bf16(y)
    assert np.array_equal(yf.cpu().numpy(), (res - m.astype(np.float32)).astype(np.float32))
    assert np.array_equal(host_bf16(yb), O.round_bf16(yf.cpu().numpy().astype(np.float64)))


# ---------------------------------------------------------------- full layer


def _layer_check(cfg, raw, xb, y_dev, margin=1e-4):
    L = O.Layer(raw)
    x = O.bf16_to_f64(xb)
    logits = O.router_logits(x, L)
    ties = near_tie_tokens(logits, cfg.k, margin)
    ref = O.layer_forward(x, L)
    got = host_bf16(y_dev)
    keep = ~ties
    err = rel_err_bf16_out(got[keep], ref[keep])
    assert err <= TOL, (err, int(ties.sum()))
    return ties


@pytest.mark.parametrize("cfg", SMALL_CFGS + INT8_CFGS, ids=lambda c: c.name)
def test_layer_fwd_matches_oracle(cfg):
    raw = host_layer(cfg)
    xb = synth.make_tokens(cfg.T, cfg.d, 21)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.int16, device="cuda")
    st = Q.Status()
    Q.tqp_moe_layer_fwd(dev_bf16(xb), device_layer(cfg), y, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    ties = _layer_check(cfg, raw, xb, y)
    assert ties.mean() < 0.01


def test_layer_fwd_deterministic():
    cfg = synth.MID
    xb = dev_bf16(synth.make_tokens(cfg.T, cfg.d, 22))
    outs = []
    for _ in range(3):
        y = torch.empty(cfg.T, cfg.d, dtype=torch.int16, device="cuda")
        Q.tqp_moe_layer_fwd(xb, device_layer(cfg), y)
        outs.append(y.cpu())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("cfg", [synth.FULL, synth.SKEWED], ids=lambda c: c.name)
def test_layer_fwd_full_size_sampled_tokens(cfg):
    """The whole layer at full size on 98 sampled tokens (the first, the last
    and 96 random ones), the oracle run on that subset of rows."""
    raw = host_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, cfg.seed)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.int16, device="cuda")
    st = Q.Status()
    Q.tqp_moe_layer_fwd(dev_bf16(xb), device_layer(cfg), y, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    got = host_bf16(y)
    x = O.bf16_to_f64(xb)
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(np.arange(1, cfg.T - 1), 96, replace=False)]))
    ref = O.layer_forward(x[toks], L)
    ok = O.routing_gap(O.router_logits(x[toks], L), cfg.k) >= 1e-4
    assert ok.sum() >= len(toks) - 2
    err = rel_err_bf16_out(got[toks][ok], ref[ok])
    assert err <= TOL, err
    # every output row is finite and the whole batch was written
    assert np.isfinite(got).all()


# ---------------------------------------------------------------- reversible coupling


def _rev_layers(cfgF, cfgG):
    return host_layer(cfgF, cfgF.seed), host_layer(cfgG, cfgG.seed)


REV_SMALL = (synth.TINY, dataclasses.replace(synth.TINY, seed=1))
REV_MID = (synth.LayerConfig("rev_mid", T=512, d=256, E=16, k=4, f=256, g=64, r=16),
           synth.LayerConfig("rev_mid", T=512, d=256, E=16, k=4, f=256, g=64, r=16, seed=1))


@pytest.mark.parametrize("cfgs", [REV_SMALL, REV_MID], ids=["tiny", "mid"])
def test_rev_couple_fwd_inverse(cfgs):
    cfgF, cfgG = cfgs
    rawF, rawG = _rev_layers(cfgF, cfgG)
    F, G = device_layer(cfgF, cfgF.seed), device_layer(cfgG, cfgG.seed)
    T, d = cfgF.T, cfgF.d
    x1b = synth.make_tokens(T, d, 2)
    x2b = synth.make_tokens(T, d, 3)
    y1 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    y2 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    st = Q.Status()
    Q.rev_couple_fwd(dev_bf16(x1b), dev_bf16(x2b), F, G, y1, y2, status=st)
    r1 = torch.empty(T, d, dtype=torch.int16, device="cuda")
    r2 = torch.empty(T, d, dtype=torch.int16, device="cuda")
    Q.rev_couple_inv(y1, y2, F, G, r1, r2, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    x1, x2 = O.bf16_to_f64(x1b), O.bf16_to_f64(x2b)
    rms = np.sqrt(np.mean(np.concatenate([x1, x2]) ** 2))
    err = max(np.max(np.abs(host_bf16(r1) - x1)), np.max(np.abs(host_bf16(r2) - x2))) / rms
    assert err <= 5e-3
    # forward values against the oracle (tokens away from routing ties in both layers)
    LF, LG = O.Layer(rawF), O.Layer(rawG)
    o1, _ = O.coupling_forward(x1, x2, LF, LG)
    f_ref = o1 - x1
    tieF = near_tie_tokens(O.router_logits(x2, LF), cfgF.k, 1e-4)
    # G reads bf16(y1) of the GPU's own y1: the oracle's G runs on exactly that
    # input, so G's branch is compared without F's rounding in between.
    z = O.round_bf16(y1.cpu().numpy().astype(np.float64))
    tieG = near_tie_tokens(O.router_logits(z, LG), cfgG.k, 1e-4)
    g_ref = O.layer_forward(z, LG)
    e1 = rel_err_bf16_out(y1.cpu().numpy()[~tieF] - x1[~tieF], f_ref[~tieF])
    e2 = rel_err_bf16_out(y2.cpu().numpy()[~tieG] - x2[~tieG], g_ref[~tieG])
    print(f"COUPLING {T}x{d}: y1 - x1 err {e1:.3e}, y2 - x2 err {e2:.3e} (tokens kept {np.mean(~tieF):.3f}, "
          f"{np.mean(~tieG):.3f})")
    assert np.mean(~tieF) > 0.95 and np.mean(~tieG) > 0.95
    assert e1 <= TOL, e1
    assert e2 <= TOL, e2


def test_rev_couple_full_size_reconstruction():
    cfgF, cfgG = synth.REV_F, synth.REV_G
    F, G = device_layer(cfgF, cfgF.seed), device_layer(cfgG, cfgG.seed)
    T, d = cfgF.T, cfgF.d
    x1 = dev_bf16(synth.make_tokens(T, d, synth.REV_SEEDS["x1"]))
    x2 = dev_bf16(synth.make_tokens(T, d, synth.REV_SEEDS["x2"]))
    y1 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    y2 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    st = Q.Status()
    Q.rev_couple_fwd(x1, x2, F, G, y1, y2, status=st)
    r1 = torch.empty_like(x1)
    r2 = torch.empty_like(x2)
    Q.rev_couple_inv(y1, y2, F, G, r1, r2, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    f = lambda t: t.view(torch.bfloat16).float()
    rms = torch.sqrt(torch.mean(torch.cat([f(x1), f(x2)]) ** 2))
    err = max((f(r1) - f(x1)).abs().max(), (f(r2) - f(x2)).abs().max()) / rms
    assert float(err) <= 5e-3
    # exact: the inverse returns the inputs on the stream grid bit for bit
    for r, x in ((r1, x1), (r2, x2)):
        assert np.array_equal(host_bf16(r), stream_grid(host_bf16(x)))


def test_rev_couple_stream_out_of_range_raises_range_status():
    """A stream value of magnitude 256 or more leaves the grid's exact range:
    the coupling raises TQP_STATUS_RANGE (and nothing else)."""
    cfgF, cfgG = REV_SMALL
    F, G = device_layer(cfgF, cfgF.seed), device_layer(cfgG, cfgG.seed)
    T, d = cfgF.T, cfgF.d
    x1b = synth.make_tokens(T, d, 2).copy()
    x1b[5, 7] = np.float32(300.0).view(np.uint32) >> 16        # bf16 300, exact
    x2b = synth.make_tokens(T, d, 3)
    y1 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    st = Q.Status()
    Q.rev_couple_fwd(dev_bf16(x1b), dev_bf16(x2b), F, G, y1, y2, status=st)
    torch.cuda.synchronize()
    assert st.read() == Q.STATUS_RANGE
    st = Q.Status()
    Q.rev_couple_fwd(dev_bf16(synth.make_tokens(T, d, 2)), dev_bf16(x2b), F, G, y1, y2, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
