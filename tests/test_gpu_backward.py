"""GPU parity of the backward path (layer backward, reversible block backward
with activation reconstruction) against the fp64 oracle.

Bars: dx, dA, dB max|err|/RMS(ref) <= 2e-2 per tensor; reconstruction of x1,
x2 from the block outputs max|x - rec|/RMS(x) <= 5e-3. Tokens whose routing is
ambiguous at the arithmetic's precision are excluded from the elementwise
comparison, and so are the experts they touch (their gradient sums would
differ by that token's contribution either way).

In the block tests G's input is bf16(y1) of the GPU's own forward output: the
backward reads exactly that, so both sides route G on the same bf16 values and
the comparison isolates the backward's arithmetic. (How far y1 itself is from
the oracle's forward is the forward tests' concern.)
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O
from tests.gpu_util import dev, dev_bf16, host_bf16, near_tie_tokens, rel_err, stream_grid

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_moe_b200 as Q

TOL = 2e-2
BW1 = synth.LayerConfig("bw1", T=300, d=256, E=10, k=3, f=256, g=64, r=16)
BW_ONE = synth.LayerConfig("bw_one", T=37, d=128, E=1, k=1, f=128, g=32, r=8)
BW_R0 = synth.LayerConfig("bw_r0", T=50, d=128, E=4, k=4, f=128, g=128, r=0)
BW_SKEW = synth.LayerConfig("bw_skew", T=600, d=256, E=12, k=2, f=256, g=64, r=16, zipf_s=1.1)
BW_I8 = synth.LayerConfig("bw_i8", T=300, d=256, E=10, k=3, f=256, g=64, r=16, bits=8)
BW_R32 = synth.LayerConfig("bw_r32", T=300, d=256, E=10, k=3, f=256, g=64, r=32)   # the full config's rank
LAYER_CFGS = [synth.TINY, BW1, BW_ONE, BW_R0, BW_SKEW, synth.MID, BW_I8, BW_R32]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    Q.lib()


def ambiguous_experts(logits, k, margin):
    """Experts at the k-th / (k+1)-th place of tokens whose gap is below margin."""
    tie = near_tie_tokens(logits, k, margin)
    srt = np.argsort(-logits[tie], axis=1, kind="stable")
    ex = set(srt[:, k - 1].tolist()) | set(srt[:, k].tolist()) if k < logits.shape[1] and tie.any() else set()
    return tie, ex


def gpu_layer_bwd(cfg, raw, xb, dy):
    L = Q.DeviceLayer(raw)
    dx = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    dA, dB, g = L.grads()
    st = Q.Status()
    Q.tqp_moe_layer_bwd(dev_bf16(xb), dev(dy), L, dx, g, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    return dx.cpu().numpy(), [t.cpu().numpy() for t in dA], [t.cpu().numpy() for t in dB]


@pytest.mark.parametrize("cfg", LAYER_CFGS, ids=lambda c: c.name)
def test_layer_bwd_matches_oracle(cfg):
    raw = synth.make_layer(cfg)
    L = O.Layer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, 31)
    dy = synth.make_grad(cfg.T, cfg.d, 32, "dy1")
    x = O.bf16_to_f64(xb)
    dx, dA, dB = gpu_layer_bwd(cfg, raw, xb, dy)
    rdx, rdA, rdB = O.layer_backward(x, dy.astype(np.float64), L)
    tie, amb = ambiguous_experts(O.router_logits(x, L), cfg.k, 1e-4)
    assert tie.mean() < 0.02
    assert rel_err(dx[~tie], rdx[~tie]) <= TOL
    keep = np.array([e not in amb for e in range(cfg.E)])
    if cfg.r > 0:
        for p in range(3):
            assert rel_err(dA[p][keep], rdA[p][keep]) <= TOL, ("dA", p)
            assert rel_err(dB[p][keep], rdB[p][keep]) <= TOL, ("dB", p)


def test_layer_bwd_rejects_ffn_not_multiple_of_128():
    cfg = synth.LayerConfig("f192", T=16, d=128, E=4, k=2, f=192, g=64, r=8)
    raw = synth.make_layer(cfg)
    with pytest.raises(Q.TQPError) as ei:
        gpu_layer_bwd(cfg, raw, synth.make_tokens(16, 128, 1), synth.make_grad(16, 128, 1, "dy1"))
    assert ei.value.code == -2


def test_layer_bwd_deterministic():
    cfg = BW1
    raw = synth.make_layer(cfg)
    xb = synth.make_tokens(cfg.T, cfg.d, 33)
    dy = synth.make_grad(cfg.T, cfg.d, 34, "dy1")
    a = gpu_layer_bwd(cfg, raw, xb, dy)
    b = gpu_layer_bwd(cfg, raw, xb, dy)
    assert np.array_equal(a[0], b[0])
    for p in range(3):
        assert np.array_equal(a[1][p], b[1][p]) and np.array_equal(a[2][p], b[2][p])


# ---------------------------------------------------------------- reversible block


REV_TINY = (synth.TINY, dataclasses.replace(synth.TINY, seed=1))
REV_MID = (synth.LayerConfig("rb", T=512, d=256, E=16, k=4, f=256, g=64, r=16),
           synth.LayerConfig("rb", T=512, d=256, E=16, k=4, f=256, g=64, r=16, seed=1))


def gpu_block(cfgF, cfgG, rawF, rawG, x1b, x2b, dy1, dy2):
    F, G = Q.DeviceLayer(rawF), Q.DeviceLayer(rawG)
    T, d = x1b.shape
    y1 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    st = Q.Status()
    Q.rev_couple_fwd(dev_bf16(x1b), dev_bf16(x2b), F, G, y1, y2, status=st)
    r1 = torch.empty(T, d, dtype=torch.int16, device="cuda")
    r2 = torch.empty_like(r1)
    dx1 = torch.empty(T, d, dtype=torch.float32, device="cuda")
    dx2 = torch.empty_like(dx1)
    dAF, dBF, gF = F.grads()
    dAG, dBG, gG = G.grads()
    Q.tqp_adapter_bwd(y1, y2, dev(dy1), dev(dy2), F, G, r1, r2, dx1, dx2, gF, gG, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    c = lambda ts: [t.cpu().numpy() for t in ts]
    return {"y1": y1.cpu().numpy(), "x1": host_bf16(r1), "x2": host_bf16(r2), "dx1": dx1.cpu().numpy(),
            "dx2": dx2.cpu().numpy(), "dA_F": c(dAF), "dB_F": c(dBF), "dA_G": c(dAG), "dB_G": c(dBG)}


def g_input(y1_gpu):
    """bf16(y1) of the GPU's fp32 y1: the input the block backward gives G."""
    return O.round_bf16(y1_gpu.astype(np.float64))


@pytest.mark.parametrize("cfgs", [REV_TINY, REV_MID], ids=["tiny", "mid"])
def test_adapter_bwd_block_matches_oracle(cfgs):
    cfgF, cfgG = cfgs
    rawF, rawG = synth.make_layer(cfgF, cfgF.seed), synth.make_layer(cfgG, cfgG.seed)
    T, d = cfgF.T, cfgF.d
    x1b, x2b = synth.make_tokens(T, d, 2), synth.make_tokens(T, d, 3)
    dy1, dy2 = synth.make_grad(T, d, 4, "dy1"), synth.make_grad(T, d, 4, "dy2")
    got = gpu_block(cfgF, cfgG, rawF, rawG, x1b, x2b, dy1, dy2)
    x1, x2 = O.bf16_to_f64(x1b), O.bf16_to_f64(x2b)
    # reconstruction is exact: the backward recomputes bit-identical F and G, and
    # the stream adds are exact on the stream grid
    rms = np.sqrt(np.mean(np.concatenate([x1, x2]) ** 2))
    assert max(np.max(np.abs(got["x1"] - x1)), np.max(np.abs(got["x2"] - x2))) / rms <= 5e-3
    assert np.array_equal(got["x1"], stream_grid(x1)) and np.array_equal(got["x2"], stream_grid(x2))
    LF, LG = O.Layer(rawF), O.Layer(rawG)
    z = g_input(got["y1"])
    dy1_, dy2_ = dy1.astype(np.float64), dy2.astype(np.float64)
    dxG, dAG, dBG = O.layer_backward(z, dy2_, LG)
    dz1 = dy1_ + dxG
    dxF, dAF, dBF = O.layer_backward(x2, dz1, LF)
    ref = {"dx1": dz1, "dx2": dy2_ + dxF, "dA_F": dAF, "dB_F": dBF, "dA_G": dAG, "dB_G": dBG}
    tieF, ambF = ambiguous_experts(O.router_logits(x2, LF), cfgF.k, 1e-4)
    tieG, ambG = ambiguous_experts(O.router_logits(z, LG), cfgG.k, 1e-4)
    # a G-ambiguous token also changes F's cotangent dz1 at that token, so F's experts of that token too
    if tieG.any():
        ambF |= set(O.topk(O.router_logits(x2[tieG], LF), cfgF.k).ravel().tolist())
    keep_t = ~(tieF | tieG)
    assert keep_t.mean() > 0.95
    kF = np.array([e not in ambF for e in range(cfgF.E)])
    kG = np.array([e not in ambG for e in range(cfgG.E)])
    assert kF.mean() >= 0.5 and kG.mean() >= 0.5, (kF.sum(), kG.sum())

    def check(key, sel, p=None):
        g = got[key] if p is None else got[key][p]
        r = ref[key] if p is None else ref[key][p]
        err = rel_err(g[sel], r[sel])
        print(f"BLOCK {cfgF.T}x{cfgF.d} {key}{'' if p is None else p}: err {err:.3e}")
        assert err <= TOL, (key, p, err)

    check("dx1", keep_t)
    check("dx2", keep_t)
    for p in range(3):
        for key, keep in (("dA_F", kF), ("dB_F", kF), ("dA_G", kG), ("dB_G", kG)):
            check(key, keep, p)


_FULL_BLOCK = {}


def full_block():
    """The 460-expert top-12 block (F, G independent instances) at T=8192, run
    once on the GPU (forward, then the adapter backward from its outputs)."""
    if not _FULL_BLOCK:
        cfgF, cfgG = synth.REV_F, synth.REV_G
        rawF, rawG = synth.make_layer(cfgF, cfgF.seed), synth.make_layer(cfgG, cfgG.seed)
        T, d = cfgF.T, cfgF.d
        x1b = synth.make_tokens(T, d, synth.REV_SEEDS["x1"])
        x2b = synth.make_tokens(T, d, synth.REV_SEEDS["x2"])
        dy1 = synth.make_grad(T, d, synth.REV_SEEDS["dy"], "dy1")
        dy2 = synth.make_grad(T, d, synth.REV_SEEDS["dy"], "dy2")
        got = gpu_block(cfgF, cfgG, rawF, rawG, x1b, x2b, dy1, dy2)
        _FULL_BLOCK.update(cfgF=cfgF, cfgG=cfgG, rawF=rawF, rawG=rawG, x1b=x1b, x2b=x2b, dy1=dy1, dy2=dy2, got=got)
    return _FULL_BLOCK


def test_adapter_bwd_full_size_reconstruction_and_sampled_tokens():
    """The 460-expert top-12 block at T=8192: reconstruction over all tokens,
    and dx1/dx2 on sampled tokens against the oracle evaluated token by token."""
    fb = full_block()
    cfgF, cfgG, rawF, rawG = fb["cfgF"], fb["cfgG"], fb["rawF"], fb["rawG"]
    x1b, x2b, dy1, dy2, got = fb["x1b"], fb["x2b"], fb["dy1"], fb["dy2"], fb["got"]
    T, d = cfgF.T, cfgF.d
    x1, x2 = O.bf16_to_f64(x1b), O.bf16_to_f64(x2b)
    rms = np.sqrt(np.mean(np.concatenate([x1, x2]) ** 2))
    assert max(np.max(np.abs(got["x1"] - x1)), np.max(np.abs(got["x2"] - x2))) / rms <= 5e-3
    assert np.array_equal(got["x1"], stream_grid(x1)) and np.array_equal(got["x2"], stream_grid(x2))
    assert all(np.isfinite(got[k]).all() for k in ("dx1", "dx2"))
    LF, LG = O.Layer(rawF), O.Layer(rawG)
    toks = [0, T - 1, 1234, 4321, 777, 6000, 100, 8000]
    ok_rows, g1, g2, r1s, r2s = [], [], [], [], []
    for t in toks:
        z = g_input(got["y1"][t:t + 1])
        amb = (O.routing_gap(O.router_logits(x2[t:t + 1], LF), cfgF.k)[0] < 1e-4) or \
            (O.routing_gap(O.router_logits(z, LG), cfgG.k)[0] < 1e-4)
        if amb:
            continue
        dy1t, dy2t = dy1[t:t + 1].astype(np.float64), dy2[t:t + 1].astype(np.float64)
        dz1 = dy1t + O.layer_backward(z, dy2t, LG)[0]
        ok_rows.append(t)
        g1.append(got["dx1"][t])
        g2.append(got["dx2"][t])
        r1s.append(dz1[0])
        r2s.append(dy2t[0] + O.layer_backward(x2[t:t + 1], dz1, LF)[0][0])
    assert len(ok_rows) >= 6
    e1 = rel_err(np.array(g1), np.array(r1s))
    e2 = rel_err(np.array(g2), np.array(r2s))
    print(f"BLOCK full sampled tokens {ok_rows}: dx1 err {e1:.3e}; dx2 err {e2:.3e}")
    assert e1 <= TOL and e2 <= TOL, (e1, e2)


def _pick_experts(counts, amb_per_expert, n_between=2):
    """The busiest expert, the least-loaded non-empty one and n_between in
    between, among those that no ambiguous token touches."""
    nz = np.nonzero(counts)[0]
    order = nz[np.lexsort((amb_per_expert[nz], -counts[nz]))]     # busiest first, fewest ambiguous first
    clean = [e for e in order if amb_per_expert[e] == 0] or list(order)
    picks = [clean[0], clean[-1]]
    for q in np.linspace(0, len(clean) - 1, n_between + 2)[1:-1]:
        picks.append(clean[int(round(q))])
    return list(dict.fromkeys(int(e) for e in picks))


def _expert_grads(X, dO, L, e):
    """The oracle's adapter gradients of expert e for its routed rows X and upstream dO."""
    P = L.expert(e)
    fwd = O.expert_forward(X, P, L.s)
    res = O.expert_backward(X, dO, P, L.s, fwd)
    return res["dA"], res["dB"]


def _routed_rows(ids, gam, e):
    t_idx, j_idx = np.nonzero(ids == e)
    return t_idx, gam[t_idx, j_idx]


def test_adapter_bwd_full_size_sampled_expert_gradients():
    """dA and dB of F and G at full size, element by element, on sampled
    experts (the busiest, the least-loaded non-empty one and two in between,
    none touched by a token whose routing is a near tie).

    An expert's gradient sums over the tokens routed to it, so it is the
    oracle's expert backward over those tokens with dO = gate * cotangent. G's
    input is bf16 of the GPU's y1; F's cotangent dz1 = dy1 + J_G^T dy2 is the
    oracle's layer backward of G at the tokens of F's picked experts."""
    fb = full_block()
    cfgF, cfgG, rawF, rawG = fb["cfgF"], fb["cfgG"], fb["rawF"], fb["rawG"]
    x2 = O.bf16_to_f64(fb["x2b"])
    dy1, dy2 = fb["dy1"].astype(np.float64), fb["dy2"].astype(np.float64)
    got = fb["got"]
    LF, LG = O.Layer(rawF), O.Layer(rawG)
    kF, kG = cfgF.k, cfgG.k
    z = g_input(got["y1"])
    lF, lG = O.router_logits(x2, LF), O.router_logits(z, LG)
    idsF, idsG = O.topk(lF, kF), O.topk(lG, kG)
    gF, gG = O.gates(lF, idsF), O.gates(lG, idsG)
    ambG_tok = O.routing_gap(lG, kG) < 1e-4
    ambF_tok = O.routing_gap(lF, kF) < 1e-4
    E = cfgF.E
    countsG = np.bincount(idsG.ravel(), minlength=E)
    countsF = np.bincount(idsF.ravel(), minlength=E)
    ambG_e = np.bincount(idsG[ambG_tok].ravel(), minlength=E)
    ambF_e = np.bincount(idsF[ambF_tok | ambG_tok].ravel(), minlength=E)   # a G-ambiguous token moves dz1
    picksG = _pick_experts(countsG, ambG_e)
    picksF = _pick_experts(countsF, ambF_e)
    assert len(picksG) >= 4 and len(picksF) >= 4
    assert all(ambG_e[e] == 0 for e in picksG) and all(ambF_e[e] == 0 for e in picksF)

    def check(name, g, r):
        err = rel_err(g, r)
        print(f"BLOCK full {name}: err {err:.3e}")
        assert err <= TOL, (name, err)

    for e in picksG:
        t, gam = _routed_rows(idsG, gG, e)
        dA, dB = _expert_grads(z[t], gam[:, None] * dy2[t], LG, e)
        for p in range(3):
            check(f"dA_G[{p}] expert {e} ({len(t)} rows)", got["dA_G"][p][e], dA[p])
            check(f"dB_G[{p}] expert {e} ({len(t)} rows)", got["dB_G"][p][e], dB[p])
    S = np.unique(np.concatenate([np.nonzero(np.any(idsF == e, axis=1))[0] for e in picksF]))
    dz1 = np.zeros_like(dy1)
    dz1[S] = dy1[S] + O.layer_backward(z[S], dy2[S], LG)[0]
    for e in picksF:
        t, gam = _routed_rows(idsF, gF, e)
        dA, dB = _expert_grads(x2[t], gam[:, None] * dz1[t], LF, e)
        for p in range(3):
            check(f"dA_F[{p}] expert {e} ({len(t)} rows)", got["dA_F"][p][e], dA[p])
            check(f"dB_F[{p}] expert {e} ({len(t)} rows)", got["dB_F"][p][e], dB[p])
