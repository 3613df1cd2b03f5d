"""GPU parity of the adapter optimizer step and of the data-parallel gradient
composition.

* tqp_adamw_step against the oracle's fp64 AdamW over three steps on seeded
  buffers (n with a ragged tail): parameters and moments within fp32 rounding,
  the bf16 copy bit-exact as the round-to-nearest-even of the fp32 result.
* AdapterAdamW rewrites the layer's bf16 adapter factors: the next layer
  forward matches the oracle run with the updated factors.
* Data parallelism by tokens: the adapter gradients of two token shards,
  computed by two layer backward calls, add up to the gradient of the whole
  batch (one GPU here; across GPUs the sum is the all-reduce in dp.py).
"""
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


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    Q.lib()


def test_adamw_step_matches_oracle():
    n = 1_000_003                              # not a multiple of 4: the tail path runs too
    rng = np.random.default_rng(51)
    p = (rng.standard_normal(n) * 0.05).astype(np.float32)
    m = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    v = (rng.random(n) * 1e-5).astype(np.float32)
    P, M, V = dev(p), dev(m), dev(v)
    pb = torch.empty(n, dtype=torch.int16, device="cuda")
    rp, rm, rv = p.astype(np.float64), m.astype(np.float64), v.astype(np.float64)
    lr, b1, b2, eps, wd = 2e-3, 0.9, 0.999, 1e-8, 0.01
    # the C ABI takes the hyperparameters as fp32: the oracle gets the same values
    f32 = lambda v_: float(np.float32(v_))
    st = Q.Status()
    # m is a sum of terms of either sign and can cancel to ~0: its fp32 error is
    # bounded by the size of the terms summed into it, tracked here as mag
    mag = np.abs(m).astype(np.float64)
    for t in range(1, 4):
        g = (rng.standard_normal(n) * (1.0 if t != 2 else 1e-3)).astype(np.float32)
        Q.tqp_adamw_step(P, M, V, dev(g), t, lr, b1, b2, eps, wd, grad_scale=0.5, param_bf16=pb, status=st)
        rp, rm, rv = O.adamw_step(rp, rm, rv, g.astype(np.float64), f32(lr), f32(b1), f32(b2), f32(eps), f32(wd), t,
                                  grad_scale=0.5)
        mag = f32(b1) * mag + (1.0 - f32(b1)) * np.abs(0.5 * g.astype(np.float64))
    torch.cuda.synchronize()
    assert st.read() == 0
    gp, gm, gv = P.cpu().numpy(), M.cpu().numpy(), V.cpu().numpy()
    assert np.max(np.abs(gp - rp) / (np.abs(rp) + lr)) <= 1e-5
    assert np.max(np.abs(gm - rm) / (mag + 1e-30)) <= 1e-5           # a few fp32 ulps of the terms
    assert np.max(np.abs(gv - rv) / (np.abs(rv) + 1e-12)) <= 1e-5    # v sums non-negative terms
    assert np.array_equal(pb.cpu().numpy().view(np.uint16), synth.f32_to_bf16_bits(gp))


def test_adamw_nonfinite_gradient_raises_status():
    n = 4096
    P, M, V = (torch.zeros(n, device="cuda") for _ in range(3))
    g = torch.zeros(n, device="cuda")
    g[17] = float("inf")
    st = Q.Status()
    Q.tqp_adamw_step(P, M, V, g, 1, 1e-3, status=st)
    torch.cuda.synchronize()
    assert st.read() & Q.STATUS_NONFINITE


def test_adapter_adamw_updates_the_layer_the_forward_reads():
    cfg = synth.LayerConfig("opt", T=256, d=256, E=8, k=2, f=256, g=64, r=16)
    raw = synth.make_layer(cfg)
    L = Q.DeviceLayer(raw)
    opt = Q.AdapterAdamW(L, lr=5e-2, weight_decay=0.01)
    grads = L.flat_grads()
    rng = np.random.default_rng(52)
    g = rng.standard_normal(grads.flat.numel()).astype(np.float32)
    grads.flat.copy_(torch.from_numpy(g))
    opt.step(grads)
    torch.cuda.synchronize()
    # the oracle's step on the same (bf16) starting factors
    parts = [raw[f"la{p}"] for p in range(3)] + [raw[f"lb{p}"] for p in range(3)]
    p0 = np.concatenate([O.bf16_to_f64(a).ravel() for a in parts])
    f32 = lambda v_: float(np.float32(v_))
    rp, _, _ = O.adamw_step(p0, np.zeros_like(p0), np.zeros_like(p0), g.astype(np.float64), f32(5e-2), f32(0.9),
                            f32(0.999), f32(1e-8), f32(0.01), 1)
    assert np.max(np.abs(opt.master.cpu().numpy() - rp) / (np.abs(rp) + 5e-2)) <= 1e-5
    # the layer's bf16 factors now hold the new values and the forward uses them
    new = dict(raw)
    off = 0
    for i, a in enumerate(parts):
        bits = L.lora_flat[off:off + a.size].cpu().numpy().view(np.uint16).reshape(a.shape)
        new[("la" if i < 3 else "lb") + str(i % 3)] = bits
        off += a.size
    xb = synth.make_tokens(cfg.T, cfg.d, 53)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.int16, device="cuda")
    Q.tqp_moe_layer_fwd(dev_bf16(xb), L, y)
    torch.cuda.synchronize()
    x = O.bf16_to_f64(xb)
    Lo = O.Layer(new)
    keep = ~near_tie_tokens(O.router_logits(x, Lo), cfg.k, 1e-4)
    ref = O.layer_forward(x, Lo)
    assert rel_err_bf16_out(host_bf16(y)[keep], ref[keep]) <= TOL
    # and the old factors would not have matched: the step changed the output
    assert rel_err(ref, O.layer_forward(x, O.Layer(raw))) > 1e-3


def test_token_shards_gradients_add_up_to_the_batch_gradient():
    from quantized_base_lora_moe_b200.dp import adapter_dp_step
    cfg = synth.LayerConfig("dps", T=600, d=256, E=10, k=3, f=256, g=64, r=16)
    raw = synth.make_layer(cfg)
    L = Q.DeviceLayer(raw)
    xb = synth.make_tokens(cfg.T, cfg.d, 54)
    dy = synth.make_grad(cfg.T, cfg.d, 55, "dy1")
    x_dev, dy_dev = dev_bf16(xb), dev(dy)
    full = L.flat_grads()
    dx = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    st = Q.Status()
    Q.tqp_moe_layer_bwd(x_dev, dy_dev, L, dx, full, status=st)
    total = torch.zeros_like(full.flat)
    for lo, hi in ((0, 250), (250, cfg.T)):     # two shards of different sizes
        part = L.flat_grads()
        dxs = torch.empty(hi - lo, cfg.d, dtype=torch.float32, device="cuda")

        def local(g, lo=lo, hi=hi, dxs=dxs):
            Q.tqp_moe_layer_bwd(x_dev[lo:hi].contiguous(), dy_dev[lo:hi].contiguous(), L, dxs, g, status=st)

        adapter_dp_step(local, part)           # no process group: the all-reduce is the identity
        total += part.flat
    torch.cuda.synchronize()
    assert st.read() == 0
    # the same sums in another grouping: equal up to fp32 summation order
    assert rel_err(total.cpu().numpy(), full.flat.cpu().numpy()) <= 1e-4
    # and the batch gradient is the oracle's (tokens away from routing ties)
    x = O.bf16_to_f64(xb)
    Lo = O.Layer(raw)
    _, rdA, rdB = O.layer_backward(x, dy.astype(np.float64), Lo)
    logits = O.router_logits(x, Lo)
    tie = near_tie_tokens(logits, cfg.k, 1e-4)
    srt = np.argsort(-logits[tie], axis=1, kind="stable")
    amb = set(srt[:, cfg.k - 1].tolist()) | set(srt[:, cfg.k].tolist()) if tie.any() else set()
    keep = np.array([e not in amb for e in range(cfg.E)])
    for p in range(3):
        assert rel_err(full.dA[p].cpu().numpy()[keep], rdA[p][keep]) <= TOL
        assert rel_err(full.dB[p].cpu().numpy()[keep], rdB[p][keep]) <= TOL
