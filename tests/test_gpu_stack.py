"""GPU parity of the reversible stack (rev_stack_fwd / _inv / _bwd) against the
fp64 oracle.

* One block is the coupling: rev_stack_* at L = 1 equals rev_couple_fwd,
  rev_couple_inv and tqp_adapter_bwd bit for bit.
* Reconstruction of the inputs after the inverse at every depth 1..8 of a
  sparse (16 experts, top-4) stack: the streams are fp32 multiples of 2^-16
  below 256 in magnitude, on which every coupling add and subtract is exact,
  so the inverse returns the inputs put on that grid bit for bit at any depth
  (a bf16 input changes only where it is below 2^-9, by at most 2^-17), far
  inside max|x - inv(fwd(x))| / RMS(x) <= 5e-3.
* Three blocks against the oracle: the forward's residual branches (y - x) and
  dx1, dx2 and the adapter gradients of all six layers from the backward. The
  GPU carries bf16-rounded layer outputs through its own trajectory, so the
  layers after the first see inputs that differ from the oracle's by that
  rounding. With sparse routing a handful of those differences flip a token's
  expert set and move whole expert sums; this comparison therefore uses layers
  whose every token reaches every expert (top-4 of 4, gates still a softmax of
  the logits), where the outputs are smooth in the inputs. The bound is TOL;
  the oracle's own spread when every layer output moves by 2^-8 relative is
  printed beside each error for scale.

The layers' base weights and LoRA B are scaled by 1/2 (synth's w_mult): with
unscaled random weights the un-normalised SwiGLU branches grow quadratically
from block to block and the streams leave fp16's range after two or three
blocks; at 1/2 each branch adds about 8 % of the stream's RMS.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import tqp_oracle as O
from tests.gpu_util import dev, dev_bf16, host_bf16, rel_err, stream_grid

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import quantized_base_lora_moe_b200 as Q

TOL = 2e-2
STK = synth.LayerConfig("stk", T=384, d=256, E=16, k=4, f=256, g=64, r=16, w_mult=0.5)
STK_DENSE = synth.LayerConfig("stkd", T=384, d=256, E=4, k=4, f=256, g=64, r=16, w_mult=0.5)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    Q.lib()


def layers(L, cfg=STK):
    raws = [synth.make_layer(dataclasses.replace(cfg, seed=s), s) for s in range(2 * L)]
    return raws[0::2], raws[1::2]


def gpu_stack(rawF, rawG):
    F = [Q.DeviceLayer(r) for r in rawF]
    G = [Q.DeviceLayer(r) for r in rawG]
    return F, G, Q.ReversibleStack(F, G)


def test_stack_of_one_block_equals_the_coupling_calls():
    cfg = STK
    rawF, rawG = layers(1)
    F, G, stack = gpu_stack(rawF, rawG)
    T, d = cfg.T, cfg.d
    x1, x2 = dev_bf16(synth.make_tokens(T, d, 2)), dev_bf16(synth.make_tokens(T, d, 3))
    dy1, dy2 = dev(synth.make_grad(T, d, 4, "dy1")), dev(synth.make_grad(T, d, 4, "dy2"))
    st = Q.Status()
    f32 = lambda: torch.empty(T, d, dtype=torch.float32, device="cuda")
    b16 = lambda: torch.empty(T, d, dtype=torch.int16, device="cuda")
    ya, yb, za, zb = f32(), f32(), f32(), f32()
    Q.rev_couple_fwd(x1, x2, F[0], G[0], ya, yb, status=st)
    Q.rev_stack_fwd(x1, x2, stack, za, zb, status=st)
    ra, rb, sa, sb = b16(), b16(), b16(), b16()
    Q.rev_couple_inv(ya, yb, F[0], G[0], ra, rb, status=st)
    Q.rev_stack_inv(za, zb, stack, sa, sb, status=st)
    dA1, dB1, g1 = F[0].grads()
    dA2, dB2, g2 = G[0].grads()
    gF, gG, arrays = stack.grads()
    p1, p2, q1, q2 = b16(), b16(), b16(), b16()
    dxa, dxb, dxc, dxd = f32(), f32(), f32(), f32()
    Q.tqp_adapter_bwd(ya, yb, dy1, dy2, F[0], G[0], p1, p2, dxa, dxb, g1, g2, status=st)
    Q.rev_stack_bwd(za, zb, dy1, dy2, stack, q1, q2, dxc, dxd, arrays, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    assert torch.equal(ya, za) and torch.equal(yb, zb)
    assert torch.equal(ra, sa) and torch.equal(rb, sb)
    assert torch.equal(p1, q1) and torch.equal(p2, q2)
    assert torch.equal(dxa, dxc) and torch.equal(dxb, dxd)
    for p in range(3):
        assert torch.equal(dA1[p], gF[0].dA[p]) and torch.equal(dB1[p], gF[0].dB[p])
        assert torch.equal(dA2[p], gG[0].dA[p]) and torch.equal(dB2[p], gG[0].dB[p])


def _perturbed_forward(x1, x2, blocks, rng):
    """The oracle's stack forward with every layer output moved by up to 2^-8
    relative (the size of the bf16 rounding the GPU applies to it)."""
    a1, a2 = x1, x2
    for F, G in blocks:
        f = O.layer_forward(O.round_bf16(a2), F)
        b1 = a1 + f * (1.0 + 2.0 ** -8 * rng.uniform(-1.0, 1.0, f.shape))
        g = O.layer_forward(O.round_bf16(b1), G)
        b2 = a2 + g * (1.0 + 2.0 ** -8 * rng.uniform(-1.0, 1.0, g.shape))
        a1, a2 = b1, b2
    return a1, a2


def test_stack_reconstruction_at_every_depth():
    cfg, L = STK, 8
    rawF, rawG = layers(L)
    F, G, _ = gpu_stack(rawF, rawG)
    T, d = cfg.T, cfg.d
    x1b, x2b = synth.make_tokens(T, d, 2), synth.make_tokens(T, d, 3)
    x1, x2 = O.bf16_to_f64(x1b), O.bf16_to_f64(x2b)
    rms = np.sqrt(np.mean(np.concatenate([x1, x2]) ** 2))
    st = Q.Status()
    for depth in range(1, L + 1):
        sub = Q.ReversibleStack(F[:depth], G[:depth])
        y1 = torch.empty(T, d, dtype=torch.float32, device="cuda")
        y2 = torch.empty_like(y1)
        Q.rev_stack_fwd(dev_bf16(x1b), dev_bf16(x2b), sub, y1, y2, status=st)
        r1 = torch.empty(T, d, dtype=torch.int16, device="cuda")
        r2 = torch.empty_like(r1)
        Q.rev_stack_inv(y1, y2, sub, r1, r2, status=st)
        torch.cuda.synchronize()
        assert st.read() == 0
        err = max(np.max(np.abs(host_bf16(r1) - x1)), np.max(np.abs(host_bf16(r2) - x2))) / rms
        print(f"STACK depth {depth}: reconstruction max|x - inv(fwd(x))| / RMS(x) = {err:.3e}")
        assert np.array_equal(host_bf16(r1), stream_grid(x1)), depth
        assert np.array_equal(host_bf16(r2), stream_grid(x2)), depth
        assert err <= 2.0 ** -17 / rms, (depth, err)


def test_stack_of_three_blocks_matches_oracle():
    cfg, L = STK_DENSE, 3
    rawF, rawG = layers(L, cfg)
    F, G, stack = gpu_stack(rawF, rawG)
    blocks = [(O.Layer(f), O.Layer(g)) for f, g in zip(rawF, rawG)]
    T, d = cfg.T, cfg.d
    x1b, x2b = synth.make_tokens(T, d, 2), synth.make_tokens(T, d, 3)
    dy1n, dy2n = synth.make_grad(T, d, 4, "dy1"), synth.make_grad(T, d, 4, "dy2")
    x1, x2 = O.bf16_to_f64(x1b), O.bf16_to_f64(x2b)
    rms = np.sqrt(np.mean(np.concatenate([x1, x2]) ** 2))
    st = Q.Status()
    f32 = lambda: torch.empty(T, d, dtype=torch.float32, device="cuda")
    b16 = lambda: torch.empty(T, d, dtype=torch.int16, device="cuda")
    # forward values (the residual branches) against the oracle
    y1, y2 = f32(), f32()
    Q.rev_stack_fwd(dev_bf16(x1b), dev_bf16(x2b), stack, y1, y2, status=st)
    o1, o2 = O.stack_forward(x1, x2, blocks)
    p1, p2 = _perturbed_forward(x1, x2, blocks, np.random.default_rng(31))
    g1, g2 = y1.cpu().numpy().astype(np.float64), y2.cpu().numpy().astype(np.float64)
    for name, g, o, p, x in (("y1", g1, o1, p1, x1), ("y2", g2, o2, p2, x2)):
        err, spread = rel_err(g - x, o - x), rel_err(p - x, o - x)
        print(f"SPREAD stack-3 {name} - x: err {err:.3e} spread {spread:.3e} bound {TOL:.1e}")
        assert err <= TOL, (name, err, spread)
    # backward from the GPU's outputs
    gF, gG, arrays = stack.grads()
    r1, r2, dx1, dx2 = b16(), b16(), f32(), f32()
    Q.rev_stack_bwd(y1, y2, dev(dy1n), dev(dy2n), stack, r1, r2, dx1, dx2, arrays, status=st)
    torch.cuda.synchronize()
    assert st.read() == 0
    err = max(np.max(np.abs(host_bf16(r1) - x1)), np.max(np.abs(host_bf16(r2) - x2))) / rms
    assert err <= 5e-3, err
    dy1, dy2 = dy1n.astype(np.float64), dy2n.astype(np.float64)
    ref = O.stack_backward(o1, o2, dy1, dy2, blocks)
    pert = O.stack_backward(p1, p2, dy1, dy2, blocks)

    def check(name, g, r, q):
        err, spread = rel_err(g, r), rel_err(q, r)
        print(f"SPREAD stack-3 {name}: err {err:.3e} spread {spread:.3e} bound {TOL:.1e}")
        assert err <= TOL, (name, err, spread)

    check("dx1", dx1.cpu().numpy(), ref["dx1"], pert["dx1"])
    check("dx2", dx2.cpu().numpy(), ref["dx2"], pert["dx2"])
    for l in range(L):
        for p in range(3):
            check(f"block {l} dA_F[{p}]", gF[l].dA[p].cpu().numpy(), ref["grads"][l][0][p], pert["grads"][l][0][p])
            check(f"block {l} dB_F[{p}]", gF[l].dB[p].cpu().numpy(), ref["grads"][l][1][p], pert["grads"][l][1][p])
            check(f"block {l} dA_G[{p}]", gG[l].dA[p].cpu().numpy(), ref["grads"][l][2][p], pert["grads"][l][2][p])
            check(f"block {l} dB_G[{p}]", gG[l].dB[p].cpu().numpy(), ref["grads"][l][3][p], pert["grads"][l][3][p])


def test_stack_workspace_does_not_grow_with_depth():
    rawF, rawG = layers(1)
    F, G, _ = gpu_stack(rawF, rawG)
    sizes = [Q.ReversibleStack([F[0]] * L, [G[0]] * L).workspace_size(STK.T) for L in (1, 2, 8, 64)]
    assert len(set(sizes)) == 1, sizes
