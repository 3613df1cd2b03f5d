"""Host-only checks of the C-ABI library: it loads, exports every function the
header declares, answers workspace queries, and rejects bad arguments before
touching the GPU. No compute call is made."""
import ctypes
import dataclasses

import pytest

import synth
import quantized_base_lora_moe_b200 as Q


def _struct(cfg, **over):
    w = Q.Weights()
    w.E, w.d, w.ffn, w.group, w.rank, w.top_k = cfg.E, cfg.d, cfg.f, cfg.g, cfg.r, cfg.k
    w.lora_scale = cfg.lora_scale
    fake = 0x10000
    w.router_w = fake
    for p in range(3):
        w.wq[p] = fake
        w.wscale[p] = fake
        w.lora_a[p] = fake
        w.lora_b[p] = fake
    for k_, v in over.items():
        setattr(w, k_, v)
    return w


def test_library_loads_and_exports_header_functions():
    L = Q.lib()
    names = Q.header_functions()
    assert len(names) >= 19
    for n in names:
        assert hasattr(L, n), n
    assert L.tqp_version() >= 100
    assert L.tqp_error_string(-3) == b"workspace too small"


@pytest.mark.parametrize("cfg", [synth.TINY, synth.MID, synth.FULL, synth.SKEWED], ids=lambda c: c.name)
def test_workspace_queries(cfg):
    L = Q.lib()
    w = _struct(cfg)
    assert L.moe_router_gemm_workspace_size(cfg.T, ctypes.byref(w)) >= 3 * cfg.E * cfg.d * 2
    assert L.moe_permute_workspace_size(cfg.T, cfg.E, cfg.k) >= ((cfg.T + 31) // 32) * cfg.E * 4
    assert L.tqp_grouped_ffn_workspace_size(cfg.T, ctypes.byref(w)) >= cfg.T * cfg.k * 3 * cfg.r * 2
    lw = L.tqp_moe_layer_workspace_size(cfg.T, ctypes.byref(w))
    assert lw >= cfg.T * cfg.k * (cfg.f + cfg.d) * 2
    assert L.rev_couple_workspace_size(cfg.T, ctypes.byref(w), ctypes.byref(w)) > lw
    assert L.tqp_adapter_bwd_workspace_size(cfg.T, ctypes.byref(w), ctypes.byref(w)) > lw


BAD = [
    dict(E=0), dict(top_k=0), dict(top_k=33), dict(d=100), dict(d=192), dict(ffn=96), dict(group=48),
    dict(rank=12), dict(rank=72), dict(router_w=None), dict(router_w=0x10004), dict(bits=3), dict(bits=16),
]


@pytest.mark.parametrize("over", BAD, ids=[str(b) for b in BAD])
def test_invalid_weights_rejected_on_host(over):
    L = Q.lib()
    w = _struct(synth.TINY, **over)
    assert L.tqp_moe_layer_workspace_size(64, ctypes.byref(w)) == 0
    rc = L.tqp_moe_layer_fwd(0x20000, 64, ctypes.byref(w), 0x30000, 0x40000, 1 << 30, None, None)
    assert rc in (-1, -2)


def test_small_workspace_and_null_pointers_rejected():
    L = Q.lib()
    w = _struct(synth.TINY)
    assert L.tqp_moe_layer_fwd(0x20000, 64, ctypes.byref(w), 0x30000, 0x40000, 16, None, None) == -3
    assert L.tqp_moe_layer_fwd(None, 64, ctypes.byref(w), 0x30000, 0x40000, 1 << 30, None, None) == -1
    assert L.moe_route(None, 4, 8, 2, None, None, None, None) == -1
    assert L.moe_route(0x1000, 4, 8, 9, 0x1000, 0x1000, None, None) == -1
    assert L.moe_permute(0x1000, 4, 8, 2, 0x1000, 0x1000, 0x1000, 0x1000, 0, None, None) == -3
    assert L.moe_combine(0x1000, 0x1000, 0x1000, 4, 2, 12, None, 0, 1.0, 0x1000, 0, None, None) == -1
    # T == 0 is a no-op that succeeds without touching the device
    assert L.tqp_moe_layer_fwd(None, 0, ctypes.byref(w), None, None, 0, None, None) == 0


def test_mismatched_coupling_widths_rejected():
    L = Q.lib()
    F = _struct(synth.TINY)
    G = _struct(synth.MID)
    assert L.rev_couple_workspace_size(64, ctypes.byref(F), ctypes.byref(G)) == 0
    assert L.rev_couple_fwd(0x1000, 0x1000, 64, ctypes.byref(F), ctypes.byref(G), 0x1000, 0x1000, 0x1000,
                            1 << 30, None, None) == -1


def test_grouped_ffn_part_rejects_unknown_part():
    L = Q.lib()
    w = _struct(synth.TINY)
    for part in (-1, 4):
        rc = L.tqp_grouped_ffn_part(part, None, 0, None, None, ctypes.byref(w), None, None, None, 0, None, None)
        assert rc == -1, (part, rc)
    # a valid part with an empty batch is a no-op that enqueues nothing
    rc = L.tqp_grouped_ffn_part(Q.FFN_GATE_UP, None, 0, None, None, ctypes.byref(w), None, None, None, 0, None, None)
    assert rc == 0


@pytest.mark.parametrize("cfg", [synth.TINY, synth.MID, synth.FULL], ids=lambda c: c.name)
def test_backward_workspace_holds_its_scratch(cfg):
    # the backward adds, per routed row, G|U and dG|dU (2f each), dO (d), dha (r) and
    # dxa (2r) as fp16, plus the K-major fp16 B operand of the rank-space products:
    # Bd as [E][r][d] or blockdiag(Bg, Bu) as [E][2r][2f], whichever is larger, and
    # the row copy of the A factors for the dgrads: Ad as [E][f][r] or [Ag|Au] as
    # [E][d][2r], whichever is larger
    L = Q.lib()
    w = _struct(cfg)
    A = cfg.T * cfg.k
    extra = (L.tqp_moe_layer_bwd_workspace_size(cfg.T, ctypes.byref(w))
             - L.tqp_moe_layer_workspace_size(cfg.T, ctypes.byref(w)))
    need = (A * (4 * cfg.f + cfg.d + 3 * cfg.r) * 2 + cfg.E * max(cfg.r * cfg.d, 4 * cfg.r * cfg.f) * 2
            + cfg.E * max(cfg.f * cfg.r, 2 * cfg.d * cfg.r) * 2)
    assert need <= extra <= need + 9 * 256 + 256


def _grads(**bad):
    g = Q.Grads()
    for p in range(3):
        g.dA[p] = 0x50000 + 0x1000 * p
        g.dB[p] = 0x60000 + 0x1000 * p
    for k_, (p, v) in bad.items():
        getattr(g, k_)[p] = v
    return g


@pytest.mark.parametrize("bad", [dict(dA=(1, None)), dict(dB=(2, None)), dict(dA=(0, 0x50004)), dict(dB=(0, 0x60008))],
                         ids=["dA1-null", "dB2-null", "dA0-misaligned", "dB0-misaligned"])
def test_backward_rejects_bad_gradient_buffers_before_any_launch(bad):
    # both layers' gradient buffers are checked on the host before the first launch
    L = Q.lib()
    F, G = _struct(synth.TINY), _struct(synth.TINY)
    good, wrong = _grads(), _grads(**bad)
    p = 0x70000
    for gF, gG in ((wrong, good), (good, wrong)):
        rc = L.tqp_adapter_bwd(p, p, p, p, 64, ctypes.byref(F), ctypes.byref(G), p, p, p, p, ctypes.byref(gF),
                               ctypes.byref(gG), p, 1 << 30, None, None)
        assert rc == -1, rc
    assert L.tqp_moe_layer_bwd(p, p, 64, ctypes.byref(F), p, ctypes.byref(wrong), p, 1 << 30, None, None) == -1
    # rank 0 has no adapters: null gradient buffers are fine (T = 0: nothing is enqueued)
    F0 = _struct(synth.TINY, rank=0)
    null = Q.Grads()
    assert L.tqp_moe_layer_bwd(None, None, 0, ctypes.byref(F0), None, ctypes.byref(null), None, 0, None, None) == 0


def test_int8_needs_ffn_multiple_of_128():
    L = Q.lib()
    cfg = synth.LayerConfig("i8", T=64, d=128, E=4, k=2, f=192, g=64, r=8)
    assert L.tqp_moe_layer_workspace_size(64, ctypes.byref(_struct(cfg, bits=8))) == 0
    assert L.tqp_moe_layer_fwd(0x20000, 64, ctypes.byref(_struct(cfg, bits=8)), 0x30000, 0x40000, 1 << 30, None,
                               None) == -2
    assert L.tqp_moe_layer_workspace_size(64, ctypes.byref(_struct(cfg, bits=4))) > 0
    assert L.tqp_moe_layer_workspace_size(64, ctypes.byref(_struct(synth.TINY, bits=8))) > 0


def _stack_arrays(ws_list):
    arr = (ctypes.POINTER(Q.Weights) * len(ws_list))(*[ctypes.pointer(w) for w in ws_list])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def test_stack_workspace_is_flat_in_depth_and_bad_stacks_are_rejected():
    L = Q.lib()
    w = _struct(synth.MID)
    sizes = []
    for depth in (1, 2, 16, 256):
        p, keep = _stack_arrays([w] * depth)
        sizes.append(L.rev_stack_workspace_size(synth.MID.T, depth, p, p))
    assert sizes[0] > 0 and len(set(sizes)) == 1
    p, keep = _stack_arrays([w] * 2)
    assert L.rev_stack_workspace_size(synth.MID.T, 0, p, p) == 0                 # L = 0
    other = _struct(dataclasses.replace(synth.MID, d=512))
    q, keep2 = _stack_arrays([w, other])
    assert L.rev_stack_workspace_size(synth.MID.T, 2, q, q) == 0                  # mixed widths
    # the backward needs gradient arrays: refused before anything is enqueued
    rc = L.rev_stack_bwd(0x20000, 0x20000, 0x20000, 0x20000, synth.MID.T, 2, p, p, 0x20000, 0x20000, 0x20000,
                         0x20000, None, None, 0x30000, 1 << 40, None, None)
    assert rc == -1


def test_adamw_rejects_bad_hyperparameters_on_host():
    L = Q.lib()
    f = ctypes.c_void_p(0x10000)
    assert L.tqp_adamw_step(f, f, f, f, None, 16, 1e-3, 0.9, 0.999, 1e-8, 0.0, 0, 1.0, None, None) == -1  # step 0
    assert L.tqp_adamw_step(f, f, f, f, None, 16, 1e-3, 1.0, 0.999, 1e-8, 0.0, 1, 1.0, None, None) == -1  # beta1 = 1
    assert L.tqp_adamw_step(f, f, f, f, None, 16, 1e-3, 0.9, 0.999, 0.0, 0.0, 1, 1.0, None, None) == -1   # eps = 0
    assert L.tqp_adamw_step(ctypes.c_void_p(0x10004), f, f, f, None, 16, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, 1.0, None,
                            None) == -1                                                                   # misaligned
    assert L.tqp_adamw_step(f, f, f, f, None, 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, 1.0, None, None) == 0    # n = 0: no-op
