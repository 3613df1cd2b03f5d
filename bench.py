"""Benchmark of the TQP MoE layer forward on B200 (one process per GPU).

python bench.py [--gpus N --steps K --warmup W --config full|skewed|mid|tiny] [--impl tqp|reference]

A step is one full layer forward (router GEMM, top-k routing, permutation,
grouped int4+LoRA SwiGLU experts, combine) over one batch of T synthetic
tokens, through the library's one-call C-ABI entry point tqp_moe_layer_fwd.
Inputs are resident in HBM when the timed region starts; L2 is flushed between
steps by writing a buffer larger than L2 (the layer's weights, 1.4 GB for the
460-expert config, are larger than L2 as well). CUDA events on the launching
stream time every step; the timed region is bracketed by a barrier and a device
synchronisation on both sides; multi-GPU time is the max over ranks. Each rank
processes its own batch (weak scaling, no collective on the data path). The
per-kernel breakdown (`per_call_ms`, and the gate/up kernel's roofline) comes
from a second loop of the same passes issued as the per-part calls (router
GEMM, route, permute, the four grouped-FFN parts, combine) with events between
them.

The `e2e` leg measures the same metric through the Python API with the token
batch copied from pinned host memory and the layer output copied back inside
the timed region. `cpu_baseline` times the fp64 oracle on a bounded sample of
the same workload on this host's cores. `--impl reference` times that oracle
as the reference arm (there is no other implementation of this layer).
On one GPU with the full config, `rev_block` adds the reversible block built
from two such layers (coupling forward, its inverse, adapter backward), each
call timed with CUDA events outside the headline region.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "routed tokens/s and TFLOP/s, 460-expert top-12 TQP MoE layer; % of roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 512 << 20


def layer_flops(cfg: synth.LayerConfig) -> dict:
    """Algorithmic FLOPs of one layer forward (router, experts, LoRA)."""
    A = cfg.T * cfg.k
    router = 2.0 * cfg.T * cfg.d * cfg.E
    expert = A * 6.0 * cfg.d * cfg.f
    lora = A * 2.0 * cfg.r * (cfg.d + cfg.f) * 3
    # the gate/up expert kernel: both projections plus their rank-space products (xa) B
    gate_up = A * 4.0 * cfg.d * cfg.f + A * 4.0 * cfg.r * cfg.f
    return {"router": router, "expert": expert, "lora": lora, "total": router + expert + lora,
            "ffn": expert + lora, "gate_up": gate_up}


def layer_bwd_flops(cfg: synth.LayerConfig) -> float:
    """Algorithmic FLOPs of one layer's adapter-only backward (base and router frozen).

    Expert dgrads dH = dO Wd and dX = dG Wg + dU Wu: 6 A d f. Adapter terms, each
    a 2 A r n product (n = d or f): down dBd, dha, dAd and the rank term of dH;
    gate/up dBg, dBu, dxa, dAg, dAu and the rank term of dX: 12 A r (d + f).
    Gate dot products and the router's input gradient: 4 A d.
    """
    A = cfg.T * cfg.k
    return 6.0 * A * cfg.d * cfg.f + 12.0 * A * cfg.r * (cfg.d + cfg.f) + 4.0 * A * cfg.d


def workload_config(cfg: synth.LayerConfig) -> dict:
    """The workload as both arms report it in `config`."""
    return {"workload": f"{cfg.name}: T={cfg.T} d={cfg.d} E={cfg.E} top-{cfg.k} ffn={cfg.f} int{cfg.bits} g{cfg.g} LoRA r{cfg.r}"
                        f"{' zipf-bias' if cfg.zipf_s else ''}, layer forward",
            "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "ffn": cfg.f, "group": cfg.g, "rank": cfg.r}


def rank_token_seed(cfg: synth.LayerConfig, rank: int) -> int:
    """Each rank draws its own token batch (data parallel, weak scaling)."""
    return cfg.seed + rank


def max_over_ranks(value: float, device, dist: bool) -> float:
    """The slowest rank's time: MAX all-reduce across the process group (identity on one rank)."""
    if not dist:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job routed tokens/s: every rank processes its own batch in the (max-over-ranks) step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def measured_traffic(kernel: str) -> int | None:
    """DRAM bytes per launch of `kernel` from the committed ncu capture, if the
    expert-kernel sources are still the ones that were captured; else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "expert_traffic_full.json")
    if not os.path.exists(path):
        return None
    doc = json.load(open(path))
    h = hashlib.sha256()
    for f in ("expert_gateup.cu", "expert_down.cu", "expert_common.cuh", "gemm_common.cuh", "tqp_device.cuh"):
        with open(os.path.join(ROOT, "quantized_base_lora_moe_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != doc.get("kernel_sources_sha256_16"):
        return None
    k = doc["kernels"].get(kernel)
    return None if k is None else int(k["dram_read_bytes"] + k["dram_write_bytes"])


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- CPU oracle timing


def time_oracle(cfg: synth.LayerConfig, host: dict, x_bits: np.ndarray, sample_tokens: int) -> dict:
    """Time the fp64 oracle's layer forward on the first `sample_tokens` tokens."""
    from oracle import tqp_oracle as O
    L = O.Layer(host)
    x = O.bf16_to_f64(x_bits[:sample_tokens])
    t0 = time.perf_counter()
    O.layer_forward(x, L)
    dt = time.perf_counter() - t0
    return {"value": sample_tokens / dt, "unit": UNIT, "cores": cores(), "kind": "oracle",
            "sample": f"first {sample_tokens} of {cfg.T} tokens of the {cfg.name} workload, fp64 NumPy "
                      f"(dequantises every touched expert), {dt:.1f} s wall"}


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = tempfile.mktemp(suffix=".csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        load = [v for v in sm if smax and v > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- GPU arm


def time_rev_block(L_F, cfgF: synth.LayerConfig, dev, steps: int, warmup: int, flush) -> dict:
    """The reversible block, timed per call with CUDA events.

    F is the bench's layer, G a second independent instance (seed 1); streams
    x1, x2 of T x d bf16 and upstream gradients dy1, dy2 ~ N(0, 1) fp32.
    One block step is rev_couple_fwd then tqp_adapter_bwd, which reconstructs
    x1, x2 with the inverse coupling before the adapter gradients; the inverse
    alone (rev_couple_inv) is timed beside it. L2 is flushed before each call.
    """
    import torch
    import quantized_base_lora_moe_b200 as Q
    cfgG = synth.REV_G if cfgF == synth.FULL else dataclasses.replace(cfgF, name=cfgF.name + "_g", seed=1)
    G = Q.DeviceLayer(synth.make_layer(cfgG, cfgG.seed), device=dev)
    T, d = cfgF.T, cfgF.d
    tok = lambda seed: torch.from_numpy(synth.make_tokens(T, d, seed).view(np.int16)).to(dev)
    x1, x2 = tok(synth.REV_SEEDS["x1"]), tok(synth.REV_SEEDS["x2"])
    dy1 = torch.from_numpy(synth.make_grad(T, d, synth.REV_SEEDS["dy"], "dy1")).to(dev)
    dy2 = torch.from_numpy(synth.make_grad(T, d, synth.REV_SEEDS["dy"], "dy2")).to(dev)
    y1 = torch.empty(T, d, dtype=torch.float32, device=dev)
    y2 = torch.empty_like(y1)
    r1, r2 = torch.empty_like(x1), torch.empty_like(x2)
    dx1, dx2 = torch.empty_like(y1), torch.empty_like(y1)
    _, _, gF = L_F.grads(dev)
    _, _, gG = G.grads(dev)
    lib = Q.lib()
    ws = Q.workspace(max(lib.rev_couple_workspace_size(T, L_F.ref(), G.ref()),
                         lib.tqp_adapter_bwd_workspace_size(T, L_F.ref(), G.ref())), dev)
    st = Q.Status(dev)
    stream = torch.cuda.current_stream(dev)
    calls = [("fwd", lambda: Q.rev_couple_fwd(x1, x2, L_F, G, y1, y2, ws, st)),
             ("inv", lambda: Q.rev_couple_inv(y1, y2, L_F, G, r1, r2, ws, st)),
             ("adapter_bwd", lambda: Q.tqp_adapter_bwd(y1, y2, dy1, dy2, L_F, G, r1, r2, dx1, dx2, gF, gG, ws, st))]
    for _ in range(warmup):
        for _, c in calls:
            flush.zero_()
            c()
    torch.cuda.synchronize(dev)
    ms = {n: [] for n, _ in calls}
    for _ in range(steps):
        for n, c in calls:
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            c()
            e1.record(stream)
            e1.synchronize()
            ms[n].append(e0.elapsed_time(e1))
    if st.read() != 0:
        raise RuntimeError(f"device status {st.read()} in the reversible block")
    f = lambda t: t.view(torch.bfloat16).float()
    rms = torch.sqrt(torch.mean(torch.cat([f(x1), f(x2)]) ** 2))
    err = float(max((f(r1) - f(x1)).abs().max(), (f(r2) - f(x2)).abs().max()) / rms)
    exact = exact_on_stream_grid(r1, x1) and exact_on_stream_grid(r2, x2)
    mean = {n: statistics.mean(v) for n, v in ms.items()}
    step_ms = mean["fwd"] + mean["adapter_bwd"]
    # forward: F and G; adapter backward: the inverse (F and G again) and both layers' backward
    fwd_flop = layer_flops(cfgF)["total"] + layer_flops(cfgG)["total"]
    step_flop = 2.0 * fwd_flop + layer_bwd_flops(cfgF) + layer_bwd_flops(cfgG)
    pk = peaks()
    tflops = step_flop / (step_ms * 1e-3) / 1e12
    return {"workload": f"two {cfgF.name} layers F, G; streams 2 x {T}x{d}; forward, inverse, adapter backward",
            "ms_per_step": step_ms, "tokens_per_s": T / (step_ms * 1e-3), "ms": mean, "steps": steps,
            "flop_per_step": step_flop, "tflops": tflops,
            "roofline_frac_measured": tflops / pk["bf16_tflops"], "roofline_frac_nominal": tflops / 2250.0,
            "reconstruction_max_err_rel_rms": err, "reconstruction_exact_on_stream_grid": exact,
            "l2": "flushed before every call"}


def exact_on_stream_grid(r, x) -> bool:
    """Whether the reconstructed bf16 r is x put on the coupling's stream grid
    (multiples of 2^-16, half to even) bit for bit."""
    import torch
    f = lambda t: t.view(torch.bfloat16).double()
    return bool(torch.equal(f(r), torch.round(f(x) * 65536.0) / 65536.0))


def time_stack(dev, flush, depths=(1, 2, 4, 8)) -> dict:
    """The reversible stack against its depth L at full size: peak device
    memory, workspace, time of the forward and of the backward from the outputs
    alone, and the reconstruction error of the inputs.

    The blocks are built from two full-size layers F, G (460 experts, top-12,
    T = 8192, d = 2048) whose base weights and LoRA B are scaled by 1/2, so
    that the un-normalised SwiGLU branches stay small against the streams over
    8 blocks (at scale 1 they grow quadratically from block to block). Every
    block uses the same two weight sets; each layer of each block has its own
    adapter-gradient buffers. The activation memory is measured with torch's
    allocator statistics over one forward + backward, beyond the weights, the
    gradient buffers and the call's inputs and outputs (so: the workspace and
    anything transient); a store-everything backward would instead keep every
    block's input streams and every layer's saved intermediates.
    """
    import torch
    import quantized_base_lora_moe_b200 as Q
    cfgF = dataclasses.replace(synth.FULL, name="stack_f", w_mult=0.5)
    cfgG = dataclasses.replace(synth.FULL, name="stack_g", seed=1, w_mult=0.5)
    F = Q.DeviceLayer(synth.make_layer(cfgF, cfgF.seed), device=dev)
    G = Q.DeviceLayer(synth.make_layer(cfgG, cfgG.seed), device=dev)
    T, d = cfgF.T, cfgF.d
    tok = lambda seed: torch.from_numpy(synth.make_tokens(T, d, seed).view(np.int16)).to(dev)
    x1, x2 = tok(synth.REV_SEEDS["x1"]), tok(synth.REV_SEEDS["x2"])
    dy1 = torch.from_numpy(synth.make_grad(T, d, synth.REV_SEEDS["dy"], "dy1")).to(dev)
    dy2 = torch.from_numpy(synth.make_grad(T, d, synth.REV_SEEDS["dy"], "dy2")).to(dev)
    f32 = lambda: torch.empty(T, d, dtype=torch.float32, device=dev)
    y1, y2, dx1, dx2 = f32(), f32(), f32(), f32()
    r1, r2 = torch.empty_like(x1), torch.empty_like(x2)
    st = Q.Status(dev)
    stream = torch.cuda.current_stream(dev)
    lib = Q.lib()
    per_layer_bwd_ws = max(lib.tqp_moe_layer_bwd_workspace_size(T, F.ref()), lib.tqp_moe_layer_bwd_workspace_size(T, G.ref()))
    out = {"workload": "L blocks of two full-size layers (460 experts, top-12, T=8192, d=2048; base weights and "
                       "LoRA B x 1/2), fp32 streams on the 2^-16 grid between blocks", "depths": {}}
    bf = lambda t: t.view(torch.bfloat16).float()
    rms = float(torch.sqrt(torch.mean(torch.cat([bf(x1), bf(x2)]) ** 2)))
    for L in depths:
        stack = Q.ReversibleStack([F] * L, [G] * L)
        gF, gG, arrays = stack.grads(dev)
        torch.cuda.synchronize(dev)
        base = torch.cuda.memory_allocated(dev)      # weights, gradient buffers, inputs and outputs
        torch.cuda.reset_peak_memory_stats(dev)
        ws = Q.workspace(stack.workspace_size(T), dev)
        ms = {"fwd": [], "bwd": []}
        for i in range(2):                     # the first pass is the warm-up
            for name, call in (("fwd", lambda: Q.rev_stack_fwd(x1, x2, stack, y1, y2, ws, st)),
                               ("bwd", lambda: Q.rev_stack_bwd(y1, y2, dy1, dy2, stack, r1, r2, dx1, dx2, arrays,
                                                              ws, st))):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                call()
                e1.record(stream)
                e1.synchronize()
                if i:
                    ms[name].append(e0.elapsed_time(e1))
        peak = torch.cuda.max_memory_allocated(dev) - base
        if st.read() != 0:
            raise RuntimeError(f"device status {st.read()} in the reversible stack (L={L})")
        err = float(max((bf(r1) - bf(x1)).abs().max(), (bf(r2) - bf(x2)).abs().max())) / rms
        exact = exact_on_stream_grid(r1, x1) and exact_on_stream_grid(r2, x2)
        store_all = L * (2 * T * d * 4 + 2 * per_layer_bwd_ws)
        out["depths"][str(L)] = {"fwd_ms": ms["fwd"][0], "bwd_ms": ms["bwd"][0],
                                 "workspace_bytes": ws.numel(), "peak_activation_bytes": peak,
                                 "store_all_estimate_bytes": store_all,
                                 "reconstruction_max_err_rel_rms": err,
                                 "reconstruction_exact_on_stream_grid": exact}
        del stack, gF, gG, arrays, ws
        torch.cuda.empty_cache()
    return out


def layer_bytes(cfg: synth.LayerConfig, touched: int) -> float:
    """Algorithmic bytes of one layer forward: int4 (or int8) codes, bf16 group scales and
    bf16 LoRA factors of the touched experts, fp32 router weights, x and y in
    bf16, ids and gates. Intermediates (logits, H, O) are implementation traffic."""
    d, f, g, r = cfg.d, cfg.f, cfg.g, cfg.r
    per_expert = 3 * d * f * cfg.bits / 8 + (2 * (d // g) * f + (f // g) * d) * 2 + 3 * r * (d + f) * 2
    return touched * per_expert + cfg.E * d * 4 + 2 * cfg.T * d * 2 + cfg.T * cfg.k * 8


def layer_roofline(cfg: synth.LayerConfig, touched: int, ms: float) -> dict:
    """The layer against its roofline: the slower of its FLOPs at the tensor
    peak and its algorithmic bytes at the HBM peak, for the nominal peaks
    (2.25 PFLOP/s dense bf16, 8 TB/s) and for the measured ones."""
    fl = layer_flops(cfg)["total"]
    by = layer_bytes(cfg, touched)
    pk = peaks()
    t_nom = max(fl / 2.25e15, by / 8.0e12)
    t_meas = max(fl / (pk["bf16_tflops"] * 1e12), by / (pk["hbm_gbs"] * 1e9))
    return {"bound": "tensor" if fl / 2.25e15 >= by / 8.0e12 else "hbm", "flop": fl, "bytes": by,
            "touched_experts": touched, "achieved_tflops": fl / (ms * 1e-3) / 1e12,
            "roofline_ms_nominal": t_nom * 1e3, "frac_nominal": t_nom / (ms * 1e-3),
            "roofline_ms_measured": t_meas * 1e3, "frac_measured": t_meas / (ms * 1e-3),
            "peaks": {"nominal": "2.25 PFLOP/s dense bf16, 8 TB/s HBM",
                      "measured": f"{pk['bf16_tflops']} TFLOP/s bf16 burst, {pk['hbm_gbs']} GB/s ({pk['source']})"}}


CALLS = ["router_gemm", "route", "permute", "ffn_prepare", "ffn_gate_up", "ffn_rank", "ffn_down", "combine"]


class LayerBench:
    """One configuration's weights, batch and buffers on the device, and the
    layer forward step issued as the public C-ABI calls (the grouped FFN as its
    four parts, so that the gate/up expert kernel is timed on its own)."""

    def __init__(self, cfg: synth.LayerConfig, dev, token_seed: int, host: dict | None = None):
        import torch
        import quantized_base_lora_moe_b200 as Q
        self.Q, self.cfg, self.dev = Q, cfg, dev
        self.host = host if host is not None else synth.make_layer(cfg)
        self.x_bits = synth.make_tokens(cfg.T, cfg.d, token_seed)
        self.L = Q.DeviceLayer(self.host, device=dev)
        T, E, k, d, f = cfg.T, cfg.E, cfg.k, cfg.d, cfg.f
        A = T * k
        self.x = torch.from_numpy(self.x_bits.view(np.int16)).to(dev)
        self.y = torch.empty(T, d, dtype=torch.int16, device=dev)
        self.logits = torch.empty(T, E, dtype=torch.float32, device=dev)
        self.ids = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.gates = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.perm = torch.empty(A, dtype=torch.int32, device=dev)
        self.inv = torch.empty(A, dtype=torch.int32, device=dev)
        self.h = torch.empty(A, f, dtype=torch.int16, device=dev)
        self.o = torch.empty(A, d, dtype=torch.int16, device=dev)
        lib = Q.lib()
        self.ws_r = Q.workspace(lib.moe_router_gemm_workspace_size(T, self.L.ref()), dev)
        self.ws_p = Q.workspace(lib.moe_permute_workspace_size(T, E, k), dev)
        self.ws_f = Q.workspace(lib.tqp_grouped_ffn_workspace_size(T, self.L.ref()), dev)
        self.ws_l = Q.workspace(lib.tqp_moe_layer_workspace_size(T, self.L.ref()), dev)
        self.st = Q.Status(dev)
        self.stream = torch.cuda.current_stream(dev)
        lora = cfg.r > 0
        # kernels per call: router split + GEMM; route; permute count, column scan,
        # scatter; prepare = two block schedules, x (and Ad) to fp16, s X [Ag|Au];
        # gate/up and down = unit table + expert kernel; rank = s H Ad; combine
        self.launches = {"router_gemm": 2, "route": 1, "permute": 3, "ffn_prepare": 5 if lora else 3,
                         "ffn_gate_up": 2, "ffn_rank": 1 if lora else 0, "ffn_down": 2, "combine": 1}

    def step(self, evs=None):
        Q, c = self.Q, self.cfg

        def mark(i):
            if evs is not None:
                evs[i].record(self.stream)
        mark(0)
        Q.moe_router_gemm(self.x, self.L, self.logits, self.ws_r, self.st)
        mark(1)
        Q.moe_route(self.logits, c.k, self.ids, self.gates, self.st)
        mark(2)
        Q.moe_permute(self.ids, c.E, self.offsets, self.perm, self.inv, self.ws_p, self.st)
        mark(3)
        for j, part in enumerate([Q.FFN_PREPARE, Q.FFN_GATE_UP, Q.FFN_RANK, Q.FFN_DOWN]):
            Q.tqp_grouped_ffn_part(part, self.x, self.offsets, self.perm, self.L, self.h, self.o, self.ws_f, self.st)
            mark(4 + j)
        Q.moe_combine(self.o, self.inv, self.gates, self.y)
        mark(8)

    def layer_step(self):
        """The same pass as step() through the one-call entry point
        tqp_moe_layer_fwd (the same kernels, no events between the parts)."""
        self.Q.tqp_moe_layer_fwd(self.x, self.L, self.y, self.ws_l, self.st)

    def run(self, steps: int, warmup: int, flush, before_timed=None) -> dict:
        """Warm-up, then `steps` timed steps with an L2 flush before each (outside
        the per-step events). Returns per-call mean ms and the per-step ms."""
        import torch
        for _ in range(warmup):
            flush.zero_()
            self.step()
        torch.cuda.synchronize(self.dev)
        if self.st.read() != 0:
            raise RuntimeError(f"device status {self.st.read()} after warm-up ({self.cfg.name})")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(CALLS) + 1)] for _ in range(steps)]
        if before_timed:
            before_timed()
        torch.cuda.synchronize(self.dev)
        for i in range(steps):
            flush.zero_()
            self.step(evs[i])
        torch.cuda.synchronize(self.dev)
        if self.st.read() != 0:
            raise RuntimeError(f"device status {self.st.read()} after the timed steps ({self.cfg.name})")
        per_call = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(CALLS)}
        step_ms = [e[0].elapsed_time(e[len(CALLS)]) for e in evs]
        return {"per_call_ms": per_call, "step_ms": step_ms}

    def run_layer(self, steps: int, warmup: int, flush, before_timed=None) -> list:
        """Warm-up, then `steps` timed one-call layer steps (layer_step), an L2
        flush before each outside its events. Returns the per-step ms."""
        import torch
        for _ in range(warmup):
            flush.zero_()
            self.layer_step()
        torch.cuda.synchronize(self.dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        if before_timed:
            before_timed()
        torch.cuda.synchronize(self.dev)
        for e0, e1 in evs:
            flush.zero_()
            e0.record(self.stream)
            self.layer_step()
            e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        if self.st.read() != 0:
            raise RuntimeError(f"device status {self.st.read()} after the timed layer steps ({self.cfg.name})")
        return [e0.elapsed_time(e1) for e0, e1 in evs]

    def touched_experts(self) -> int:
        off = self.offsets.cpu().numpy()
        return int(np.count_nonzero(np.diff(off)))

    def summary(self, timing: dict, layer_ms: list) -> dict:
        """Throughput (from the one-call layer steps layer_ms), per-call times
        and rooflines of one configuration."""
        cfg = self.cfg
        fl = layer_flops(cfg)
        pk = peaks()
        ms = statistics.mean(layer_ms)
        pc = timing["per_call_ms"]
        gu_tflops = fl["gate_up"] / (pc["ffn_gate_up"] * 1e-3) / 1e12
        return {"workload": workload_config(cfg)["workload"], "ms_per_step": ms,
                "tokens_per_s": cfg.T / (ms * 1e-3), "assignments_per_s": cfg.T * cfg.k / (ms * 1e-3),
                "tflops": fl["total"] / (ms * 1e-3) / 1e12, "per_call_ms": pc,
                "gate_up_frac": gu_tflops / pk["bf16_tflops"],
                "layer_roofline": layer_roofline(cfg, self.touched_experts(), ms)}


def time_e2e(lb: LayerBench, steps: int, dev, dist: bool, world: int) -> dict:
    """The metric through the public API from pinned host memory: each step
    copies its token batch in, runs tqp_moe_layer_fwd and copies the layer
    output back. Two device buffers alternate, so that the copies of one step
    overlap the compute of the neighbouring steps (copy-in and copy-out streams,
    ordered by events)."""
    import torch
    Q, cfg = lb.Q, lb.cfg
    T, d = cfg.T, cfg.d
    x_host = torch.from_numpy(lb.x_bits.view(np.int16)).pin_memory()
    y_host = [torch.empty(T, d, dtype=torch.int16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(lb.x) for _ in range(2)]
    y_dev = [torch.empty_like(lb.y) for _ in range(2)]
    comp = lb.stream
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for b in range(2):
        comp_done[b].record(comp)
        out_done[b].record(comp)

    def one(i):
        b = i % 2
        s_in.wait_event(comp_done[b])            # step i-2's layer has read x_dev[b]
        with torch.cuda.stream(s_in):
            x_dev[b].copy_(x_host, non_blocking=True)
        in_done[b].record(s_in)
        comp.wait_event(in_done[b])
        comp.wait_event(out_done[b])             # step i-2's output has left y_dev[b]
        Q.tqp_moe_layer_fwd(x_dev[b], lb.L, y_dev[b], lb.ws_l, lb.st)
        comp_done[b].record(comp)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(y_dev[b], non_blocking=True)
        out_done[b].record(s_out)

    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    if dist:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    for i in range(steps):
        one(i)
    comp.wait_event(out_done[(steps - 1) % 2])
    comp.wait_event(out_done[steps % 2])
    e1.record(comp)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev, dist) / steps
    return {"value": weak_scaling_value(world, T, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": int(T * d * 2),
            "d2h_bytes_per_step": int(T * d * 2), "ms_per_step": e2e_ms,
            "note": "tqp_moe_layer_fwd per step; copy-in, compute and copy-out of neighbouring steps overlap "
                    "(two device buffers, three streams)"}


def run_tqp(args, rank: int, world: int, local_rank: int) -> dict | None:
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = synth.CONFIGS[args.config]
    lb = LayerBench(cfg, dev, rank_token_seed(cfg, rank))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    dist = world > 1
    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[0])
                          if "CUDA_VISIBLE_DEVICES" in os.environ else local_rank)

    def before_timed():
        if rank == 0:
            clocks.start()
            time.sleep(0.4)
        if dist:
            torch.distributed.barrier()

    # the headline: K passes of the layer through its one-call entry point; then
    # the same K passes through the per-part calls with events between the parts
    # for the per-kernel breakdown (the events add about 1.5 % to a step)
    step_ms = lb.run_layer(args.steps, args.warmup, flush, before_timed)
    if dist:
        torch.distributed.barrier()
    clk = clocks.stop() if rank == 0 else None
    max_ms = max_over_ranks(float(sum(step_ms)), dev, dist)
    timing = lb.run(args.steps, 1, flush)
    e2e = None if args.no_e2e else time_e2e(lb, args.steps, dev, dist, world)
    if lb.st.read() != 0:
        raise RuntimeError(f"device status {lb.st.read()} after the e2e steps")
    if rank != 0:
        return None

    T, A = cfg.T, cfg.T * cfg.k
    ms = max_ms / args.steps
    fl = layer_flops(cfg)
    pk = peaks()
    per_call_ms = timing["per_call_ms"]
    ffn_ms = sum(per_call_ms[n] for n in CALLS if n.startswith("ffn_"))
    ffn_tflops = fl["ffn"] / (ffn_ms * 1e-3) / 1e12
    gu_ms = per_call_ms["ffn_gate_up"]
    gu_tflops = fl["gate_up"] / (gu_ms * 1e-3) / 1e12
    result = {
        "metric": METRIC, "value": weak_scaling_value(world, T, ms), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded N(0,1) tokens, N(0,1/d) weights int4-quantised, random-init LoRA)",
        "config": dict(workload_config(cfg), l2="flushed before every step (512 MB write); weights 1.4 GB > L2",
                       parallelism=f"dp{world} (independent token batches, replicated weights)"),
        "tflops": fl["total"] / (ms * 1e-3) / 1e12 * world,
        "assignments_per_s": world * A / (ms * 1e-3),
        "per_call_ms": dict(per_call_ms, grouped_ffn=ffn_ms),
        "roofline": {"bound": "tensor",
                     "kernel": "gateup_wide_kernel (int4 -> fp16 weights in TMEM, 64 gate + 64 up features x up to 256 rows per unit, tcgen05 + SwiGLU)",
                     "achieved": gu_tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": gu_tflops / pk["bf16_tflops"],
                     "traffic": measured_traffic("gateup_wide_kernel") if args.config == "full" else None,
                     "traffic_source": "profiles/expert_traffic_full.md (ncu dram__bytes_read+write, one launch)",
                     "peak_source": f"{pk['source']} bf16 dense burst (fp16 has the same nominal rate)",
                     "flop_per_launch": fl["gate_up"], "ms_per_launch": gu_ms},
        "layer_roofline": layer_roofline(cfg, lb.touched_experts(), ms),
        "ffn_call": {"achieved_tflops": ffn_tflops, "frac": ffn_tflops / pk["bf16_tflops"], "ms": ffn_ms,
                     "flop": fl["ffn"]},
        "gpu_launches": args.steps * sum(lb.launches.values()),
        "clocks": clk,
        "e2e": e2e,
    }
    if world == 1 and args.config == "full" and not args.no_extra_configs:
        extra = {}
        n = min(args.steps, 10)
        mid = LayerBench(synth.MID, dev, synth.MID.seed)
        extra["mid"] = mid.summary(mid.run(n, args.warmup, flush), mid.run_layer(n, 1, flush))
        del mid
        sk_host = dict(lb.host, cfg=synth.SKEWED, bias=synth.zipf_bias(synth.SKEWED.E, synth.SKEWED.zipf_s))
        sk = LayerBench(synth.SKEWED, dev, synth.SKEWED.seed, host=sk_host)
        extra["skewed"] = sk.summary(sk.run(n, args.warmup, flush), sk.run_layer(n, 1, flush))
        del sk
        torch.cuda.empty_cache()
        i8cfg = dataclasses.replace(synth.FULL, name="full_int8", bits=8)
        i8 = LayerBench(i8cfg, dev, i8cfg.seed)
        extra["full_int8"] = i8.summary(i8.run(n, args.warmup, flush), i8.run_layer(n, 1, flush))
        del i8
        torch.cuda.empty_cache()
        result["configs"] = extra
    if world == 1 and not args.no_rev:
        result["rev_block"] = time_rev_block(lb.L, cfg, dev, min(args.steps, 5), 2, flush)
    host, x_bits = lb.host, lb.x_bits
    if world == 1 and args.config == "full" and not args.no_stack:
        del lb
        torch.cuda.empty_cache()
        result["rev_stack"] = time_stack(dev, flush)
    if world == 1 and not args.no_cpu_baseline:
        sample = min(T, args.cpu_sample)
        result["cpu_baseline"] = time_oracle(cfg, host, x_bits, sample)
    return result


def run_reference(args, rank: int) -> dict | None:
    """The reference arm: the fp64 CPU oracle (the only other implementation)."""
    if rank != 0:
        return None
    cfg = synth.CONFIGS[args.config]
    host = synth.make_layer(cfg)
    x_bits = synth.make_tokens(cfg.T, cfg.d, cfg.seed)
    sample = min(cfg.T, args.ref_sample)
    for _ in range(args.warmup):
        time_oracle(cfg, host, x_bits, 1)    # untimed
    vals = []
    for _ in range(args.steps):
        vals.append(time_oracle(cfg, host, x_bits, sample))
    v = statistics.mean(r["value"] for r in vals)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sample / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(workload_config(cfg), sample=f"oracle on the first {sample} tokens per step"),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores(), "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="full", choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="tqp", choices=["tqp", "reference"])
    ap.add_argument("--cpu-sample", type=int, default=256, help="tokens of the cpu_baseline sample")
    ap.add_argument("--ref-sample", type=int, default=8, help="tokens per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-rev", action="store_true", help="skip timing the reversible block (forward, inverse, "
                                                             "adapter backward)")
    ap.add_argument("--no-extra-configs", action="store_true", help="skip the mid and skewed configurations")
    ap.add_argument("--no-stack", action="store_true", help="skip the reversible stack's memory and time against depth")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res))
        return
    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_tqp(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if res is not None:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
