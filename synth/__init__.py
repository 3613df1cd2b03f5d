"""Seeded synthetic inputs for the TQP MoE layer and its reversible block.

This module is shared by the CPU oracle, the GPU tests and the benchmark. It
only draws random numbers and encodes them into the storage formats that both
sides consume (bf16 bit patterns, packed int4 codes with bf16 group scales). It
contains none of the layer's arithmetic: no routing, no expert FFN, no combine,
no coupling.

The frozen base expert weights of a TQP layer are stored quantised (the TQP
strategy of "Reversible Sparse MoE Single Node", section "Principle 3: TQP
Optimizer Strategy", and its "TQP Quantization" list: base weights int8 or
int4, adapters and router full precision). The quantiser below runs once on the
host to produce those frozen codes; the hot path only ever dequantises them.

Storage formats (shared contract with the C-ABI, see include/tqp_moe.h):

* bf16 values are carried as uint16 bit patterns (round-to-nearest-even from
  fp32).
* int8 codes (bits = 8) of one projection, per expert, are an [out][in] array of
  two's-complement bytes.
* int4 codes of one projection, per expert, are a [out][in/2] uint8 array made of
  little-endian 32-bit words. Each word holds 8 consecutive input-dimension
  values k0..k7 of one output row as two's-complement nibbles: k(2i) sits in bits
  [4i, 4i+4) and k(2i+1) in bits [16+4i, 16+4i+4), i = 0..3 (evens in the low
  half-word, odds in the high half-word).
* group scales are bf16, laid out [in/g][out] per expert (group-major, output
  rows contiguous).
* LoRA factors are stored transposed: A^T [r][in] and B^T [out][r], both bf16,
  for the update W' = W + s * A B in x @ W form.

Every tensor is drawn from its own PCG64 stream keyed by
SeedSequence([seed, tag, expert]), so any single expert can be regenerated on
its own and generation runs in parallel threads.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# ----------------------------------------------------------------------------
# configurations
# ----------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shape of one TQP MoE layer and of the token batch it runs on."""

    name: str
    T: int          # tokens
    d: int          # d_model
    E: int          # routed experts
    k: int          # top-k
    f: int          # expert SwiGLU hidden width
    g: int          # quantisation group along the input dimension
    r: int          # LoRA rank
    lora_scale: float = 2.0   # alpha / r
    zipf_s: float = 0.0       # >0: additive router bias ln(p_e), p_e ~ (e+1)^-s
    seed: int = 0
    w_mult: float = 1.0       # multiplies the base weights (before quantising) and LoRA B
    bits: int = 4             # base-weight code width: 4 (packed int4) or 8 (int8)

    @property
    def A(self) -> int:
        return self.T * self.k


TINY = LayerConfig("tiny", T=64, d=128, E=8, k=2, f=256, g=32, r=8)
MID = LayerConfig("mid", T=2048, d=1024, E=64, k=8, f=512, g=64, r=16)
FULL = LayerConfig("full", T=8192, d=2048, E=460, k=12, f=768, g=64, r=32)
SKEWED = LayerConfig("skewed", T=16384, d=2048, E=460, k=12, f=768, g=64, r=32,
                     zipf_s=1.1)
# reversible block: F = FULL with seed 0, G = FULL with seed 1; x1 seed 2,
# x2 seed 3, upstream gradients seed 4.
REV_F = FULL
REV_G = dataclasses.replace(FULL, name="full_g", seed=1)
REV_SEEDS = {"x1": 2, "x2": 3, "dy": 4}

# profiling case: the full layer's shapes with 64 experts (151 MB of int4 codes,
# larger than L2, a few hundred MB on the device in total)
PROF = LayerConfig("prof", T=4096, d=2048, E=64, k=8, f=768, g=64, r=32)

CONFIGS = {c.name: c for c in (TINY, MID, FULL, SKEWED, PROF)}

# stream tags
_TAG = {"router": 1, "w0": 2, "w1": 3, "w2": 4, "a0": 5, "a1": 6, "a2": 7,
        "b0": 8, "b1": 9, "b2": 10, "x": 11, "dy1": 12, "dy2": 13}

PROJ = ("gate", "up", "down")


def _rng(seed: int, tag: str, e: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAG[tag], e])))


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


# ----------------------------------------------------------------------------
# encodings
# ----------------------------------------------------------------------------


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (NaN kept quiet)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    nan = np.isnan(a)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = ((u[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Signed codes q[..., K] in [-8, 7] -> packed uint8 [..., K/2] (format in module doc)."""
    q = np.asarray(q)
    K = q.shape[-1]
    assert K % 8 == 0
    nib = (q.astype(np.int32) & 0xF).astype(np.uint32).reshape(q.shape[:-1] + (K // 8, 8))
    word = np.zeros(nib.shape[:-1], dtype=np.uint32)
    for i in range(4):
        word |= nib[..., 2 * i] << np.uint32(4 * i)
        word |= nib[..., 2 * i + 1] << np.uint32(16 + 4 * i)
    return np.ascontiguousarray(word.astype("<u4")).view(np.uint8).reshape(q.shape[:-1] + (K // 2,))


def quantise_int4(w: np.ndarray, g: int) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric group-wise int4 quantiser for one expert's [out][in] fp32 weight.

    scale = bf16(absmax / 7) per group of g consecutive inputs; q = clamp(rint(w /
    scale), -7, 7); an all-zero group gets scale 0 and codes 0. Returns the
    packed codes [out][in/2] and the scale bits laid out [in/g][out].
    """
    w = np.asarray(w, dtype=np.float32)
    out, inn = w.shape
    wg = w.reshape(out, inn // g, g)
    amax = np.abs(wg).max(axis=2)
    sbits = f32_to_bf16_bits(amax / np.float32(7.0))
    s = bf16_bits_to_f32(sbits)
    safe = np.where(s == 0, np.float32(1.0), s)
    q = np.rint(wg / safe[:, :, None])
    q = np.clip(q, -7, 7)
    q[s == 0] = 0
    q = q.astype(np.int8).reshape(out, inn)
    return pack_int4(q), np.ascontiguousarray(sbits.T)


def quantise_int8(w: np.ndarray, g: int) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric group-wise int8 quantiser for one expert's [out][in] fp32 weight.

    scale = bf16(absmax / 127) per group of g consecutive inputs; q = clamp(rint(w /
    scale), -127, 127); an all-zero group gets scale 0 and codes 0. Returns the
    codes [out][in] as int8 bytes (two's complement, stored uint8) and the scale
    bits laid out [in/g][out].
    """
    w = np.asarray(w, dtype=np.float32)
    out, inn = w.shape
    wg = w.reshape(out, inn // g, g)
    amax = np.abs(wg).max(axis=2)
    sbits = f32_to_bf16_bits(amax / np.float32(127.0))
    s = bf16_bits_to_f32(sbits)
    safe = np.where(s == 0, np.float32(1.0), s)
    q = np.rint(wg / safe[:, :, None])
    q = np.clip(q, -127, 127)
    q[s == 0] = 0
    q = q.astype(np.int8).reshape(out, inn)
    return np.ascontiguousarray(q.view(np.uint8)), np.ascontiguousarray(sbits.T)


# ----------------------------------------------------------------------------
# layer weights and activations
# ----------------------------------------------------------------------------


def zipf_bias(E: int, s: float) -> np.ndarray:
    """Additive router bias b_e = ln p_e with p_e proportional to (e+1)^-s."""
    i = np.arange(1, E + 1, dtype=np.float64)
    p = i ** (-s)
    p /= p.sum()
    return np.log(p).astype(np.float32)


def proj_dims(cfg: LayerConfig, p: int) -> tuple[int, int]:
    """(out, in) of projection p (0 gate, 1 up, 2 down)."""
    return (cfg.f, cfg.d) if p < 2 else (cfg.d, cfg.f)


def _expert_tensors(cfg: LayerConfig, seed: int, p: int, e: int):
    out, inn = proj_dims(cfg, p)
    std_w = np.float32(1.0 / np.sqrt(cfg.d))
    mult = np.float32(cfg.w_mult)
    w = _rng(seed, f"w{p}", e).standard_normal((out, inn), dtype=np.float32) * std_w * mult
    codes, scales = quantise_int4(w, cfg.g) if cfg.bits == 4 else quantise_int8(w, cfg.g)
    at = f32_to_bf16_bits(_rng(seed, f"a{p}", e).standard_normal((cfg.r, inn), dtype=np.float32) * std_w)
    bt = f32_to_bf16_bits(_rng(seed, f"b{p}", e).standard_normal((out, cfg.r), dtype=np.float32)
                          * np.float32(0.1) * mult)
    return codes, scales, at, bt


def make_layer(cfg: LayerConfig, seed: int | None = None, threads: int | None = None) -> dict:
    """All weights of one TQP MoE layer as numpy arrays (host memory).

    keys: router_w [E][d] f32; bias [E] f32 or None; for p in 0,1,2:
    wq{p} [E][out][in/2] u8, ws{p} [E][in/g][out] u16 (bf16), la{p} [E][r][in]
    u16 (A^T), lb{p} [E][out][r] u16 (B^T); plus the scalar config fields.
    """
    seed = cfg.seed if seed is None else seed
    E = cfg.E
    layer = {"cfg": cfg, "seed": seed}
    layer["router_w"] = (_rng(seed, "router").standard_normal((E, cfg.d), dtype=np.float32)
                         * np.float32(1.0 / np.sqrt(cfg.d)))
    layer["bias"] = zipf_bias(E, cfg.zipf_s) if cfg.zipf_s > 0 else None
    for p in range(3):
        out, inn = proj_dims(cfg, p)
        layer[f"wq{p}"] = np.empty((E, out, inn * cfg.bits // 8), np.uint8)
        layer[f"ws{p}"] = np.empty((E, inn // cfg.g, out), np.uint16)
        layer[f"la{p}"] = np.empty((E, cfg.r, inn), np.uint16)
        layer[f"lb{p}"] = np.empty((E, out, cfg.r), np.uint16)

    def job(pe):
        p, e = pe
        c, s, a, b = _expert_tensors(cfg, seed, p, e)
        layer[f"wq{p}"][e] = c
        layer[f"ws{p}"][e] = s
        layer[f"la{p}"][e] = a
        layer[f"lb{p}"][e] = b

    jobs = [(p, e) for p in range(3) for e in range(E)]
    n = threads or _threads()
    if n == 1 or len(jobs) < 8:
        for j in jobs:
            job(j)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(job, jobs))
    return layer


def expert_slice(layer: dict, e: int) -> dict:
    """Views of one expert's weights (for per-expert oracle work)."""
    out = {"cfg": layer["cfg"]}
    for p in range(3):
        for key in ("wq", "ws", "la", "lb"):
            out[f"{key}{p}"] = layer[f"{key}{p}"][e]
    return out


def make_tokens(T: int, d: int, seed: int, tag: str = "x") -> np.ndarray:
    """Activations [T][d] ~ N(0, 1) as bf16 bits."""
    return f32_to_bf16_bits(_rng(seed, tag).standard_normal((T, d), dtype=np.float32))


def make_grad(T: int, d: int, seed: int, tag: str) -> np.ndarray:
    """Upstream gradient [T][d] ~ N(0, 1) fp32."""
    return _rng(seed, tag).standard_normal((T, d), dtype=np.float32)


def make_inputs(cfg: LayerConfig) -> dict:
    """Layer weights plus the token batch x for a forward config."""
    layer = make_layer(cfg)
    return {"layer": layer, "x": make_tokens(cfg.T, cfg.d, cfg.seed)}


def make_rev_inputs(cfgF: LayerConfig = REV_F, cfgG: LayerConfig = REV_G, T: int | None = None,
                    seeds: dict | None = None) -> dict:
    """Reversible block inputs: layers F, G, streams x1, x2 (bf16), grads dy1, dy2 (f32)."""
    seeds = seeds or REV_SEEDS
    T = T or cfgF.T
    return {
        "F": make_layer(cfgF, cfgF.seed),
        "G": make_layer(cfgG, cfgG.seed),
        "x1": make_tokens(T, cfgF.d, seeds["x1"]),
        "x2": make_tokens(T, cfgF.d, seeds["x2"]),
        "dy1": make_grad(T, cfgF.d, seeds["dy"], "dy1"),
        "dy2": make_grad(T, cfgF.d, seeds["dy"], "dy2"),
    }


def make_logits(T: int, E: int, seed: int, ties: bool = False, bias: np.ndarray | None = None) -> np.ndarray:
    """Router-logit stand-ins [T][E] fp32 ~ N(0, 1) (the router's logit scale).

    ties=True snaps every other token's row to a coarse grid (multiples of 1/4)
    and plants +0.0 / -0.0 pairs, so exact ties are frequent. bias (optional)
    is added in fp32, as the skewed-load workload's router does.
    """
    rng = _rng(seed, "x", 7)
    l = rng.standard_normal((T, E), dtype=np.float32)
    if ties:
        l[::2] = np.round(l[::2] * 4) / 4
        if E >= 4:
            l[::3, 1] = np.float32(0.0)
            l[::3, 2] = np.float32(-0.0)
    if bias is not None:
        l = (l + bias[None, :].astype(np.float32)).astype(np.float32)
    return np.ascontiguousarray(l)
