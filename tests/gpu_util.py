"""Shared helpers of the GPU parity tests (device transfers, error metrics)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import tqp_oracle as O


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def host_bf16(t: torch.Tensor) -> np.ndarray:
    return O.bf16_to_f64(t.cpu().numpy().view(np.uint16))


def host_f16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.float16).astype(np.float64)


def dev_f16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16).view(np.int16)).cuda()


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(dtype) if dtype is not None else t).cuda()


def stream_grid(x: np.ndarray) -> np.ndarray:
    """x rounded to the coupling's stream grid, multiples of 2^-16 (half to
    even): what the coupling's inverse returns for a bf16 input x. Every bf16
    value of magnitude 2^-9 or more is unchanged."""
    return np.rint(np.asarray(x, np.float64) * 65536.0) / 65536.0


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(got - ref)) / max(np.sqrt(np.mean(ref * ref)), 1e-30))


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 values at |v| (8 significant bits)."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    return np.where(v > 0, np.ldexp(1.0, (e - 8).astype(np.int64)), 0.0)


def rel_err_bf16_out(got, ref) -> float:
    """max(|got - ref| - half-ulp of the bf16 output) / RMS(ref).

    A bf16 output carries its own rounding error of up to half an ulp (2^-9 of
    |ref|); for heavy-tailed layer outputs that alone reaches about 2% of the
    RMS. This metric measures the computation's error beyond that rounding.
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    slack = np.maximum(bf16_half_ulp(ref), bf16_half_ulp(got))
    excess = np.maximum(np.abs(got - ref) - slack, 0.0)
    return float(np.max(excess) / max(np.sqrt(np.mean(ref * ref)), 1e-30))


def near_tie_tokens(logits64: np.ndarray, k: int, margin: float) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th logits are closer than margin (routing ambiguous at fp32)."""
    return O.routing_gap(logits64, k) < margin
