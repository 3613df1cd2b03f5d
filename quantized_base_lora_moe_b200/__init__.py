"""Python binding of the B200 TQP MoE library (libtqpmoe.so, C ABI in include/tqp_moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch provides device memory and the current CUDA stream. There is
no fallback: if the shared library is missing or the device is not a CUDA GPU
the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

__all__ = [
    "lib", "TQPError", "DeviceLayer", "Status", "workspace",
    "moe_router_gemm", "moe_route", "moe_permute", "moe_permute_noalloc", "tqp_grouped_ffn", "tqp_grouped_ffn_part",
    "moe_combine", "tqp_moe_layer_fwd",
    "rev_couple_fwd", "rev_couple_inv", "tqp_moe_layer_bwd", "tqp_adapter_bwd",
    "header_functions", "tqp_debug_set_wait_limit_ns",
    "ReversibleStack", "rev_stack_fwd", "rev_stack_inv", "rev_stack_bwd",
    "tqp_adamw_step", "AdapterAdamW",
]

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libtqpmoe.so")
HEADER = os.path.join(ROOT, "include", "tqp_moe.h")

TQP_OK = 0
ERRORS = {-1: "invalid argument", -2: "unsupported configuration", -3: "workspace too small",
          -4: "CUDA launch or runtime error"}
STATUS_NONFINITE, STATUS_BAD_ID, STATUS_TIMEOUT, STATUS_RANGE = 1, 2, 4, 8
FFN_PREPARE, FFN_GATE_UP, FFN_RANK, FFN_DOWN = 0, 1, 2, 3
DTYPE_BF16, DTYPE_F32 = 0, 1


class TQPError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {ERRORS.get(code, 'unknown')} ({code})")
        self.code = code


class Weights(ctypes.Structure):
    _fields_ = [
        ("E", ctypes.c_int), ("d", ctypes.c_int), ("ffn", ctypes.c_int), ("group", ctypes.c_int),
        ("rank", ctypes.c_int), ("top_k", ctypes.c_int), ("lora_scale", ctypes.c_float),
        ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
        ("wq", ctypes.c_void_p * 3), ("wscale", ctypes.c_void_p * 3),
        ("lora_a", ctypes.c_void_p * 3), ("lora_b", ctypes.c_void_p * 3), ("bits", ctypes.c_int),
    ]


class Grads(ctypes.Structure):
    _fields_ = [("dA", ctypes.c_void_p * 3), ("dB", ctypes.c_void_p * 3)]


_VP, _I, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_WP = ctypes.POINTER(Weights)
_GP = ctypes.POINTER(Grads)
_SIGS = {
    "tqp_version": (_I, []),
    "tqp_error_string": (ctypes.c_char_p, [_I]),
    "moe_router_gemm_workspace_size": (_SZ, [_I, _WP]),
    "moe_router_gemm": (_I, [_VP, _I, _WP, _VP, _VP, _SZ, _VP, _VP]),
    "moe_route": (_I, [_VP, _I, _I, _I, _VP, _VP, _VP, _VP]),
    "moe_permute_workspace_size": (_SZ, [_I, _I, _I]),
    "moe_permute": (_I, [_VP, _I, _I, _I, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "moe_permute_noalloc_max_bytes": (_SZ, []),
    "moe_permute_noalloc": (_I, [_VP, _I, _I, _I, _VP, _VP, _VP, _VP, _VP]),
    "tqp_grouped_ffn_workspace_size": (_SZ, [_I, _WP]),
    "tqp_grouped_ffn": (_I, [_VP, _I, _VP, _VP, _WP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "tqp_grouped_ffn_part": (_I, [_I, _VP, _I, _VP, _VP, _WP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "moe_combine": (_I, [_VP, _VP, _VP, _I, _I, _I, _VP, _I, _F, _VP, _I, _VP, _VP]),
    "tqp_moe_layer_workspace_size": (_SZ, [_I, _WP]),
    "tqp_moe_layer_fwd": (_I, [_VP, _I, _WP, _VP, _VP, _SZ, _VP, _VP]),
    "rev_couple_workspace_size": (_SZ, [_I, _WP, _WP]),
    "rev_couple_fwd": (_I, [_VP, _VP, _I, _WP, _WP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "rev_couple_inv": (_I, [_VP, _VP, _I, _WP, _WP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "tqp_moe_layer_bwd_workspace_size": (_SZ, [_I, _WP]),
    "tqp_moe_layer_bwd": (_I, [_VP, _VP, _I, _WP, _VP, _GP, _VP, _SZ, _VP, _VP]),
    "tqp_adapter_bwd_workspace_size": (_SZ, [_I, _WP, _WP]),
    "tqp_adapter_bwd": (_I, [_VP, _VP, _VP, _VP, _I, _WP, _WP, _VP, _VP, _VP, _VP, _GP, _GP, _VP, _SZ, _VP,
                             _VP]),
    "tqp_debug_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "tqp_adamw_step": (_I, [_VP, _VP, _VP, _VP, _VP, _SZ, _F, _F, _F, _F, _F, _I, _F, _VP, _VP]),
    "rev_stack_workspace_size": (_SZ, [_I, _I, _VP, _VP]),
    "rev_stack_fwd": (_I, [_VP, _VP, _I, _I, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "rev_stack_inv": (_I, [_VP, _VP, _I, _I, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "rev_stack_bwd": (_I, [_VP, _VP, _VP, _VP, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP,
                           _VP]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libtqpmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m quantized_base_lora_moe_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/tqp_moe.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(\w+)\s*\(", text, flags=re.M)))


def _check(name: str, rc: int) -> None:
    if rc != TQP_OK:
        raise TQPError(name, rc)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _require_cuda(*tensors) -> None:
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors passed to the TQP library must live on a CUDA device")


def _require_int32(name: str, t, min_numel: int, ndim: int | None = None) -> None:
    """The C ABI reads int32 arrays through raw pointers: refuse anything else
    (an int64 tensor would be read as pairs of int32, an undersized output
    would be written past its end)."""
    import torch
    if t.dtype != torch.int32 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 tensor (got {t.dtype}, contiguous={t.is_contiguous()})")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions (got {t.dim()})")
    if t.numel() < min_numel:
        raise ValueError(f"{name} needs at least {min_numel} elements (got {t.numel()})")


def _permute_args(ids, E: int, offsets, perm_token, inv) -> tuple[int, int]:
    _require_int32("ids", ids, 0, ndim=2)
    T, k = ids.shape
    _require_int32("offsets", offsets, E + 1)
    _require_int32("perm_token", perm_token, T * k)
    _require_int32("inv", inv, T * k)
    _require_cuda(ids, offsets, perm_token, inv)
    return T, k


class Status:
    """Device status word (int32, zeroed); read() synchronises and returns the bits."""

    def __init__(self, device="cuda"):
        import torch
        self.t = torch.zeros(1, dtype=torch.int32, device=device)

    def ptr(self) -> int:
        return self.t.data_ptr()

    def read(self) -> int:
        return int(self.t.item())

    def clear(self) -> None:
        self.t.zero_()


def workspace(nbytes: int, device="cuda"):
    import torch
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def _bf16_tensor(a: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)


class DeviceLayer:
    """One TQP layer's weights resident on the GPU plus its tqp_moe_weights struct.

    Built from the host arrays produced by synth.make_layer (storage formats as
    in include/tqp_moe.h).
    """

    def __init__(self, host: dict, device="cuda", top_k: int | None = None):
        import torch
        cfg = host["cfg"]
        self.cfg = cfg
        self.E, self.d, self.f, self.g, self.r = cfg.E, cfg.d, cfg.f, cfg.g, cfg.r
        self.k = top_k or cfg.k
        self.s = float(cfg.lora_scale)
        self.bits = int(getattr(cfg, "bits", 4))
        self.router_w = torch.from_numpy(np.ascontiguousarray(host["router_w"], np.float32)).to(device)
        self.bias = None if host.get("bias") is None else torch.from_numpy(
            np.ascontiguousarray(host["bias"], np.float32)).to(device)
        self.wq = [torch.from_numpy(np.ascontiguousarray(host[f"wq{p}"])).to(device) for p in range(3)]
        self.ws = [_bf16_tensor(host[f"ws{p}"], device) for p in range(3)]
        # the six adapter factors as views of one flat bf16 buffer, in the order of
        # the flat gradient buffer (A_gate, A_up, A_down, B_gate, B_up, B_down), so
        # that one optimizer call updates the whole layer
        parts = [np.ascontiguousarray(host[f"la{p}"]) for p in range(3)] + \
                [np.ascontiguousarray(host[f"lb{p}"]) for p in range(3)]
        self.lora_flat = torch.from_numpy(np.concatenate([a.reshape(-1) for a in parts]).view(np.int16)).to(device)
        views, off = [], 0
        for a in parts:
            views.append(self.lora_flat[off:off + a.size].view(a.shape))
            off += a.size
        self.la, self.lb = views[:3], views[3:]
        self._struct = None

    @property
    def struct(self) -> Weights:
        if self._struct is None:
            w = Weights()
            w.E, w.d, w.ffn, w.group, w.rank, w.top_k = self.E, self.d, self.f, self.g, self.r, self.k
            w.lora_scale = self.s
            w.bits = self.bits
            w.router_w = self.router_w.data_ptr()
            w.router_bias = _ptr(self.bias)
            for p in range(3):
                w.wq[p] = self.wq[p].data_ptr()
                w.wscale[p] = self.ws[p].data_ptr()
                w.lora_a[p] = self.la[p].data_ptr() if self.r > 0 else None
                w.lora_b[p] = self.lb[p].data_ptr() if self.r > 0 else None
            self._struct = w
        return self._struct

    def ref(self):
        return ctypes.byref(self.struct)

    def grads(self, device="cuda"):
        """Zeroed fp32 adapter-gradient buffers and their tqp_adapter_grads struct."""
        import torch
        dims = [(self.f, self.d), (self.f, self.d), (self.d, self.f)]
        dA = [torch.zeros(self.E, self.r, inn, dtype=torch.float32, device=device) for (_, inn) in dims]
        dB = [torch.zeros(self.E, out, self.r, dtype=torch.float32, device=device) for (out, _) in dims]
        g = Grads()
        for p in range(3):
            g.dA[p] = dA[p].data_ptr()
            g.dB[p] = dB[p].data_ptr()
        return dA, dB, g

    def flat_grads(self, device="cuda"):
        """The same buffers as views of one flat fp32 tensor (dp.FlatGrads), so a
        data-parallel backward sums them over ranks in a single all-reduce."""
        from .dp import FlatGrads
        return FlatGrads(self.E, self.d, self.f, self.r, device)


# ---------------------------------------------------------------- entry points (same names as the C ABI)


def _grads(g):
    """A tqp_adapter_grads struct, or a dp.FlatGrads (its struct)."""
    return g.struct if hasattr(g, "struct") and not isinstance(g, Grads) else g


def moe_router_gemm(x, layer: DeviceLayer, logits, ws=None, status: Status | None = None, stream=None):
    _require_cuda(x, logits)
    T = x.shape[0]
    n = lib().moe_router_gemm_workspace_size(T, layer.ref())
    ws = ws if ws is not None else workspace(n, x.device)
    _check("moe_router_gemm", lib().moe_router_gemm(x.data_ptr(), T, layer.ref(), logits.data_ptr(), ws.data_ptr(),
                                                     ws.numel(), status.ptr() if status else None, _stream(stream)))
    return logits


def moe_route(logits, k: int, ids, gates, status: Status | None = None, stream=None):
    _require_cuda(logits, ids, gates)
    T, E = logits.shape
    _check("moe_route", lib().moe_route(logits.data_ptr(), T, E, k, ids.data_ptr(), gates.data_ptr(),
                                        status.ptr() if status else None, _stream(stream)))
    return ids, gates


def moe_permute(ids, E: int, offsets, perm_token, inv, ws=None, status: Status | None = None, stream=None):
    T, k = _permute_args(ids, E, offsets, perm_token, inv)
    n = lib().moe_permute_workspace_size(T, E, k)
    ws = ws if ws is not None else workspace(n, ids.device)
    _check("moe_permute", lib().moe_permute(ids.data_ptr(), T, E, k, offsets.data_ptr(), perm_token.data_ptr(),
                                            inv.data_ptr(), ws.data_ptr(), ws.numel(),
                                            status.ptr() if status else None, _stream(stream)))
    return offsets, perm_token, inv


def moe_permute_noalloc(ids, E: int, offsets, perm_token, inv, status: Status | None = None, stream=None):
    """moe_permute with its scratch in the library's fixed device array (no workspace)."""
    T, k = _permute_args(ids, E, offsets, perm_token, inv)
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(ids.data_ptr(), T, E, k, offsets.data_ptr(),
                                                            perm_token.data_ptr(), inv.data_ptr(),
                                                            status.ptr() if status else None, _stream(stream)))
    return offsets, perm_token, inv


def tqp_grouped_ffn(x, offsets, perm_token, layer: DeviceLayer, h, out_perm, ws=None, status: Status | None = None,
                    stream=None):
    _require_cuda(x, offsets, perm_token, h, out_perm)
    T = x.shape[0]
    n = lib().tqp_grouped_ffn_workspace_size(T, layer.ref())
    ws = ws if ws is not None else workspace(n, x.device)
    _check("tqp_grouped_ffn", lib().tqp_grouped_ffn(x.data_ptr(), T, offsets.data_ptr(), perm_token.data_ptr(),
                                                    layer.ref(), h.data_ptr(), out_perm.data_ptr(), ws.data_ptr(),
                                                    ws.numel(), status.ptr() if status else None, _stream(stream)))
    return h, out_perm


def tqp_grouped_ffn_part(part: int, x, offsets, perm_token, layer: DeviceLayer, h, out_perm, ws,
                         status: Status | None = None, stream=None):
    """One part of tqp_grouped_ffn (FFN_PREPARE, FFN_GATE_UP, FFN_RANK, FFN_DOWN, in order, same ws)."""
    _require_cuda(x, offsets, perm_token, h, out_perm)
    _check("tqp_grouped_ffn_part", lib().tqp_grouped_ffn_part(
        int(part), x.data_ptr(), x.shape[0], offsets.data_ptr(), perm_token.data_ptr(), layer.ref(), h.data_ptr(),
        out_perm.data_ptr(), ws.data_ptr(), ws.numel(), status.ptr() if status else None, _stream(stream)))
    return h, out_perm


def moe_combine(out_perm, inv, gates, y, residual=None, sign: float = 1.0, y_bf16=None, stream=None):
    import torch
    _require_cuda(out_perm, inv, gates, y, residual, y_bf16)
    T, k = gates.shape
    d = out_perm.shape[1]
    rdt = DTYPE_F32 if (residual is not None and residual.dtype == torch.float32) else DTYPE_BF16
    ydt = DTYPE_F32 if y.dtype == torch.float32 else DTYPE_BF16
    _check("moe_combine", lib().moe_combine(out_perm.data_ptr(), inv.data_ptr(), gates.data_ptr(), T, k, d,
                                            _ptr(residual), rdt, sign, y.data_ptr(), ydt, _ptr(y_bf16),
                                            _stream(stream)))
    return y


def tqp_moe_layer_fwd(x, layer: DeviceLayer, y, ws=None, status: Status | None = None, stream=None):
    _require_cuda(x, y)
    T = x.shape[0]
    n = lib().tqp_moe_layer_workspace_size(T, layer.ref())
    ws = ws if ws is not None else workspace(n, x.device)
    _check("tqp_moe_layer_fwd", lib().tqp_moe_layer_fwd(x.data_ptr(), T, layer.ref(), y.data_ptr(), ws.data_ptr(),
                                                        ws.numel(), status.ptr() if status else None,
                                                        _stream(stream)))
    return y


def rev_couple_fwd(x1, x2, F: DeviceLayer, G: DeviceLayer, y1, y2, ws=None, status: Status | None = None,
                   stream=None):
    _require_cuda(x1, x2, y1, y2)
    T = x1.shape[0]
    n = lib().rev_couple_workspace_size(T, F.ref(), G.ref())
    ws = ws if ws is not None else workspace(n, x1.device)
    _check("rev_couple_fwd", lib().rev_couple_fwd(x1.data_ptr(), x2.data_ptr(), T, F.ref(), G.ref(), y1.data_ptr(),
                                                  y2.data_ptr(), ws.data_ptr(), ws.numel(),
                                                  status.ptr() if status else None, _stream(stream)))
    return y1, y2


def rev_couple_inv(y1, y2, F: DeviceLayer, G: DeviceLayer, x1, x2, ws=None, status: Status | None = None,
                   stream=None):
    _require_cuda(x1, x2, y1, y2)
    T = y1.shape[0]
    n = lib().rev_couple_workspace_size(T, F.ref(), G.ref())
    ws = ws if ws is not None else workspace(n, y1.device)
    _check("rev_couple_inv", lib().rev_couple_inv(y1.data_ptr(), y2.data_ptr(), T, F.ref(), G.ref(), x1.data_ptr(),
                                                  x2.data_ptr(), ws.data_ptr(), ws.numel(),
                                                  status.ptr() if status else None, _stream(stream)))
    return x1, x2


def tqp_moe_layer_bwd(x, dy, layer: DeviceLayer, dx, grads, ws=None, status: Status | None = None, stream=None):
    _require_cuda(x, dy, dx)
    T = x.shape[0]
    n = lib().tqp_moe_layer_bwd_workspace_size(T, layer.ref())
    ws = ws if ws is not None else workspace(n, x.device)
    _check("tqp_moe_layer_bwd", lib().tqp_moe_layer_bwd(x.data_ptr(), dy.data_ptr(), T, layer.ref(), dx.data_ptr(),
                                                        ctypes.byref(_grads(grads)), ws.data_ptr(), ws.numel(),
                                                        status.ptr() if status else None, _stream(stream)))
    return dx


def tqp_adapter_bwd(y1, y2, dy1, dy2, F: DeviceLayer, G: DeviceLayer, x1, x2, dx1, dx2, gF, gG, ws=None,
                    status: Status | None = None, stream=None):
    _require_cuda(y1, y2, dy1, dy2, x1, x2, dx1, dx2)
    T = y1.shape[0]
    n = lib().tqp_adapter_bwd_workspace_size(T, F.ref(), G.ref())
    ws = ws if ws is not None else workspace(n, y1.device)
    _check("tqp_adapter_bwd", lib().tqp_adapter_bwd(y1.data_ptr(), y2.data_ptr(), dy1.data_ptr(), dy2.data_ptr(), T,
                                                    F.ref(), G.ref(), x1.data_ptr(), x2.data_ptr(), dx1.data_ptr(),
                                                    dx2.data_ptr(), ctypes.byref(_grads(gF)), ctypes.byref(_grads(gG)),
                                                    ws.data_ptr(), ws.numel(), status.ptr() if status else None,
                                                    _stream(stream)))
    return x1, x2, dx1, dx2


def tqp_debug_set_wait_limit_ns(ns: int) -> None:
    """Test hook: bound of every device-side barrier wait of the launches that
    follow (0 restores the 2 s default). See include/tqp_moe.h."""
    _check("tqp_debug_set_wait_limit_ns", lib().tqp_debug_set_wait_limit_ns(int(ns)))


# ---------------------------------------------------------------- reversible stack


class ReversibleStack:
    """L coupling blocks (F[l], G[l]) as the C ABI takes them: arrays of
    tqp_moe_weights pointers, kept alive with the layers."""

    def __init__(self, F: list, G: list):
        if len(F) != len(G) or not F:
            raise ValueError("a stack needs L >= 1 pairs of layers")
        self.F, self.G, self.L = list(F), list(G), len(F)
        self._fw = (ctypes.POINTER(Weights) * self.L)(*[ctypes.pointer(l.struct) for l in self.F])
        self._gw = (ctypes.POINTER(Weights) * self.L)(*[ctypes.pointer(l.struct) for l in self.G])

    def ptrs(self):
        return ctypes.cast(self._fw, ctypes.c_void_p), ctypes.cast(self._gw, ctypes.c_void_p)

    def workspace_size(self, T: int) -> int:
        f, g = self.ptrs()
        return int(lib().rev_stack_workspace_size(T, self.L, f, g))

    def grads(self, device="cuda"):
        """Per-layer FlatGrads for F and G, and the two pointer arrays the C ABI takes."""
        gF = [l.flat_grads(device) for l in self.F]
        gG = [l.flat_grads(device) for l in self.G]
        aF = (ctypes.POINTER(Grads) * self.L)(*[ctypes.pointer(g.struct) for g in gF])
        aG = (ctypes.POINTER(Grads) * self.L)(*[ctypes.pointer(g.struct) for g in gG])
        return gF, gG, (aF, aG)


def rev_stack_fwd(x1, x2, stack: ReversibleStack, y1, y2, ws=None, status: Status | None = None, stream=None):
    _require_cuda(x1, x2, y1, y2)
    T = x1.shape[0]
    ws = ws if ws is not None else workspace(stack.workspace_size(T), x1.device)
    f, g = stack.ptrs()
    _check("rev_stack_fwd", lib().rev_stack_fwd(x1.data_ptr(), x2.data_ptr(), T, stack.L, f, g, y1.data_ptr(),
                                                y2.data_ptr(), ws.data_ptr(), ws.numel(),
                                                status.ptr() if status else None, _stream(stream)))
    return y1, y2


def rev_stack_inv(y1, y2, stack: ReversibleStack, x1, x2, ws=None, status: Status | None = None, stream=None):
    _require_cuda(x1, x2, y1, y2)
    T = y1.shape[0]
    ws = ws if ws is not None else workspace(stack.workspace_size(T), y1.device)
    f, g = stack.ptrs()
    _check("rev_stack_inv", lib().rev_stack_inv(y1.data_ptr(), y2.data_ptr(), T, stack.L, f, g, x1.data_ptr(),
                                                x2.data_ptr(), ws.data_ptr(), ws.numel(),
                                                status.ptr() if status else None, _stream(stream)))
    return x1, x2


def rev_stack_bwd(y1, y2, dy1, dy2, stack: ReversibleStack, x1, x2, dx1, dx2, grad_arrays, ws=None,
                  status: Status | None = None, stream=None):
    """grad_arrays: the pointer arrays from ReversibleStack.grads()."""
    _require_cuda(y1, y2, dy1, dy2, x1, x2, dx1, dx2)
    T = y1.shape[0]
    ws = ws if ws is not None else workspace(stack.workspace_size(T), y1.device)
    f, g = stack.ptrs()
    aF, aG = grad_arrays
    _check("rev_stack_bwd", lib().rev_stack_bwd(
        y1.data_ptr(), y2.data_ptr(), dy1.data_ptr(), dy2.data_ptr(), T, stack.L, f, g, x1.data_ptr(),
        x2.data_ptr(), dx1.data_ptr(), dx2.data_ptr(), ctypes.cast(aF, ctypes.c_void_p),
        ctypes.cast(aG, ctypes.c_void_p), ws.data_ptr(), ws.numel(), status.ptr() if status else None,
        _stream(stream)))
    return x1, x2, dx1, dx2


# ---------------------------------------------------------------- adapter optimizer


def tqp_adamw_step(param, exp_avg, exp_avg_sq, grad, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                   eps: float = 1e-8, weight_decay: float = 0.0, grad_scale: float = 1.0, param_bf16=None,
                   status: Status | None = None, stream=None):
    """One fused AdamW step over flat fp32 buffers (see include/tqp_moe.h)."""
    import torch
    _require_cuda(param, exp_avg, exp_avg_sq, grad, param_bf16)
    n = param.numel()
    for name, t in (("exp_avg", exp_avg), ("exp_avg_sq", exp_avg_sq), ("grad", grad)):
        if t.numel() != n or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 tensor of {n} elements")
    if param.dtype != torch.float32 or not param.is_contiguous():
        raise ValueError("param must be a contiguous fp32 tensor")
    if param_bf16 is not None and (param_bf16.numel() != n or param_bf16.element_size() != 2):
        raise ValueError("param_bf16 must hold n 16-bit values")
    _check("tqp_adamw_step", lib().tqp_adamw_step(param.data_ptr(), exp_avg.data_ptr(), exp_avg_sq.data_ptr(),
                                                  grad.data_ptr(), _ptr(param_bf16), n, lr, beta1, beta2, eps,
                                                  weight_decay, int(step), grad_scale,
                                                  status.ptr() if status else None, _stream(stream)))


class AdapterAdamW:
    """AdamW over one layer's adapters: fp32 master copy and moments in the
    flat gradient layout, and the layer's bf16 factors rewritten by each step.

    step(grads) takes the layer's FlatGrads (summed over data-parallel ranks
    already, if any)."""

    def __init__(self, layer: DeviceLayer, lr: float, betas=(0.9, 0.999), eps: float = 1e-8,
                 weight_decay: float = 0.0):
        import torch
        self.layer, self.lr, self.betas, self.eps, self.wd = layer, lr, betas, eps, weight_decay
        self.master = layer.lora_flat.view(torch.bfloat16).float()
        self.exp_avg = torch.zeros_like(self.master)
        self.exp_avg_sq = torch.zeros_like(self.master)
        self.t = 0

    def step(self, grads, grad_scale: float = 1.0, status: Status | None = None, stream=None):
        flat = grads.flat if hasattr(grads, "flat") else grads
        self.t += 1
        tqp_adamw_step(self.master, self.exp_avg, self.exp_avg_sq, flat, self.t, self.lr, self.betas[0],
                       self.betas[1], self.eps, self.wd, grad_scale, self.layer.lora_flat, status, stream)
