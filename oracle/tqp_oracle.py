"""Plain fp64 CPU oracle for the TQP MoE layer and its reversible coupling.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import or call this
module: only the tests, the smoke check in __graft_entry__ and the benchmark's
CPU-baseline leg do. It shares no code with the CUDA path and decodes the input
formats itself.

What it computes, and where that comes from ("Reversible Sparse MoE Single
Node" = the skills-directory page; "Abstract" = the arXiv abstract of
"Reversible Foundations: Training a 120B Sparse MoE through State-Preserving
Scaling"):

* frozen base expert weights are quantised, adapters are trained low-rank
  factors, the router is full precision: TQP ("Principle 3: TQP Optimizer
  Strategy"; "TQP Quantization" under "Implementation Considerations";
  Abstract, "Single-node economics").
* 460 routed experts with top-12 routing ("Architecture Details"; Abstract).
* routing is stateless, so it is recomputed from the inputs during the inverse
  (the routing item of "Reversibility Implementation").
* reversible residual (RevNet-style) blocks whose inverse uses subtraction, and
  the backward pass reconstructs activations from the final state instead of
  storing them ("Principle 1: Reversible Recurrence Stack"; "Pattern 1";
  "Reversibility Implementation"; Abstract, "Reversibility").

The pages give no equations for the router gate, the expert FFN, the quantiser
or the coupling. The readings used here (renormalised softmax over the top-k
logits, lowest-id tie-break, SwiGLU experts with LoRA W' = W + s*A*B on gate, up
and down, symmetric int4 with bf16 group scales, additive coupling y1 = x1 +
F(x2), y2 = x2 + G(y1) with bf16 layer inputs) are listed with their reasons in
the design notes at the repository root.

Parity status: every function here is pinned by the CPU tests in
tests/test_oracle_pins.py (brute force, closed forms, library reductions,
invariants, finite differences). None is "parity unpinned".

Precision: all arithmetic in float64. The only roundings are the ones that are
part of the definition: the layer consumes bf16 activations, so G's input
bf16(y1) is rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# input format decoding
# ----------------------------------------------------------------------------


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned as float64.

    bf16 keeps 8 significant bits: x = m * 2^e with 0.5 <= |m| < 1, so the
    rounded value is rint(m * 2^8) * 2^(e-8). Normal range only (the layer's
    activations are O(1)); zeros pass through.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def unpack_int4(codes) -> np.ndarray:
    """Packed int4 codes [..., K/2] uint8 -> signed integers [..., K].

    Each little-endian 32-bit word covers 8 consecutive K positions; position
    2i sits in bits [4i, 4i+4), position 2i+1 in bits [16+4i, 16+4i+4), as
    two's-complement nibbles.
    """
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    words = c.view("<u4").astype(np.int64)
    K = c.shape[-1] * 2
    out = np.empty(c.shape[:-1] + (K // 8, 8), dtype=np.int64)
    for i in range(4):
        out[..., 2 * i] = (words >> (4 * i)) & 0xF
        out[..., 2 * i + 1] = (words >> (16 + 4 * i)) & 0xF
    out = np.where(out >= 8, out - 16, out)
    return out.reshape(c.shape[:-1] + (K,))


def unpack_int8(codes) -> np.ndarray:
    """int8 codes [..., K] (two's-complement bytes) -> signed integers [..., K]."""
    return np.ascontiguousarray(codes, dtype=np.uint8).view(np.int8).astype(np.int64)


def dequant(codes, scales, g: int, bits: int = 4) -> np.ndarray:
    """Dequantised weight W[n, k] = q[n, k] * scale[k // g, n], exact in fp64.

    codes [out][in/2] (packed int4) or [out][in] (int8, bits = 8), scales
    [in/g][out] bf16 bits. Base expert weights are stored as int8 or int4
    ("TQP Quantization").
    """
    q = (unpack_int4(codes) if bits == 4 else unpack_int8(codes)).astype(np.float64)
    s = bf16_to_f64(scales)                      # [in/g][out]
    return q * np.repeat(s.T, g, axis=1)


# ----------------------------------------------------------------------------
# layer parameters, decoded per expert
# ----------------------------------------------------------------------------


class Layer:
    """Decoded fp64 view of one TQP layer's weights, one expert at a time.

    Parameters follow the x @ W convention: projection p maps rows of width
    in_p to width out_p as  x @ W_p^T + s * (x @ A_p) @ B_p  with W_p [out][in]
    (dequantised base), A_p [in][r], B_p [r][out].
    """

    def __init__(self, raw: dict, overrides: dict | None = None):
        cfg = raw["cfg"]
        self.raw = raw
        self.E, self.d, self.f, self.g, self.r = cfg.E, cfg.d, cfg.f, cfg.g, cfg.r
        self.bits = getattr(cfg, "bits", 4)
        self.k = cfg.k
        self.s = float(cfg.lora_scale)
        self.router_w = np.asarray(raw["router_w"], dtype=np.float64)   # [E][d]
        b = raw.get("bias")
        self.bias = None if b is None else np.asarray(b, dtype=np.float64)
        self.overrides = overrides or {}
        self._cache: dict = {}
        # keep every decoded expert for small layers, a few for large ones
        self._cache_cap = self.E if self.E * self.d * self.f <= (1 << 26) else 4

    def expert(self, e: int) -> dict:
        if e in self._cache:
            return self._cache[e]
        raw = self.raw
        p_ = {}
        for p, name in enumerate(("g", "u", "d")):
            p_[f"W{name}"] = dequant(raw[f"wq{p}"][e], raw[f"ws{p}"][e], self.g, self.bits)
            p_[f"A{name}"] = bf16_to_f64(raw[f"la{p}"][e]).T          # [in][r]
            p_[f"B{name}"] = bf16_to_f64(raw[f"lb{p}"][e]).T          # [r][out]
        p_.update(self.overrides.get(e, {}))
        if len(self._cache) >= self._cache_cap:
            self._cache.pop(next(iter(self._cache)))
        self._cache[e] = p_
        return p_


# ----------------------------------------------------------------------------
# router, top-k, gates
# ----------------------------------------------------------------------------


def router_logits(x, L: Layer) -> np.ndarray:
    """Full-precision router: l[t, e] = sum_i x[t, i] * W_r[e, i] (+ bias[e]).

    The pages keep the router at full precision because routing quality
    depends on it (the router item of the TQP Quantization list). The additive bias is the skewed-load workload's per-expert
    popularity term, added before both top-k and the gates.
    """
    l = np.asarray(x, dtype=np.float64) @ L.router_w.T
    if L.bias is not None:
        l = l + L.bias[None, :]
    return l


def topk(logits, k: int) -> np.ndarray:
    """Top-k expert ids per token, by descending logit; exact ties -> lower id first.

    Top-12 routing ("Architecture Details"). Implemented as a full stable sort
    of each row on (is-NaN, -logit, expert id), keeping the first k: NaN ranks
    below every number (-inf included) and +0.0 ties with -0.0.
    """
    l = np.asarray(logits, dtype=np.float64)
    nan = np.isnan(l)
    neg = np.where(nan, 0.0, -l)
    T, E = l.shape
    ids = np.empty((T, k), dtype=np.int32)
    eidx = np.arange(E)
    for t in range(T):
        order = np.lexsort((eidx, neg[t], nan[t]))   # last key is the primary one
        ids[t] = order[:k]
    return ids


def gates(logits, ids) -> np.ndarray:
    """Renormalised softmax over the chosen logits.

    gamma[t, j] = exp(l[t, id_j] - m) / sum_j' exp(l[t, id_j'] - m), m the largest
    chosen logit. Equal to the full softmax over all experts renormalised over
    the top k (the common factor cancels).
    """
    l = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(l, np.asarray(ids, dtype=np.int64), axis=1)
    m = sel.max(axis=1, keepdims=True)
    e = np.exp(sel - m)
    return e / e.sum(axis=1, keepdims=True)


def routing_gap(logits, k: int) -> np.ndarray:
    """Per token: (k-th largest logit) - ((k+1)-th largest); +inf when k == E."""
    l = np.sort(np.asarray(logits, dtype=np.float64), axis=1)[:, ::-1]
    if k >= l.shape[1]:
        return np.full(l.shape[0], np.inf)
    return l[:, k - 1] - l[:, k]


# ----------------------------------------------------------------------------
# token -> expert permutation
# ----------------------------------------------------------------------------


def permute(ids, E: int):
    """Stable counting sort of the (token, slot) assignments by expert.

    offsets[e] = number of assignments to experts < e (offsets[E] = T*k);
    inside an expert, rows are in increasing token order (a token picks an
    expert at most once). perm_token[row] = token of that row;
    inv[t*k + j] = row that holds assignment (t, j).
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    counts = np.zeros(E, dtype=np.int64)
    for e in ids.ravel():
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].copy()
    perm_token = np.empty(T * k, dtype=np.int64)
    inv = np.empty(T * k, dtype=np.int64)
    # walk tokens in order: rows of each expert come out sorted by token
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            row = fill[e]
            fill[e] += 1
            perm_token[row] = t
            inv[t * k + j] = row
    return offsets, perm_token, inv


# ----------------------------------------------------------------------------
# experts
# ----------------------------------------------------------------------------


def silu(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def sigmoid(z):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def expert_forward(X, P: dict, s: float) -> dict:
    """SwiGLU expert with LoRA on gate, up and down (rows of X are routed tokens).

    gate = X Wg^T + s (X Ag) Bg ; up = X Wu^T + s (X Au) Bu ;
    h = silu(gate) * up ; o = h Wd^T + s (h Ad) Bd.
    The base W comes from the frozen int4 codes, A and B are the trained
    low-rank adapters ("Principle 3"; "Pattern 3: TQP Optimizer for Sparse
    Models").
    """
    X = np.asarray(X, dtype=np.float64)
    xa_g = X @ P["Ag"]
    xa_u = X @ P["Au"]
    gate = X @ P["Wg"].T + s * (xa_g @ P["Bg"])
    up = X @ P["Wu"].T + s * (xa_u @ P["Bu"])
    h = silu(gate) * up
    ha = h @ P["Ad"]
    o = h @ P["Wd"].T + s * (ha @ P["Bd"])
    return {"xa_g": xa_g, "xa_u": xa_u, "gate": gate, "up": up, "h": h, "ha": ha, "o": o}


def layer_forward(x, L: Layer, ids=None, want_cache: bool = False):
    """TQP MoE layer: y[t] = sum_j gamma[t, j] * expert_{id[t, j]}(x[t]).

    x is a float64 [T][d] array holding bf16 values. The routing (ids) is
    recomputed from x unless given. Returns y (and the per-expert cache used by
    the backward when want_cache).
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    logits = router_logits(x, L)
    if ids is None:
        ids = topk(logits, L.k)
    gam = gates(logits, ids)
    y = np.zeros_like(x)
    cache = {"logits": logits, "ids": ids, "gates": gam, "experts": {}}
    for e in np.unique(ids):
        t_idx, j_idx = np.nonzero(ids == e)
        out = expert_forward(x[t_idx], L.expert(int(e)), L.s)
        y[t_idx] += gam[t_idx, j_idx][:, None] * out["o"]
        if want_cache:
            cache["experts"][int(e)] = (t_idx, j_idx, out)
    return (y, cache) if want_cache else y


def combine(o_rows, gam, inv, T: int, k: int) -> np.ndarray:
    """y[t] = sum_j gamma[t, j] * o[inv[t*k + j]] (permuted expert outputs back to tokens)."""
    o_rows = np.asarray(o_rows, dtype=np.float64)
    y = np.zeros((T, o_rows.shape[1]))
    for t in range(T):
        for j in range(k):
            y[t] += gam[t, j] * o_rows[inv[t * k + j]]
    return y


# ----------------------------------------------------------------------------
# reversible additive coupling
# ----------------------------------------------------------------------------


def coupling_forward(x1, x2, F: Layer, G: Layer, round_g_input: bool = True):
    """y1 = x1 + F(x2); y2 = x2 + G(bf16(y1)).

    RevNet-style additive coupling ("Reversibility Implementation": reversible
    residual blocks; "Pattern 1": addition/subtraction are invertible). Layers
    take bf16 activations, so G sees y1 rounded to bf16 (round_g_input=False
    drops that rounding; the tests use it for smooth finite differences).
    """
    x1 = np.asarray(x1, dtype=np.float64)
    x2 = np.asarray(x2, dtype=np.float64)
    y1 = x1 + layer_forward(x2, F)
    y2 = x2 + layer_forward(round_bf16(y1) if round_g_input else y1, G)
    return y1, y2


def coupling_inverse(y1, y2, F: Layer, G: Layer):
    """x2 = y2 - G(bf16(y1)); x1 = y1 - F(x2): the backward's reconstruction
    from the block's outputs ("Principle 1": layer.inverse(state) walking the
    stack in reverse)."""
    y1 = np.asarray(y1, dtype=np.float64)
    y2 = np.asarray(y2, dtype=np.float64)
    x2 = y2 - layer_forward(round_bf16(y1), G)
    x1 = y1 - layer_forward(x2, F)
    return x1, x2


# ----------------------------------------------------------------------------
# backward (adapters only; base and router frozen)
# ----------------------------------------------------------------------------


def expert_backward(X, dO, P: dict, s: float, fwd: dict) -> dict:
    """Closed-form gradients of one expert for upstream dO (rows of X).

    Returns dX and the adapter gradients in storage layout: dA^T [r][in],
    dB^T [out][r] for gate, up, down. Base weights get no gradient: they stay
    frozen in their quantised form (the base-weight item of the TQP
    Quantization list).
    """
    h, gate, up = fwd["h"], fwd["gate"], fwd["up"]
    ha, xa_g, xa_u = fwd["ha"], fwd["xa_g"], fwd["xa_u"]
    X = np.asarray(X, dtype=np.float64)
    # down projection
    dBd = s * ha.T @ dO                       # [r][d]
    dha = s * dO @ P["Bd"].T                  # [n][r]
    dAd = h.T @ dha                           # [f][r]
    dh = dO @ P["Wd"] + dha @ P["Ad"].T       # [n][f]
    # SwiGLU
    sg = sigmoid(gate)
    sl = gate * sg
    dsl = sg * (1.0 + gate * (1.0 - sg))
    dgate = dh * up * dsl
    dup = dh * sl
    # gate / up projections
    dBg = s * xa_g.T @ dgate
    dBu = s * xa_u.T @ dup
    dxa_g = s * dgate @ P["Bg"].T
    dxa_u = s * dup @ P["Bu"].T
    dAg = X.T @ dxa_g
    dAu = X.T @ dxa_u
    dX = dgate @ P["Wg"] + dxa_g @ P["Ag"].T + dup @ P["Wu"] + dxa_u @ P["Au"].T
    return {"dX": dX,
            "dA": [dAg.T, dAu.T, dAd.T],
            "dB": [dBg.T, dBu.T, dBd.T]}


def layer_backward(x, dy, L: Layer, ids=None):
    """Gradients of <dy, layer(x)> w.r.t. x and all adapters.

    Top-k selection is piecewise constant (no gradient through the choice); the
    gates' softmax over the chosen logits passes gradient to x through the
    frozen router:  dl_j = gamma_j (dgamma_j - sum_j' gamma_j' dgamma_j'),
    dx += sum_j dl_j W_r[id_j].
    Returns (dx, dA, dB) with dA[p] [E][r][in_p], dB[p] [E][out_p][r].
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    T, d = x.shape
    y, cache = layer_forward(x, L, ids=ids, want_cache=True)
    ids, gam = cache["ids"], cache["gates"]
    dx = np.zeros_like(x)
    dgam = np.zeros_like(gam)
    dims = [(L.f, L.d), (L.f, L.d), (L.d, L.f)]
    dA = [np.zeros((L.E, L.r, inn)) for (_, inn) in dims]
    dB = [np.zeros((L.E, out, L.r)) for (out, _) in dims]
    for e, (t_idx, j_idx, fwd) in cache["experts"].items():
        g_rows = gam[t_idx, j_idx][:, None]
        dO = g_rows * dy[t_idx]
        dgam[t_idx, j_idx] = np.sum(dy[t_idx] * fwd["o"], axis=1)
        res = expert_backward(x[t_idx], dO, L.expert(e), L.s, fwd)
        np.add.at(dx, t_idx, res["dX"])
        for p in range(3):
            dA[p][e] = res["dA"][p]
            dB[p][e] = res["dB"][p]
    dl = gam * (dgam - np.sum(gam * dgam, axis=1, keepdims=True))
    for j in range(ids.shape[1]):
        dx += dl[:, j:j + 1] * L.router_w[ids[:, j]]
    return dx, dA, dB


def block_backward(y1, y2, dy1, dy2, F: Layer, G: Layer, round_g_input: bool = True):
    """Reversible block backward from its outputs only.

    G-step: recompute G on bf16(y1), reconstruct x2 = y2 - G(bf16(y1)), take G's
    adapter gradients for cotangent dy2 and dz1 = dy1 + J_G^T dy2.
    F-step: recompute F(x2), reconstruct x1 = y1 - F(x2), take F's adapter
    gradients for cotangent dz1; dx2 = dy2 + J_F^T dz1, dx1 = dz1.
    ("Principle 1": reconstruct from the final state, compute gradients
    locally.) The bf16 rounding at G's input passes gradients unchanged.
    """
    y1 = np.asarray(y1, dtype=np.float64)
    y2 = np.asarray(y2, dtype=np.float64)
    z = round_bf16(y1) if round_g_input else y1
    x2 = y2 - layer_forward(z, G)
    dxG, dAG, dBG = layer_backward(z, dy2, G)
    dz1 = np.asarray(dy1, dtype=np.float64) + dxG
    x1 = y1 - layer_forward(x2, F)
    dxF, dAF, dBF = layer_backward(x2, dz1, F)
    dx2 = np.asarray(dy2, dtype=np.float64) + dxF
    return {"x1": x1, "x2": x2, "dx1": dz1, "dx2": dx2,
            "dA_F": dAF, "dB_F": dBF, "dA_G": dAG, "dB_G": dBG}


def block_backward_stored(x1, x2, dy1, dy2, F: Layer, G: Layer):
    """Same gradients from the stored block inputs (the non-reversible baseline)."""
    x1 = np.asarray(x1, dtype=np.float64)
    x2 = np.asarray(x2, dtype=np.float64)
    y1 = x1 + layer_forward(x2, F)
    z = round_bf16(y1)
    dxG, dAG, dBG = layer_backward(z, dy2, G)
    dz1 = np.asarray(dy1, dtype=np.float64) + dxG
    dxF, dAF, dBF = layer_backward(x2, dz1, F)
    return {"dx1": dz1, "dx2": np.asarray(dy2, dtype=np.float64) + dxF,
            "dA_F": dAF, "dB_F": dBF, "dA_G": dAG, "dB_G": dBG}


# ----------------------------------------------------------------------------
# reversible stack of coupling blocks
# ----------------------------------------------------------------------------


def stack_forward(x1, x2, blocks, round_inputs: bool = True):
    """L coupling blocks applied in order ("Principle 1: Reversible Recurrence
    Stack": the forward pass runs the blocks one after the other, keeping only
    the final state).

    blocks: list of (F, G) Layers. Block l maps the streams (a1, a2) to
    b1 = a1 + F(bf16(a2)), b2 = a2 + G(bf16(b1)): the streams are carried
    exactly (fp64 here) and each layer reads its stream rounded to bf16, its
    input format. Block 0 reads the bf16 inputs x1, x2, so one block is
    coupling_forward. round_inputs=False drops the roundings (smooth in every
    input, for finite differences).
    """
    rb = round_bf16 if round_inputs else (lambda v: v)
    a1 = np.asarray(x1, dtype=np.float64)
    a2 = np.asarray(x2, dtype=np.float64)
    for F, G in blocks:
        b1 = a1 + layer_forward(rb(a2), F)
        b2 = a2 + layer_forward(rb(b1), G)
        a1, a2 = b1, b2
    return a1, a2


def stack_inverse(y1, y2, blocks, round_inputs: bool = True):
    """Reconstruct the stack's inputs from its outputs, last block first:
    a2 = b2 - G(bf16(b1)), a1 = b1 - F(bf16(a2)) ("Principle 1": the backward
    pass walks the stack in reverse through each layer's inverse)."""
    rb = round_bf16 if round_inputs else (lambda v: v)
    b1 = np.asarray(y1, dtype=np.float64)
    b2 = np.asarray(y2, dtype=np.float64)
    for F, G in reversed(blocks):
        a2 = b2 - layer_forward(rb(b1), G)
        a1 = b1 - layer_forward(rb(a2), F)
        b1, b2 = a1, a2
    return b1, b2


def stack_backward(y1, y2, dy1, dy2, blocks, round_inputs: bool = True):
    """Gradients of <dy1, y1> + <dy2, y2> for the whole stack from its outputs
    alone ("Principle 1": reconstruct each layer's input from its output, then
    take that layer's gradients locally, last block first).

    Per block, with outputs (b1, b2) and their cotangents (g1, g2):
    z = bf16(b1); a2 = b2 - G(z); G's adapter gradients for cotangent g2 and
    dz1 = g1 + J_G(z)^T g2; a1 = b1 - F(bf16(a2)); F's adapter gradients for
    cotangent dz1; the block's input cotangents are (dz1, g2 + J_F^T dz1). The
    bf16 roundings pass gradients unchanged. Returns x1, x2 (reconstructed),
    dx1, dx2 and grads[l] = (dA_F, dB_F, dA_G, dB_G) for every block l.
    """
    rb = round_bf16 if round_inputs else (lambda v: v)
    b1 = np.asarray(y1, dtype=np.float64)
    b2 = np.asarray(y2, dtype=np.float64)
    g1 = np.asarray(dy1, dtype=np.float64)
    g2 = np.asarray(dy2, dtype=np.float64)
    grads = []
    for F, G in reversed(blocks):
        z = rb(b1)
        a2 = b2 - layer_forward(z, G)
        dxG, dAG, dBG = layer_backward(z, g2, G)
        dz1 = g1 + dxG
        ab = rb(a2)
        a1 = b1 - layer_forward(ab, F)
        dxF, dAF, dBF = layer_backward(ab, dz1, F)
        g1, g2 = dz1, g2 + dxF
        b1, b2 = a1, a2
        grads.append((dAF, dBF, dAG, dBG))
    grads.reverse()
    return {"x1": b1, "x2": b2, "dx1": g1, "dx2": g2, "grads": grads}


def stack_backward_stored(x1, x2, dy1, dy2, blocks, round_inputs: bool = True):
    """The same gradients with every block's inputs stored during the forward
    (the non-reversible baseline that reversibility replaces)."""
    rb = round_bf16 if round_inputs else (lambda v: v)
    a1 = np.asarray(x1, dtype=np.float64)
    a2 = np.asarray(x2, dtype=np.float64)
    saved = []
    for F, G in blocks:
        saved.append((a1, a2))
        b1 = a1 + layer_forward(rb(a2), F)
        b2 = a2 + layer_forward(rb(b1), G)
        a1, a2 = b1, b2
    g1 = np.asarray(dy1, dtype=np.float64)
    g2 = np.asarray(dy2, dtype=np.float64)
    grads = []
    for (a1, a2), (F, G) in zip(reversed(saved), reversed(blocks)):
        b1 = a1 + layer_forward(rb(a2), F)
        dxG, dAG, dBG = layer_backward(rb(b1), g2, G)
        dz1 = g1 + dxG
        dxF, dAF, dBF = layer_backward(rb(a2), dz1, F)
        g1, g2 = dz1, g2 + dxF
        grads.append((dAF, dBF, dAG, dBG))
    grads.reverse()
    return {"dx1": g1, "dx2": g2, "grads": grads}


# ----------------------------------------------------------------------------
# adapter optimizer step
# ----------------------------------------------------------------------------


def adamw_step(p, m, v, g, lr, beta1, beta2, eps, weight_decay, t, grad_scale=1.0):
    """One AdamW step (Adam with decoupled weight decay, Loshchilov & Hutter)
    over adapter parameters: the only trained, optimizer-carrying parameters
    ("Principle 3: TQP Optimizer Strategy"; "Pattern 3"). The pages do not name
    the optimizer; this is the reading used.

    g' = grad_scale g; m <- beta1 m + (1 - beta1) g'; v <- beta2 v + (1 - beta2) g'^2;
    m_hat = m / (1 - beta1^t); v_hat = v / (1 - beta2^t);
    p <- p - lr (m_hat / (sqrt(v_hat) + eps) + weight_decay p).
    Returns the new (p, m, v) as float64 arrays.
    """
    p = np.asarray(p, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64) * grad_scale
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    p = p - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * p)
    return p, m, v


# ----------------------------------------------------------------------------
# per-token evaluation (for sampled checks at full size)
# ----------------------------------------------------------------------------


def token_forward(xt, L: Layer):
    """One token through the layer: (y_t, ids_t, gates_t, logits_t). Same
    arithmetic as layer_forward restricted to one row."""
    xt = np.asarray(xt, dtype=np.float64)[None, :]
    logits = router_logits(xt, L)
    ids = topk(logits, L.k)
    gam = gates(logits, ids)
    y = np.zeros_like(xt)
    for j in range(L.k):
        y += gam[0, j] * expert_forward(xt, L.expert(int(ids[0, j])), L.s)["o"]
    return y[0], ids[0], gam[0], logits[0]
