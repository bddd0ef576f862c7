"""Plain CPU oracle of the HGRNBit block forward (ternary BitLinear + HGRN recurrence).

TEST INFRASTRUCTURE. Only the test suite, the package's ``__graft_entry__.smoke()`` check and
the CPU-baseline leg of ``bench.py`` may import this module. The product path (the CUDA
library and its Python binding) never calls it, and this module imports nothing from the
product package: the two share no code, only the seeded generators in ``synth``.

Everything here is a direct, unblocked restatement of the method as the MatMul-free LM pages
describe it, in float64 for floating point and int64 for integer sums. Sources (page title,
section):

* nightvoyager.top "MatMul-Free LLM 深度分析报告", table "创新之处" (innovations):
  ternary ``weight_quant`` is round-to-nearest onto {-1, 0, +1}; the token mixer is the gated
  linear recurrence h_t = g_t * h_{t-1} + x_t with O(T*D) cost.
* same page, "可复用的模式与技巧" (reusable patterns): FusedBitLinear fuses RMSNorm with INT8
  activation quantisation; the STE only matters for training.
* hysenlabs.com "HGRNBitBlock 的結構" (block structure): each of i/f/g/o_proj, gate_proj and
  down_proj is a FusedBitLinear with its own RMSNorm of eps=1e-08; g_norm is
  FusedRMSNormSwishGate; the MLP is gate_proj -> SiLU -> down_proj with gate_proj emitting
  twice the width down_proj consumes (11264 vs 5632 at hidden 2048).
* mooersco.com section 4.1: a ternary matrix-vector product is a conditional add / subtract
  (w = 1 adds, w = -1 subtracts, w = 0 skips); used here as the brute-force dot product.

The pages leave several steps open; the readings taken (absmax-to-127 activation codes, a
per-tensor absmean weight scale with floor 1e-5, ties to even, f = sigmoid(zf),
i = SiLU(zi) * (1 - f), residuals around the token mixer and the MLP, no bias, h_0 = 0,
gate half first in the GLU split) are each restated in the function that takes it.

Where floating point decides an integer code, this oracle takes the decision in float32, the
precision of the CUDA path: the weight code is rint(float32(W) / float32(s)) and the activation
code is rint(float32(r) * float32(127 / absmax)). Everything else stays in float64.

``hgrn2_recurrence`` (HGRN2's state expansion, a next step beyond the HGRN block) takes the one
step the pages leave entirely open: they name HGRN2 but print no equations, so it restates the
published HGRN2 recurrence (see its docstring). The ``*_backward`` functions give the gradients
of a training step, exact for the smooth parts and straight-through for the two quantisers.

Parity is pinned for every function here by tests/test_oracle_pins.py (closed forms, hand-worked
recurrences, brute force on tiny shapes, statistical and structural invariants).
"""
from __future__ import annotations

import numpy as np

EPS_NORM = 1e-8     # RMSNorm eps printed for every FusedBitLinear (hysenlabs.com, block structure)
EPS_QUANT = 1e-5    # floor on absmean / absmax scales (reading: the pages print no value)
QMAX = 127          # activation codes live in [-127, 127]


# ----------------------------------------------------------------------------------------------
# elementwise definitions
# ----------------------------------------------------------------------------------------------
def sigmoid(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU (Swish with beta 1): z * sigmoid(z)."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def rmsnorm(x: np.ndarray, w: np.ndarray | None, eps: float = EPS_NORM) -> np.ndarray:
    """r = x / sqrt(mean(x^2) + eps) * w over the last axis (RMSNorm, eps=1e-08 per the block
    structure printed on hysenlabs.com)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    r = x / np.sqrt(ms + eps)
    if w is not None:
        r = r * np.asarray(w, dtype=np.float64)
    return r


# ----------------------------------------------------------------------------------------------
# quantisers
# ----------------------------------------------------------------------------------------------
def weight_scale(W: np.ndarray) -> np.float32:
    """Per-tensor absmean scale s = max(mean|W|, 1e-5), summed in float64 and stored as the one
    float32 scale of the packed format."""
    W = np.asarray(W, dtype=np.float64)
    s = float(np.mean(np.abs(W))) if W.size else 0.0
    return np.float32(max(s, EPS_QUANT))


def ternarize(W: np.ndarray) -> tuple[np.ndarray, np.float32]:
    """weight_quant: codes t = clip(rint(W / s), -1, 1) in {-1, 0, +1} and the scale s, so that
    W is approximated by t * s (nightvoyager.top, innovations table: round-to-nearest ternary).

    The code decision is taken in float32 (IEEE division, ties to even)."""
    W32 = np.asarray(W, dtype=np.float32)
    s = weight_scale(W32)
    t = np.clip(np.rint(W32 / s), -1, 1).astype(np.int8)
    return t, s


def act_quant(r: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per-token absmax INT8 quantisation of the normalised rows r (last axis).

    a = max(max|r|, 1e-5); q = clip(rint(r * 127 / a), -127, 127); r is approximated by
    q * (a / 127). The decision runs in float32 on float32(r), like the kernel.

    Returns (q int8, deq = a/127 float64 per row, v = the float32 value that was rounded)."""
    r32 = np.asarray(r, dtype=np.float64).astype(np.float32)
    a = np.max(np.abs(r32), axis=-1, keepdims=True) if r32.shape[-1] else np.zeros(r32.shape[:-1] + (1,), np.float32)
    a = np.maximum(a, np.float32(EPS_QUANT)).astype(np.float32)
    sx = (np.float32(QMAX) / a).astype(np.float32)
    v = (r32 * sx).astype(np.float32)
    q = np.clip(np.rint(v), -QMAX, QMAX).astype(np.int8)
    deq = a[..., 0].astype(np.float64) / QMAX
    return q, deq, v


# ----------------------------------------------------------------------------------------------
# 2-bit packed format
# ----------------------------------------------------------------------------------------------
def packed_row_words(k: int) -> int:
    """u32 words per packed row: 16 codes per word, rows padded to 64 codes (16 bytes)."""
    return 4 * ((k + 63) // 64)


def code_bit(j: int) -> int:
    """Bit offset of the code for column k = 16*w + j inside word w (0 <= j < 16).

    Codes are grouped in quads of four consecutive columns, j = 4*quad + lane. The quad picks a
    16-bit half (quad // 2) and a 2-bit sub-position inside each nibble (2 * (quad % 2)); the
    lane picks the nibble (4 * lane)."""
    quad, lane = divmod(j, 4)
    return 16 * (quad >> 1) + 2 * (quad & 1) + 4 * lane


_FIELD = {0: 0b00, 1: 0b01, -1: 0b11}
_VALUE = {0b00: 0, 0b01: 1, 0b11: -1}


def pack_codes(t: np.ndarray) -> np.ndarray:
    """Pack ternary codes t [N, K] into u32 words [N, packed_row_words(K)]: two's-complement 2-bit
    fields (00 = 0, 01 = +1, 11 = -1) at the offsets of ``code_bit``; padding columns hold 0.
    Written as plain loops over columns."""
    t = np.asarray(t, dtype=np.int64)
    n, k = t.shape
    kw = packed_row_words(k)
    words = np.zeros((n, kw), dtype=np.uint64)
    for col in range(k):
        w, j = divmod(col, 16)
        c = t[:, col]
        if np.any((c < -1) | (c > 1)):
            raise ValueError(f"code outside {{-1, 0, 1}} at column {col}")
        field = np.where(c == 1, _FIELD[1], np.where(c == -1, _FIELD[-1], _FIELD[0])).astype(np.uint64)
        words[:, w] |= field << np.uint64(code_bit(j))
    return words.astype(np.uint32)


def unpack_codes(words: np.ndarray, k: int) -> np.ndarray:
    """Inverse of ``pack_codes``: u32 words [N, KW] -> int8 codes [N, k]. Raises on the unused
    field value 10."""
    words = np.asarray(words, dtype=np.uint64)
    n = words.shape[0]
    t = np.zeros((n, k), dtype=np.int8)
    for col in range(k):
        w, j = divmod(col, 16)
        f = (words[:, w] >> np.uint64(code_bit(j))) & np.uint64(3)
        if np.any(f == 2):
            raise ValueError(f"invalid 2-bit field 10 at column {col}")
        t[:, col] = np.where(f == _FIELD[1], 1, np.where(f == _FIELD[-1], -1, 0)).astype(np.int8)
    return t


def count_malformed_fields(words: np.ndarray, k: int) -> int:
    """Integrity of a packed matrix [N, KW] holding K real columns: the number of 2-bit fields
    that ``pack_codes`` never writes -- a real column (col < k) holding the unused pattern 10, or
    a padding column (k <= col < 16 * KW) holding anything but 00. Each field counts once.
    Written as plain loops over the columns of the format."""
    words = np.asarray(words, dtype=np.uint64)
    n, kw = words.shape
    bad = 0
    for col in range(16 * kw):
        w, j = divmod(col, 16)
        f = (words[:, w] >> np.uint64(code_bit(j))) & np.uint64(3)
        if col < k:
            bad += int(np.count_nonzero(f == 2))
        else:
            bad += int(np.count_nonzero(f != 0))
    return bad


# ----------------------------------------------------------------------------------------------
# BitLinear
# ----------------------------------------------------------------------------------------------
def ternary_dot_condadd(t_row: np.ndarray, q: np.ndarray) -> int:
    """Brute-force ternary dot product by conditional add / subtract (mooersco.com section 4.1):
    +1 adds the activation, -1 subtracts it, 0 skips. Pure Python; tiny inputs only."""
    s = 0
    for w, a in zip(t_row.tolist(), q.tolist()):
        if w == 1:
            s += a
        elif w == -1:
            s -= a
    return s


def int_matmul(q: np.ndarray, t: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[m, k] * t[n, k] in int64 (exact), asserted to fit int32."""
    acc = np.asarray(q, dtype=np.int64) @ np.asarray(t, dtype=np.int64).T
    if acc.size:
        assert np.abs(acc).max() < 2**31
    return acc


def bitlinear(x: np.ndarray, norm_w: np.ndarray | None, t: np.ndarray, s_w: float,
              eps: float = EPS_NORM) -> tuple[np.ndarray, dict]:
    """FusedBitLinear forward: RMSNorm -> per-token absmax int8 -> exact integer product with the
    ternary codes -> rescale by (a/127) * s_w (nightvoyager.top reusable patterns; hysenlabs.com
    block structure). No bias.

    Returns (y float64 [..., N], taps) with taps = {'r','q','deq','v','acc'}."""
    x = np.asarray(x, dtype=np.float64)
    lead = x.shape[:-1]
    k = x.shape[-1]
    x2 = x.reshape(-1, k)
    r = rmsnorm(x2, norm_w, eps)
    q, deq, v = act_quant(r)
    acc = int_matmul(q, t)
    y = acc.astype(np.float64) * deq[:, None] * float(s_w)
    taps = {"r": r, "q": q, "deq": deq, "v": v, "acc": acc}
    return y.reshape(lead + (t.shape[0],)), taps


def dense_reference(q: np.ndarray, deq: np.ndarray, t: np.ndarray, s_w: float) -> np.ndarray:
    """The same product computed the other way round: dequantise both operands first
    (q * deq and t * s_w) and take a dense float64 matrix product."""
    A = np.asarray(q, dtype=np.float64) * np.asarray(deq, dtype=np.float64)[:, None]
    B = np.asarray(t, dtype=np.float64) * float(s_w)
    return A @ B.T


# ----------------------------------------------------------------------------------------------
# HGRN recurrence
# ----------------------------------------------------------------------------------------------
def hgrn_gates(zf: np.ndarray, zi: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Forget gate f = sigmoid(zf); input i = SiLU(zi) * (1 - f)."""
    f = sigmoid(zf)
    i = silu(zi) * (1.0 - f)
    return f, i


def hgrn_scan(f: np.ndarray, i: np.ndarray, h0: np.ndarray | None = None) -> np.ndarray:
    """Sequential gated linear recurrence h_t = f_t * h_{t-1} + i_t over axis 1 of [B, T, D]
    (nightvoyager.top innovations table), h_{-1} = h0 or 0. Returns h [B, T, D] float64."""
    f = np.asarray(f, dtype=np.float64)
    i = np.asarray(i, dtype=np.float64)
    b, t, d = f.shape
    h = np.zeros((b, t, d), dtype=np.float64)
    prev = np.zeros((b, d)) if h0 is None else np.asarray(h0, dtype=np.float64).copy()
    for s in range(t):
        prev = f[:, s, :] * prev + i[:, s, :]
        h[:, s, :] = prev
    return h


# ----------------------------------------------------------------------------------------------
# backward: the gradients of a training step (straight-through estimator through the quantisers)
# ----------------------------------------------------------------------------------------------
def hgrn_scan_backward(f: np.ndarray, i: np.ndarray, dh: np.ndarray,
                       h0: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients through h_t = f_t h_{t-1} + i_t given dL/dh_t = dh_t for every step ([B, T, D]).

    The total gradient reaching h_t is G_t = dh_t + f_{t+1} G_{t+1} (nothing past the last step),
    taken backwards in time; then dL/di_t = G_t, dL/df_t = G_t h_{t-1} and dL/dh0 = f_0 G_0.
    Returns (df, di, dh0) in float64."""
    f = np.asarray(f, dtype=np.float64)
    dh = np.asarray(dh, dtype=np.float64)
    b, t, d = f.shape
    h = hgrn_scan(f, i, h0)
    first = np.zeros((b, d)) if h0 is None else np.asarray(h0, dtype=np.float64)
    hprev = np.concatenate([first[:, None, :], h[:, :-1, :]], axis=1)
    df = np.zeros((b, t, d))
    di = np.zeros((b, t, d))
    G = np.zeros((b, d))
    for s in reversed(range(t)):
        G = dh[:, s] + (f[:, s + 1] * G if s + 1 < t else 0.0)
        di[:, s] = G
        df[:, s] = G * hprev[:, s]
    dh0 = f[:, 0] * G if t else np.zeros((b, d))  # no step: the loss does not depend on h0
    return df, di, dh0


def hgrn_gates_backward(zf: np.ndarray, zi: np.ndarray, df: np.ndarray,
                        di: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Gradients through f = sigmoid(zf), i = SiLU(zi) (1 - f): with sigma' = f (1 - f) and
    SiLU'(z) = sigmoid(z) (1 + z (1 - sigmoid(z))),
    dzf = (df - di SiLU(zi)) f (1 - f) and dzi = di (1 - f) SiLU'(zi). Returns (dzf, dzi)."""
    zf = np.asarray(zf, dtype=np.float64)
    zi = np.asarray(zi, dtype=np.float64)
    f = sigmoid(zf)
    sz = sigmoid(zi)
    dzf = (np.asarray(df, dtype=np.float64) - np.asarray(di, dtype=np.float64) * silu(zi)) * f * (1.0 - f)
    dzi = np.asarray(di, dtype=np.float64) * (1.0 - f) * sz * (1.0 + zi * (1.0 - sz))
    return dzf, dzi


def rmsnorm_backward(x: np.ndarray, w: np.ndarray | None, dr: np.ndarray,
                     eps: float = EPS_NORM) -> tuple[np.ndarray, np.ndarray | None]:
    """Gradients through r = x rho w with rho = (mean(x^2) + eps)^(-1/2) over the last axis of n:
    with u = dr w, dx = rho u - rho^3 x mean(u x); dw = sum over rows of dr x rho (None without a
    gain). Returns (dx, dw)."""
    x = np.asarray(x, dtype=np.float64)
    dr = np.asarray(dr, dtype=np.float64)
    rho = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    u = dr * (np.asarray(w, dtype=np.float64) if w is not None else 1.0)
    dx = rho * u - rho ** 3 * x * np.mean(u * x, axis=-1, keepdims=True)
    dw = None if w is None else (dr * x * rho).reshape(-1, x.shape[-1]).sum(axis=0)
    return dx, dw


def bitlinear_backward(x: np.ndarray, norm_w: np.ndarray | None, W: np.ndarray, dy: np.ndarray,
                       eps: float = EPS_NORM) -> tuple[np.ndarray, np.ndarray | None, np.ndarray]:
    """Training gradients of FusedBitLinear with the latent float weight W [N, K], given dL/dy.

    The forward uses the dequantised operands rq = q (a/127) and Wq = t s (``act_quant`` and
    ``ternarize``); the straight-through estimator passes the gradient through both quantisers
    unchanged (nightvoyager.top, innovations table: weight_quant quantises in the forward pass
    and keeps the gradient in the backward pass; the activation quantiser is read the same way).
    So dL/dr = dy Wq, then the RMSNorm backward gives dx and the gain's gradient, and the latent
    weight receives dL/dW = dy^T rq. Returns (dx, dnorm_w, dW) in float64."""
    x = np.asarray(x, dtype=np.float64)
    k = x.shape[-1]
    x2 = x.reshape(-1, k)
    dy2 = np.asarray(dy, dtype=np.float64).reshape(x2.shape[0], -1)
    t, s_w = ternarize(W)
    Wq = t.astype(np.float64) * float(s_w)
    r = rmsnorm(x2, norm_w, eps)
    q, deq, _ = act_quant(r)
    rq = q.astype(np.float64) * deq[:, None]
    dr = dy2 @ Wq
    dx, dnw = rmsnorm_backward(x2, norm_w, dr, eps)
    dW = dy2.T @ rq
    return dx.reshape(x.shape), dnw, dW


# ----------------------------------------------------------------------------------------------
# HGRN2: the recurrence with state expansion
# ----------------------------------------------------------------------------------------------
def hgrn2_recurrence(q: np.ndarray, f: np.ndarray, i: np.ndarray,
                     S0: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Gated linear recurrence with an outer-product state, per head:

        S_t = diag(f_t) S_{t-1} + (1 - f_t)^T i_t      (S_t: dk x dv)
        o_t = q_t S_t                                 (o_t: dv)

    q, f [B, T, H, dk]; i [B, T, H, dv]; S0 [B, H, dk, dv] or None (zeros). Returns
    (o [B, T, H, dv], S_T [B, H, dk, dv]) in float64, stepping t in order.

    nightvoyager.top (MatMul-Free LLM report, innovations table and "if you study it" section)
    names HGRN2 and its module with fused-recurrent and chunked kernel forms, but prints no
    state-expansion equations. Reading: the published HGRN2 recurrence (Qin et al., 2024, "HGRN2:
    Gated Linear RNNs with State Expansion"): HGRN's element-wise forget gate becomes a per-row
    decay of a dk x dv state, the complement 1 - f of the forget gate the key, the input the value
    and the output gate the query. With dk = 1 and q = 1 it is the element-wise recurrence
    h_t = f_t h_{t-1} + (1 - f_t) i_t."""
    q = np.asarray(q, dtype=np.float64)
    f = np.asarray(f, dtype=np.float64)
    i = np.asarray(i, dtype=np.float64)
    b, t, h, dk = f.shape
    dv = i.shape[-1]
    S = np.zeros((b, h, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64).copy()
    o = np.zeros((b, t, h, dv))
    for s in range(t):
        key = 1.0 - f[:, s]                                   # [B, H, dk]
        S = f[:, s][..., :, None] * S + key[..., :, None] * i[:, s][..., None, :]
        o[:, s] = np.einsum("bhk,bhkv->bhv", q[:, s], S)
    return o, S


# ----------------------------------------------------------------------------------------------
# block, decode step and stack
# ----------------------------------------------------------------------------------------------
PROJS = ("i", "f", "g", "o", "gate", "down")


def quantize_block(params: dict[str, np.ndarray]) -> dict:
    """Ternarise every projection of a block: returns {'t_<p>', 's_<p>', 'nw_<p>', 'gnorm_w'}."""
    out: dict = {}
    for p in PROJS:
        t, s = ternarize(params[f"W_{p}"])
        out[f"t_{p}"] = t
        out[f"s_{p}"] = s
        out[f"nw_{p}"] = params[f"nw_{p}"]
    out["gnorm_w"] = params["gnorm_w"]
    return out


def block_forward(x: np.ndarray, qp: dict, h0: np.ndarray | None = None,
                  eps: float = EPS_NORM) -> tuple[np.ndarray, np.ndarray, dict]:
    """One HGRNBit block on x [B, T, d] (hysenlabs.com block structure):

    zi, zf, g = i_proj(x), f_proj(x), g_proj(x)      (three FusedBitLinear)
    f = sigmoid(zf); i = SiLU(zi) * (1 - f); h_t = f_t h_{t-1} + i_t
    u = RMSNorm(h) * gnorm_w * SiLU(g)                (g_norm, FusedRMSNormSwishGate)
    x1 = x + o_proj(u)
    [a | b] = gate_proj(x1); v = SiLU(a) * b         (GLU split, gate half first)
    y = x1 + down_proj(v)

    Returns (y [B,T,d], h_T [B,d], intermediates)."""
    x = np.asarray(x, dtype=np.float64)
    B, T, d = x.shape
    zi, _ = bitlinear(x, qp["nw_i"], qp["t_i"], qp["s_i"], eps)
    zf, _ = bitlinear(x, qp["nw_f"], qp["t_f"], qp["s_f"], eps)
    g, _ = bitlinear(x, qp["nw_g"], qp["t_g"], qp["s_g"], eps)
    f, i = hgrn_gates(zf, zi)
    h = hgrn_scan(f, i, h0)
    u = rmsnorm(h, qp["gnorm_w"], eps) * silu(g)
    o, _ = bitlinear(u, qp["nw_o"], qp["t_o"], qp["s_o"], eps)
    x1 = x + o
    gu, _ = bitlinear(x1, qp["nw_gate"], qp["t_gate"], qp["s_gate"], eps)
    inner = gu.shape[-1] // 2
    v = silu(gu[..., :inner]) * gu[..., inner:]
    dn, _ = bitlinear(v, qp["nw_down"], qp["t_down"], qp["s_down"], eps)
    y = x1 + dn
    inter = {"zi": zi, "zf": zf, "g": g, "f": f, "i": i, "h": h, "u": u, "x1": x1, "v": v}
    return y, h[:, -1, :].copy(), inter


def decode_step(x: np.ndarray, layers: list[dict], state: np.ndarray,
                eps: float = EPS_NORM) -> tuple[np.ndarray, np.ndarray]:
    """One autoregressive step through a stack: x [B, d] is the current token's hidden state,
    state [L, B, d] the carried recurrent state of every layer. Each layer runs the block of
    ``block_forward`` with T = 1, written out as its own single-step update
    h = f * h_prev + i. Returns (y [B, d], new state [L, B, d])."""
    x = np.asarray(x, dtype=np.float64)
    new_state = np.array(state, dtype=np.float64, copy=True)
    for l, qp in enumerate(layers):
        zi, _ = bitlinear(x, qp["nw_i"], qp["t_i"], qp["s_i"], eps)
        zf, _ = bitlinear(x, qp["nw_f"], qp["t_f"], qp["s_f"], eps)
        g, _ = bitlinear(x, qp["nw_g"], qp["t_g"], qp["s_g"], eps)
        f, i = hgrn_gates(zf, zi)
        h = f * new_state[l] + i
        new_state[l] = h
        u = rmsnorm(h, qp["gnorm_w"], eps) * silu(g)
        o, _ = bitlinear(u, qp["nw_o"], qp["t_o"], qp["s_o"], eps)
        x1 = x + o
        gu, _ = bitlinear(x1, qp["nw_gate"], qp["t_gate"], qp["s_gate"], eps)
        inner = gu.shape[-1] // 2
        v = silu(gu[..., :inner]) * gu[..., inner:]
        dn, _ = bitlinear(v, qp["nw_down"], qp["t_down"], qp["s_down"], eps)
        x = x1 + dn
    return x, new_state


def embed(ids: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Token embedding lookup: ids [...] -> rows of table [vocab, d]."""
    return np.asarray(table, dtype=np.float64)[np.asarray(ids, dtype=np.int64)]


def stack_forward(ids: np.ndarray, table: np.ndarray, layers: list[dict],
                  eps: float = EPS_NORM) -> tuple[np.ndarray, np.ndarray]:
    """Embedding gather then the L blocks in order (hysenlabs.com: HGRNBitModel is a stack of
    HGRNBitBlock). Returns (y [B,T,d], final states [L,B,d])."""
    x = embed(ids, table)
    states = []
    for qp in layers:
        x, hT, _ = block_forward(x, qp, None, eps)
        states.append(hT)
    return x, np.stack(states) if states else np.zeros((0,) + x.shape[::2])


# ----------------------------------------------------------------------------------------------
# language-model head and greedy generation
# ----------------------------------------------------------------------------------------------
def lm_head_logits(x: np.ndarray, norm_w: np.ndarray | None, table: np.ndarray,
                   eps: float = EPS_NORM) -> np.ndarray:
    """Logits of the tied language-model head: the final RMSNorm of the last block's output,
    then the product with the embedding table [vocab, d], which the input embedding and the
    head share (hysenlabs.com, install and model-table sections: 32000-word vocabulary, the
    causal-LM generation example). x [..., d] -> [..., vocab] float64."""
    r = rmsnorm(np.asarray(x, dtype=np.float64), norm_w, eps)
    return r @ np.asarray(table, dtype=np.float64).T


def greedy_next(logits: np.ndarray) -> np.ndarray:
    """Greedy decoding: the index of the largest logit of each row, the lowest index among
    equal maxima (argmax returns the first)."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int64)


# ----------------------------------------------------------------------------------------------
# model-size bookkeeping
# ----------------------------------------------------------------------------------------------
def block_param_count(d: int, inner: int) -> int:
    """Ternary parameters of one block: four d x d projections, gate_proj (2I x d), down_proj (d x I)."""
    return 4 * d * d + 2 * inner * d + d * inner


def model_param_count(d: int, inner: int, n_layers: int, vocab: int = 32000) -> int:
    """Blocks plus one (tied) embedding table; norm gains are negligible and excluded."""
    return n_layers * block_param_count(d, inner) + vocab * d


def bitlinear_ops(m: int, n: int, k: int) -> int:
    """Algorithmic integer operations of one BitLinear product: 2*M*N*K (a multiply-add is two)."""
    return 2 * m * n * k


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("np", "annotations")]
