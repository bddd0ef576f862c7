"""Stage-wise parity checks shared by the GPU tests.

Each stage of a kernel path is compared with the oracle's definition of that stage applied to the
kernel's own inputs to it (the debug taps), so every stage is checked element by element whatever
happened upstream: integer accumulations exactly, activation codes exactly except by one step where
the oracle's float32 value lies within a margin of a half-integer (both sides decide in float32,
so a code can flip only at such a near-tie), floats within the
stated tolerances (float32: 1e-3 relative + 1e-5 absolute; bfloat16: 2e-2 relative).
"""
import numpy as np
import torch

import oracle as O

RTOL32, ATOL32 = 1e-3, 1e-5
RTOL16 = 2e-2


def _near_tie(v, margin=1e-4):
    a = np.abs(v.astype(np.float64))
    return np.abs(a - np.floor(a) - 0.5) < margin



def _np(t):
    return t.float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float32) else t.cpu().numpy()


def _codes_match(q_gpu, v_oracle, q_oracle, margin):
    """Activation codes equal the oracle's except by one step where the oracle's float32 value
    lies within `margin` of a half-integer."""
    mism = q_gpu != q_oracle
    assert np.all(np.abs(q_gpu.astype(int) - q_oracle.astype(int)) <= 1)
    assert np.all(_near_tie(v_oracle, margin)[mism]), int(mism.sum())
    return mism


def _close(got, want, bf16):
    if bf16:
        np.testing.assert_allclose(got, want, rtol=RTOL16, atol=1e-6 * max(1.0, np.abs(want).max()))
    else:
        np.testing.assert_allclose(got, want, rtol=RTOL32, atol=ATOL32)


def check_block_stages(x, qp, taps, y_g, hl_g, h0, bf16, glu_fused=False):
    """Stage-wise parity: each stage of the kernel's block forward against the oracle's definition
    of that stage applied to the kernel's own inputs to it. Integer accumulations are exact; codes
    of the first quantisation match exactly, chained ones up to near-ties; floats elementwise."""
    m, d = x.shape[0] * x.shape[1], x.shape[2]
    B, T = x.shape[:2]
    x2 = x.reshape(m, d).astype(np.float64)
    q_ifg, deq_ifg = _np(taps["q_ifg"]), _np(taps["deq_ifg"])
    z = _np(taps["z"]).astype(np.float64)
    # 1. i/f/g input codes (first quantisation: exact) and 2. the three products z = [zi | zf | g]
    for j, p in enumerate(("i", "f", "g")):
        r = O.rmsnorm(x2, qp[f"nw_{p}"])
        qo, deqo, vo = O.act_quant(r)
        _codes_match(q_ifg[j], vo, qo, 1e-4)
        np.testing.assert_allclose(deq_ifg[j], deqo, rtol=1e-6)
        acc = O.int_matmul(q_ifg[j], qp[f"t_{p}"])
        _close(z[:, j * d:(j + 1) * d], acc * deq_ifg[j].astype(np.float64)[:, None] * float(qp[f"s_{p}"]), bf16)
    # 3. gates and scan on the kernel's pre-activations
    zi, zf, g = z[:, :d], z[:, d:2 * d], z[:, 2 * d:]
    f, i = O.hgrn_gates(zf.reshape(B, T, d), zi.reshape(B, T, d))
    h_ref = O.hgrn_scan(f, i, h0)
    h = _np(taps["h"]).astype(np.float64)
    _close(h, h_ref.reshape(m, d), bf16)
    np.testing.assert_allclose(hl_g, h_ref[:, -1], rtol=1e-3 if not bf16 else RTOL16, atol=1e-5)
    # 4. g_norm + o_proj codes, 5. o_proj + residual
    u = O.rmsnorm(h, qp["gnorm_w"]) * O.silu(g)
    qo, _, vo = O.act_quant(O.rmsnorm(u, qp["nw_o"]))
    q_o = _np(taps["q_o"])
    _codes_match(q_o, vo, qo, 1e-3)
    x1_ref = x2 + O.int_matmul(q_o, qp["t_o"]) * _np(taps["deq_o"]).astype(np.float64)[:, None] * float(qp["s_o"])
    x1 = _np(taps["x1"]).astype(np.float64)
    _close(x1, x1_ref, bf16)
    # 6. gate_proj codes and product
    qg, _, vg = O.act_quant(O.rmsnorm(x1, qp["nw_gate"]))
    q_gate = _np(taps["q_gate"])
    _codes_match(q_gate, vg, qg, 1e-3)
    gu_ref = O.int_matmul(q_gate, qp["t_gate"]) * _np(taps["deq_gate"]).astype(np.float64)[:, None] * float(qp["s_gate"])
    inner = gu_ref.shape[1] // 2
    # 7. GLU: v = SiLU(gate) * up, formed by gate_proj's epilogue or from the stored halves
    if glu_fused:
        v = _np(taps["v"]).astype(np.float64)
        _close(v, O.silu(gu_ref[:, :inner]) * gu_ref[:, inner:], bf16)
    else:
        gu = _np(taps["gu"]).astype(np.float64)
        _close(gu, gu_ref, bf16)
        v = O.silu(gu[:, :inner]) * gu[:, inner:]
    #    + down_proj codes, 8. down_proj + residual
    qd, _, vd = O.act_quant(O.rmsnorm(v, qp["nw_down"]))
    q_down = _np(taps["q_down"])
    _codes_match(q_down, vd, qd, 1e-3)
    y_ref = x1 + O.int_matmul(q_down, qp["t_down"]) * _np(taps["deq_down"]).astype(np.float64)[:, None] * float(qp["s_down"])
    _close(y_g.reshape(m, d), y_ref, bf16)


def chain_clean_rows(kernel_groups, oracle_groups, B, T, scan_groups, margins):
    """Follows every chained code decision of the forward in order and returns the rows that saw no
    code differing from the oracle's own chain, asserting that in every other row the FIRST
    difference sits at a near-tie of the oracle's float32 value (both sides decide in
    float32, so only a value within rounding of a half-integer can round the other way; after it,
    the row's later inputs differ and its later codes may differ anywhere).

    kernel_groups / oracle_groups: one entry per decision point in chain order, each a list of
    (codes [B*T, k]) / (codes, float32 value that was rounded) for the quantisations taken there
    together (i, f, g share one input). scan_groups: indices of the groups whose products enter the
    recurrence, which carries a difference at step t to every later step of that sequence.
    Returns a bool mask [B*T] of clean rows."""
    dirty = np.zeros((B, T), bool)
    for gi, (gk, go) in enumerate(zip(kernel_groups, oracle_groups)):
        hit = np.zeros(B * T, bool)
        for qg, (qo, vo) in zip(gk, go):
            mm = qg != qo
            rows = mm.any(axis=1)
            fresh = rows & ~dirty.reshape(-1)
            if fresh.any():
                d = np.abs(qg[fresh].astype(int) - qo[fresh].astype(int))[mm[fresh]]
                assert np.all(d <= 1), int(d.max())
                assert np.all(_near_tie(vo[fresh], margins[gi])[mm[fresh]]), (gi, int(mm[fresh].sum()))
            hit |= rows
        dirty |= hit.reshape(B, T)
        if gi in scan_groups:
            dirty = np.maximum.accumulate(dirty, axis=1)
    return ~dirty.reshape(-1)


def oracle_chain_groups(x, qp, inter):
    """The oracle's own code decisions of one block (x [m, d], its intermediates flattened to rows):
    groups [i, f, g], [o], [gate], [down] of (codes, value rounded)."""
    def aq(v, nw):
        q, _, val = O.act_quant(O.rmsnorm(v, nw))
        return q, val
    d = x.shape[-1]
    x2 = x.reshape(-1, d)
    return [[aq(x2, qp[f"nw_{p}"]) for p in ("i", "f", "g")],
            [aq(inter["u"].reshape(-1, d), qp["nw_o"])],
            [aq(inter["x1"].reshape(-1, d), qp["nw_gate"])],
            [aq(inter["v"].reshape(x2.shape[0], -1), qp["nw_down"])]]


def kernel_chain_groups(taps):
    """The kernel's code decisions of one block from its taps, in the order of oracle_chain_groups."""
    q_ifg = _np(taps["q_ifg"])
    return [[q_ifg[0], q_ifg[1], q_ifg[2]], [_np(taps["q_o"])], [_np(taps["q_gate"])], [_np(taps["q_down"])]]


def check_block_end_to_end(y_g, y_ref, inter, qp, bf16, taps=None, x=None, layers=1):
    """Against the oracle's own forward. float32, with the kernel's codes (`taps`) and the input
    `x`: every row whose chain of code decisions matches the oracle's is equal elementwise within
    1e-3 / 1e-5, and every other row's first differing code is a near-tie (chain_clean_rows). The
    relative L2 error of the whole output is returned and held to a sanity bound only: once a code
    flips at a near-tie, the later quantisations of that row see different inputs and flip in
    numbers (about 5e-4 relative per flipped code at K = 2560), so the whole-output norm is not a
    tolerance (it is 1e-3 .. 1e-2 for one or two float32 layers at the model widths, a few 1e-2 in
    bf16, where every stored intermediate is rounded to 8 bits and the oracle rounds none)."""
    rel = np.linalg.norm(y_g - y_ref) / np.linalg.norm(y_ref)
    assert rel < 5e-2 * np.sqrt(layers), rel
    if bf16 or taps is None:
        return rel, None
    B, T, d = x.shape
    clean = chain_clean_rows(kernel_chain_groups(taps), oracle_chain_groups(x.astype(np.float64), qp, inter),
                             B, T, scan_groups={0}, margins=[1e-4, 1e-3, 1e-3, 1e-3])
    yg, yr = y_g.reshape(B * T, d), y_ref.reshape(B * T, d)
    np.testing.assert_allclose(yg[clean], yr[clean], rtol=RTOL32, atol=ATOL32)
    return rel, clean


def check_chain_end_to_end(x, qps, kernel_taps, y_g, states_g=None, h0s=None):
    """Float32 end to end over a chain of blocks (a stack, or a decode step with T = 1): the oracle's
    own chain through the same layers, then chain_clean_rows over every code decision of every
    layer (the kernel's codes from its per-layer taps). Clean rows: the output and each layer's
    final state equal the oracle's elementwise within 1e-3 / 1e-5. Returns (relative L2 error of
    the output, fraction of clean rows)."""
    B, T, d = x.shape
    x_cur = np.asarray(x, dtype=np.float64)
    kg, og, scans, margins, states = [], [], set(), [], []
    for l, qp in enumerate(qps):
        y, hT, inter = O.block_forward(x_cur, qp, None if h0s is None else h0s[l])
        scans.add(len(og))
        og += oracle_chain_groups(x_cur, qp, inter)
        kg += kernel_chain_groups(kernel_taps[l])
        margins += [1e-4 if l == 0 else 1e-3, 1e-3, 1e-3, 1e-3]
        states.append(hT)
        x_cur = y
    y_ref = x_cur.reshape(B * T, d)
    yg = np.asarray(y_g, dtype=np.float64).reshape(B * T, d)
    rel = np.linalg.norm(yg - y_ref) / np.linalg.norm(y_ref)
    assert rel < 5e-2 * np.sqrt(len(qps)), rel
    clean = chain_clean_rows(kg, og, B, T, scans, margins)
    np.testing.assert_allclose(yg[clean], y_ref[clean], rtol=RTOL32, atol=ATOL32)
    if states_g is not None:
        # a layer's final state depends on the last step of each sequence
        last = clean.reshape(B, T)[:, -1]
        for l in range(len(qps)):
            np.testing.assert_allclose(np.asarray(states_g[l])[last], states[l][last], rtol=RTOL32, atol=ATOL32)
    return rel, float(clean.mean())


def check_decode_layer(x_in, state_in, state_out, qp, tp, bf16, z_rounded):
    """Stage-wise parity of one layer of a decode step from its taps (mmf_decode_taps): x_in [b, d]
    and state_in [b, d] the layer's inputs as the kernels saw them, state_out the state it left.
    `z_rounded`: z and h were stored in bf16 between kernels (the block path in bf16), so they are
    compared at bf16 tolerance. Returns the layer output y [b, d] (float64)."""
    b, d = x_in.shape
    x2 = np.asarray(x_in, dtype=np.float64)
    q_ifg, deq_ifg = _np(tp["q_ifg"]), _np(tp["deq_ifg"])
    z = _np(tp["z"]).astype(np.float64)
    # 1. i/f/g input codes (first quantisation of the layer's input: exact up to near-ties) and
    # 2. the three products from the kernel's own codes
    for j, p in enumerate(("i", "f", "g")):
        qo, deqo, vo = O.act_quant(O.rmsnorm(x2, qp[f"nw_{p}"]))
        _codes_match(q_ifg[j], vo, qo, 1e-4)
        np.testing.assert_allclose(deq_ifg[j], deqo, rtol=1e-6)
        acc = O.int_matmul(q_ifg[j], qp[f"t_{p}"])
        _close(z[:, j * d:(j + 1) * d], acc * deq_ifg[j].astype(np.float64)[:, None] * float(qp[f"s_{p}"]), z_rounded)
    # 3. gates and one recurrence step on the kernel's pre-activations and carried state
    zi, zf, g = z[:, :d], z[:, d:2 * d], z[:, 2 * d:]
    f, i = O.hgrn_gates(zf, zi)
    h_ref = f * np.asarray(state_in, dtype=np.float64) + i
    np.testing.assert_allclose(np.asarray(state_out, dtype=np.float64), h_ref, rtol=RTOL32, atol=ATOL32)
    h = _np(tp["h"]).astype(np.float64)
    _close(h, h_ref, z_rounded)
    # 4. g_norm + o_proj codes, 5. o_proj + residual
    u = O.rmsnorm(h, qp["gnorm_w"]) * O.silu(g)
    qo, _, vo = O.act_quant(O.rmsnorm(u, qp["nw_o"]))
    q_o = _np(tp["q_o"])
    _codes_match(q_o, vo, qo, 1e-3)
    x1_ref = x2 + O.int_matmul(q_o, qp["t_o"]) * _np(tp["deq_o"]).astype(np.float64)[:, None] * float(qp["s_o"])
    x1 = _np(tp["x1"]).astype(np.float64)
    _close(x1, x1_ref, bf16)
    # 6. gate_proj codes and product, 7. GLU
    qg, _, vg = O.act_quant(O.rmsnorm(x1, qp["nw_gate"]))
    q_gate = _np(tp["q_gate"])
    _codes_match(q_gate, vg, qg, 1e-3)
    gu_ref = O.int_matmul(q_gate, qp["t_gate"]) * _np(tp["deq_gate"]).astype(np.float64)[:, None] * float(qp["s_gate"])
    inner = gu_ref.shape[1] // 2
    v = _np(tp["v"]).astype(np.float64)
    if np.isnan(v).all():   # the step stored [gate | up] and formed v in down_proj's norm
        gu = _np(tp["gu"]).astype(np.float64)
        _close(gu, gu_ref, bf16)
        v = O.silu(gu[:, :inner]) * gu[:, inner:]
    else:
        _close(v, O.silu(gu_ref[:, :inner]) * gu_ref[:, inner:], bf16)
    # 8. down_proj codes, down_proj + residual
    qd, _, vd = O.act_quant(O.rmsnorm(v, qp["nw_down"]))
    q_down = _np(tp["q_down"])
    _codes_match(q_down, vd, qd, 1e-3)
    y_ref = x1 + O.int_matmul(q_down, qp["t_down"]) * _np(tp["deq_down"]).astype(np.float64)[:, None] * float(qp["s_down"])
    y = _np(tp["y"]).astype(np.float64)
    _close(y, y_ref, bf16)
    return y
