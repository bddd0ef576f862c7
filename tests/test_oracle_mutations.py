"""The oracle's pins catch plausible mistakes: each test here plants one mistake in a copy of an
oracle function (on the CPU, in this process only), runs the pins against the planted copy, and
requires that they fail -- for HGRN2, the backward functions and every function of the forward
(recurrence, gates, RMSNorm, both quantisers, BitLinear, the block's wiring, the packed layout and
the head). A pin set that passed a planted mistake would not be pinning the function."""
import numpy as np
import pytest

import oracle as O
import test_oracle_pins as P


def _failures(pins):
    """How many of the pins (callables) raise an AssertionError, or fail with a shape error."""
    n = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            n += 1
    return n


# ---------------------------------------------------------------------------------------------
# HGRN2 recurrence
# ---------------------------------------------------------------------------------------------
def _hgrn2_mutant(kind):
    def run(q, f, i, S0=None):
        q = np.asarray(q, dtype=np.float64)
        f = np.asarray(f, dtype=np.float64)
        i = np.asarray(i, dtype=np.float64)
        b, t, h, dk = f.shape
        dv = i.shape[-1]
        S = np.zeros((b, h, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64).copy()
        o = np.zeros((b, t, h, dv))
        for s in range(t):
            key = f[:, s] if kind == "key_is_f" else 1.0 - f[:, s]
            new = key[..., :, None] * i[:, s][..., None, :]
            if kind == "decay_after_add":
                S_next = f[:, s][..., :, None] * (S + new)
            else:
                S_next = f[:, s][..., :, None] * S + new
            qs = np.ones_like(q[:, s]) if kind == "no_query" else q[:, s]
            read = S if kind == "read_before_update" else S_next
            o[:, s] = np.einsum("bhk,bhkv->bhv", qs, read)
            S = S_next
        return o, S
    return run


def _hgrn2_pins():
    cases = P._golden("hgrn2_recurrence_handworked.json")["cases"]
    pins = [lambda c=c: P.test_hgrn2_handworked(c) for c in cases]
    pins += [P.test_hgrn2_one_key_dimension_is_the_elementwise_recurrence, P.test_hgrn2_bruteforce_attention_form,
             P.test_hgrn2_zero_forget_closed_form, P.test_hgrn2_state_passing_and_causality,
             P.test_hgrn2_chunked_form_matches_recurrence]
    return pins


def test_hgrn2_pins_pass_on_the_oracle():
    assert _failures(_hgrn2_pins()) == 0


@pytest.mark.parametrize("kind", ["key_is_f", "read_before_update", "decay_after_add", "no_query"])
def test_hgrn2_pins_catch_planted_mistakes(monkeypatch, kind):
    monkeypatch.setattr(O, "hgrn2_recurrence", _hgrn2_mutant(kind))
    pins = _hgrn2_pins()
    failed = _failures(pins)
    assert failed >= 3, f"{kind}: only {failed} of {len(pins)} pins fail"


# ---------------------------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------------------------
def _scan_backward_mutant(kind):
    def run(f, i, dh, h0=None):
        f = np.asarray(f, dtype=np.float64)
        dh = np.asarray(dh, dtype=np.float64)
        b, t, d = f.shape
        h = O.hgrn_scan(f, i, h0)
        first = np.zeros((b, d)) if h0 is None else np.asarray(h0, dtype=np.float64)
        hprev = np.concatenate([first[:, None, :], h[:, :-1, :]], axis=1)
        df, di, G = np.zeros((b, t, d)), np.zeros((b, t, d)), np.zeros((b, d))
        for s in reversed(range(t)):
            if kind == "carry_own_gate":
                G = dh[:, s] + f[:, s] * G
            else:
                G = dh[:, s] + (f[:, s + 1] * G if s + 1 < t else 0.0)
            di[:, s] = G
            df[:, s] = G * (h[:, s] if kind == "h_not_hprev" else hprev[:, s])
        if t == 0:
            return df, di, np.zeros((b, d))
        return df, di, (G if kind == "dh0_without_gate" else f[:, 0] * G)
    return run


def _gates_backward_mutant(zf, zi, df, di):
    f = O.sigmoid(np.asarray(zf, dtype=np.float64))
    sz = O.sigmoid(np.asarray(zi, dtype=np.float64))
    dzf = (df - di * O.silu(zi)) * f * (1.0 - f)
    dzi = di * (1.0 - f) * sz                          # SiLU' taken as sigmoid alone
    return dzf, dzi


def _rmsnorm_backward_mutant(x, w, dr, eps=O.EPS_NORM):
    x = np.asarray(x, dtype=np.float64)
    rho = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    u = np.asarray(dr, dtype=np.float64) * (np.asarray(w) if w is not None else 1.0)
    dx = rho * u                                        # the term through rho dropped
    dw = None if w is None else (dr * x * rho).reshape(-1, x.shape[-1]).sum(axis=0)
    return dx, dw


def _bitlinear_backward_mutant(kind):
    def run(x, norm_w, W, dy, eps=O.EPS_NORM):
        x2 = np.asarray(x, dtype=np.float64).reshape(-1, np.shape(x)[-1])
        dy2 = np.asarray(dy, dtype=np.float64).reshape(x2.shape[0], -1)
        t, s_w = O.ternarize(W)
        Wq = np.asarray(W, dtype=np.float64) if kind == "latent_weights" else t * float(s_w)
        r = O.rmsnorm(x2, norm_w, eps)
        q, deq, _ = O.act_quant(r)
        rq = r if kind == "unquantised_activations" else q * deq[:, None]
        dx, dnw = O.rmsnorm_backward(x2, norm_w, dy2 @ Wq, eps)
        dW = dy2.T @ rq
        if kind == "rows_reversed":
            dW = dW[::-1]
        return dx.reshape(np.shape(x)), dnw, dW
    return run


BACKWARD_PINS = [P.test_scan_backward_finite_differences, P.test_gates_backward_finite_differences,
                 P.test_rmsnorm_backward_finite_differences, P.test_bitlinear_backward_is_straight_through]


def test_backward_pins_pass_on_the_oracle():
    assert _failures(BACKWARD_PINS) == 0


@pytest.mark.parametrize("name,mutant", [
    ("hgrn_scan_backward", _scan_backward_mutant("h_not_hprev")),
    ("hgrn_scan_backward", _scan_backward_mutant("carry_own_gate")),
    ("hgrn_scan_backward", _scan_backward_mutant("dh0_without_gate")),
    ("hgrn_gates_backward", _gates_backward_mutant),
    ("rmsnorm_backward", _rmsnorm_backward_mutant),
    ("bitlinear_backward", _bitlinear_backward_mutant("latent_weights")),
    ("bitlinear_backward", _bitlinear_backward_mutant("unquantised_activations")),
    ("bitlinear_backward", _bitlinear_backward_mutant("rows_reversed")),
], ids=["scan:h_t", "scan:carry_gate", "scan:dh0_gate", "gates:silu_prime", "rmsnorm:rho_term",
        "bitlinear:latent_W", "bitlinear:unquantised_r", "bitlinear:dW_rows"])
def test_backward_pins_catch_planted_mistakes(monkeypatch, name, mutant):
    monkeypatch.setattr(O, name, mutant)
    assert _failures(BACKWARD_PINS) >= 1


# ---------------------------------------------------------------------------------------------
# the forward: every oracle function the block uses, each with plausible mistakes planted in the
# package and in the module (so the oracle's internal calls see the planted copy too); the whole
# pin set runs against each and at least one pin must fail
# ---------------------------------------------------------------------------------------------
def _expand(fn):
    marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
    if not marks:
        return [fn]
    names = [n.strip() for n in marks[0].args[0].split(",")]
    out = []
    for vals in marks[0].args[1]:
        vals = vals if len(names) > 1 else (vals,)
        out.append(lambda fn=fn, kw=dict(zip(names, vals)): fn(**kw))
    return out


ALL_PINS = [p for name in sorted(dir(P)) if name.startswith("test_") for p in _expand(getattr(P, name))]


def _plant(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    monkeypatch.setattr(O.mmf_oracle, name, fn)


def _scan_mutant(kind):
    def run(f, i, h0=None):
        f = np.asarray(f, dtype=np.float64)
        i = np.asarray(i, dtype=np.float64)
        b, t, d = f.shape
        h = np.zeros((b, t, d))
        prev = np.zeros((b, d)) if (h0 is None or kind == "h0_ignored") else np.asarray(h0, dtype=np.float64).copy()
        for s in range(t):
            if kind == "previous_input":
                prev = f[:, s] * prev + (i[:, s - 1] if s else 0.0)
            elif kind == "input_decayed":
                prev = f[:, s] * (prev + i[:, s])
            else:
                prev = f[:, s] * prev + i[:, s]
            h[:, s] = prev
        return h
    return run


def _gates_mutant(kind):
    def run(zf, zi):
        f = O.sigmoid(-np.asarray(zf) if kind == "sign" else zf)
        if kind == "complement_dropped":
            return f, O.silu(zi)
        if kind == "forget_as_input_gate":
            return f, O.silu(zi) * f
        return f, O.silu(zi) * (1.0 - f)
    return run


def _rmsnorm_mutant(kind):
    def run(x, w, eps=O.EPS_NORM):
        x = np.asarray(x, dtype=np.float64)
        ms = np.sum(x * x, axis=-1, keepdims=True) if kind == "sum_not_mean" else np.mean(x * x, axis=-1, keepdims=True)
        r = x / (np.sqrt(ms) + eps) if kind == "eps_outside" else x / np.sqrt(ms + eps)
        if w is not None and kind != "gain_ignored":
            r = r * np.asarray(w, dtype=np.float64)
        return r
    return run


def _ternarize_mutant(kind):
    def run(W):
        W32 = np.asarray(W, dtype=np.float32)
        if kind == "absmax_scale":
            s = np.float32(max(float(np.max(np.abs(W32))) if W32.size else 0.0, O.EPS_QUANT))
        else:
            s = O.weight_scale(W32)
        v = W32 / s
        t = np.trunc(v) if kind == "truncate" else np.rint(v)
        return np.clip(t, -1, 1).astype(np.int8), s
    return run


def _act_quant_mutant(kind):
    def run(r):
        r32 = np.asarray(r, dtype=np.float64).astype(np.float32)
        red = np.mean if kind == "absmean" else np.max
        a = red(np.abs(r32), axis=-1, keepdims=True) if r32.shape[-1] else np.zeros(r32.shape[:-1] + (1,), np.float32)
        a = np.maximum(a, np.float32(O.EPS_QUANT)).astype(np.float32)
        v = (r32 * (np.float32(127.0) / a).astype(np.float32)).astype(np.float32)
        q = np.clip(np.rint(v), -127, 127).astype(np.int8)
        deq = a[..., 0].astype(np.float64) / (128.0 if kind == "deq_128" else 127.0)
        return q, deq, v
    return run


def _bitlinear_mutant(kind):
    def run(x, norm_w, t, s_w, eps=O.EPS_NORM):
        x = np.asarray(x, dtype=np.float64)
        lead, k = x.shape[:-1], x.shape[-1]
        x2 = x.reshape(-1, k)
        r = O.rmsnorm(x2, norm_w, eps)
        q, deq, v = O.act_quant(r)
        acc = O.int_matmul(q, t)
        y = acc.astype(np.float64) * (1.0 if kind == "no_deq" else deq[:, None]) * (1.0 if kind == "no_scale" else float(s_w))
        if kind == "norm_skipped":
            q2, deq2, _ = O.act_quant(x2)
            y = O.int_matmul(q2, t) * deq2[:, None] * float(s_w)
            q, deq, acc = q2, deq2, O.int_matmul(q2, t)
        return y.reshape(lead + (t.shape[0],)), {"r": r, "q": q, "deq": deq, "v": v, "acc": acc}
    return run


def _block_mutant(kind):
    def run(x, qp, h0=None, eps=O.EPS_NORM):
        x = np.asarray(x, dtype=np.float64)
        zi, _ = O.bitlinear(x, qp["nw_i"], qp["t_i"], qp["s_i"], eps)
        zf, _ = O.bitlinear(x, qp["nw_f"], qp["t_f"], qp["s_f"], eps)
        g, _ = O.bitlinear(x, qp["nw_g"], qp["t_g"], qp["s_g"], eps)
        f, i = O.hgrn_gates(zf, zi)
        h = O.hgrn_scan(f, i, h0)
        u = O.rmsnorm(h, qp["gnorm_w"], eps) * (g if kind == "gate_without_silu" else O.silu(g))
        o, _ = O.bitlinear(u, qp["nw_o"], qp["t_o"], qp["s_o"], eps)
        x1 = o if kind == "no_first_residual" else x + o
        gu, _ = O.bitlinear(x1, qp["nw_gate"], qp["t_gate"], qp["s_gate"], eps)
        inner = gu.shape[-1] // 2
        a, b = gu[..., :inner], gu[..., inner:]
        v = O.silu(b) * a if kind == "glu_halves_swapped" else O.silu(a) * b
        dn, _ = O.bitlinear(v, qp["nw_down"], qp["t_down"], qp["s_down"], eps)
        y = x1 + dn
        inter = {"zi": zi, "zf": zf, "g": g, "f": f, "i": i, "h": h, "u": u, "x1": x1, "v": v}
        return y, h[:, -1, :].copy(), inter
    return run


def _code_bit_mutant(j):
    return 2 * j                                   # plain sequential fields, not the quad layout


def _lm_head_mutant(x, norm_w, table, eps=O.EPS_NORM):
    return np.asarray(x, dtype=np.float64) @ np.asarray(table, dtype=np.float64).T   # final norm dropped


_REAL_DECODE = O.decode_step


def _decode_mutant(x, layers, state, eps=O.EPS_NORM):
    # the carried state is not read: every step starts from h_prev = 0
    return _REAL_DECODE(x, layers, np.zeros_like(np.asarray(state, dtype=np.float64)), eps)


def _count_mutant(words, k):
    # a 10 field in a padding column counted twice (once as 10, once as nonzero padding)
    words = np.asarray(words, dtype=np.uint64)
    bad = 0
    for col in range(16 * words.shape[1]):
        w, j = divmod(col, 16)
        f = (words[:, w] >> np.uint64(O.code_bit(j))) & np.uint64(3)
        bad += int(np.count_nonzero(f == 2))
        if col >= k:
            bad += int(np.count_nonzero(f != 0))
    return bad


def _greedy_mutant(logits):
    lg = np.asarray(logits)
    return (lg.shape[-1] - 1 - np.argmax(lg[..., ::-1], axis=-1)).astype(np.int64)   # last index on ties


def _embed_mutant(ids, table):
    t = np.asarray(table, dtype=np.float64)
    return t[(np.asarray(ids, dtype=np.int64) + 1) % t.shape[0]]                    # off by one row


FORWARD_MUTANTS = [
    ("hgrn_scan", _scan_mutant("previous_input"), "scan:i_{t-1}"),
    ("hgrn_scan", _scan_mutant("input_decayed"), "scan:f(h+i)"),
    ("hgrn_scan", _scan_mutant("h0_ignored"), "scan:h0"),
    ("hgrn_gates", _gates_mutant("sign"), "gates:sign"),
    ("hgrn_gates", _gates_mutant("complement_dropped"), "gates:no_1-f"),
    ("hgrn_gates", _gates_mutant("forget_as_input_gate"), "gates:f_for_1-f"),
    ("rmsnorm", _rmsnorm_mutant("sum_not_mean"), "rmsnorm:sum"),
    ("rmsnorm", _rmsnorm_mutant("eps_outside"), "rmsnorm:eps"),
    ("rmsnorm", _rmsnorm_mutant("gain_ignored"), "rmsnorm:gain"),
    ("ternarize", _ternarize_mutant("absmax_scale"), "ternarize:absmax"),
    ("ternarize", _ternarize_mutant("truncate"), "ternarize:trunc"),
    ("act_quant", _act_quant_mutant("absmean"), "act_quant:absmean"),
    ("act_quant", _act_quant_mutant("deq_128"), "act_quant:deq/128"),
    ("bitlinear", _bitlinear_mutant("no_deq"), "bitlinear:no_a/127"),
    ("bitlinear", _bitlinear_mutant("no_scale"), "bitlinear:no_s"),
    ("bitlinear", _bitlinear_mutant("norm_skipped"), "bitlinear:no_norm"),
    ("block_forward", _block_mutant("gate_without_silu"), "block:g_no_silu"),
    ("block_forward", _block_mutant("no_first_residual"), "block:no_residual"),
    ("block_forward", _block_mutant("glu_halves_swapped"), "block:glu_swapped"),
    ("code_bit", _code_bit_mutant, "pack:code_bit"),
    ("lm_head_logits", _lm_head_mutant, "head:no_norm"),
    ("decode_step", _decode_mutant, "decode:state_dropped"),
    ("count_malformed_fields", _count_mutant, "integrity:double_count"),
    ("greedy_next", _greedy_mutant, "greedy:last_on_ties"),
    ("embed", _embed_mutant, "embed:off_by_one"),
]


def test_all_pins_pass_on_the_oracle():
    assert len(ALL_PINS) >= 40
    assert _failures(ALL_PINS) == 0


@pytest.mark.parametrize("name,mutant", [(n, m) for n, m, _ in FORWARD_MUTANTS], ids=[i for _, _, i in FORWARD_MUTANTS])
def test_forward_pins_catch_planted_mistakes(monkeypatch, name, mutant):
    _plant(monkeypatch, name, mutant)
    assert _failures(ALL_PINS) >= 1
