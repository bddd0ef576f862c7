"""The oracle's pins catch plausible mistakes: each test here plants one mistake in a copy of an
oracle function (on the CPU, in this process only), runs the pins of that function against the
planted copy, and requires that they fail. A pin set that passed a planted mistake would not be
pinning the function."""
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
