"""Pins for the CPU oracle: checks that tie it to the mathematics and to what the MatMul-free LM
pages fix, not to itself. Every check here is computed a different way from the oracle function
it pins (hand-worked values, closed forms, brute force, invariants), so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


# ---------------------------------------------------------------------------------------------
# recurrence
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("case", _golden("hgrn_scan_handworked.json")["cases"], ids=lambda c: c["name"])
def test_scan_handworked(case):
    f = np.array(case["f"])[None, :, None]
    i = np.array(case["i"])[None, :, None]
    h0 = np.array([[case["h0"]]])
    h = O.hgrn_scan(f, i, h0)[0, :, 0]
    assert np.array_equal(h, np.array(case["h"]))


def test_scan_closed_form_constant_gates():
    # constant zf, zi: h_t = SiLU(zi) * (1 - f^t) for t = 1, 2, ... with f = sigmoid(zf)
    zf, zi, T = 1.3, -0.7, 60
    f_const = 1.0 / (1.0 + math.exp(-zf))
    silu_zi = zi / (1.0 + math.exp(-zi))
    f, i = O.hgrn_gates(np.full((1, T, 1), zf), np.full((1, T, 1), zi))
    h = O.hgrn_scan(f, i)[0, :, 0]
    want = np.array([silu_zi * (1.0 - f_const ** t) for t in range(1, T + 1)])
    np.testing.assert_allclose(h, want, rtol=1e-12, atol=1e-14)


def test_scan_long_sequence_converges_to_fixed_point():
    # f = sigmoid(4) (long memory): after many steps h tends to SiLU(zi) with no drift
    T = 4096
    f, i = O.hgrn_gates(np.full((1, T, 1), 4.0), np.full((1, T, 1), 0.5))
    h = O.hgrn_scan(f, i)[0, :, 0]
    assert abs(h[-1] - 0.5 / (1.0 + math.exp(-0.5))) < 1e-12


def test_scan_bruteforce_sum_of_products():
    # h_t = sum_s (prod_{r=s+1..t} f_r) i_s + (prod_{r=0..t} f_r) h0, double loop
    g = np.random.default_rng(3)
    B, T, D = 2, 7, 3
    f = g.uniform(0, 1, (B, T, D))
    i = g.standard_normal((B, T, D))
    h0 = g.standard_normal((B, D))
    want = np.zeros((B, T, D))
    for b in range(B):
        for d in range(D):
            for t in range(T):
                acc = h0[b, d]
                for r in range(0, t + 1):
                    acc *= f[b, r, d]
                for s in range(t + 1):
                    p = i[b, s, d]
                    for r in range(s + 1, t + 1):
                        p *= f[b, r, d]
                    acc += p
                want[b, t, d] = acc
    np.testing.assert_allclose(O.hgrn_scan(f, i, h0), want, rtol=1e-12, atol=1e-12)


def test_scan_chunked_composition_matches_sequential():
    # the step h -> f h + i is affine; composing chunk maps (A, b) then applying them to the
    # carry gives the sequential result (associativity of (a,b) o (a',b') = (a a', a' b + b'))
    g = np.random.default_rng(4)
    B, T, D, C = 1, 64, 5, 16
    f = g.uniform(0.5, 1.0, (B, T, D))
    i = g.standard_normal((B, T, D))
    carry = np.zeros((B, D))
    out = np.zeros((B, T, D))
    for c0 in range(0, T, C):
        A = np.ones((B, D))
        b = np.zeros((B, D))
        for t in range(c0, c0 + C):
            A, b = f[:, t] * A, f[:, t] * b + i[:, t]
            out[:, t] = A * carry + b
        carry = A * carry + b
    np.testing.assert_allclose(O.hgrn_scan(f, i), out, rtol=1e-12, atol=1e-12)


def test_scan_causality():
    g = np.random.default_rng(5)
    f = g.uniform(0, 1, (1, 20, 4))
    i = g.standard_normal((1, 20, 4))
    h = O.hgrn_scan(f, i)
    i2 = i.copy()
    i2[0, 11, 2] += 1.0
    h2 = O.hgrn_scan(f, i2)
    assert np.array_equal(h[:, :11], h2[:, :11])
    assert h2[0, 11, 2] != h[0, 11, 2]


def test_gate_definitions():
    z = np.array([-30.0, -2.0, 0.0, 1.5, 30.0])
    np.testing.assert_allclose(O.sigmoid(z), [1 / (1 + math.exp(-v)) for v in z], rtol=1e-15)
    np.testing.assert_allclose(O.silu(z), [v / (1 + math.exp(-v)) for v in z], rtol=1e-15)
    assert O.sigmoid(np.array(0.0)) == 0.5 and O.silu(np.array(0.0)) == 0.0
    f, i = O.hgrn_gates(np.array([0.0]), np.array([2.0]))
    # f = 1/2, i = SiLU(2) * (1 - 1/2)
    assert f[0] == 0.5 and abs(i[0] - 0.5 * 2.0 / (1 + math.exp(-2.0))) < 1e-15


# ---------------------------------------------------------------------------------------------
# RMSNorm and quantisers
# ---------------------------------------------------------------------------------------------
def test_rmsnorm_closed_forms():
    c, eps = 0.37, 1e-8
    w = np.array([2.0, -1.0, 0.5, 3.0])
    r = O.rmsnorm(np.full(4, c), w, eps)
    np.testing.assert_allclose(r, w * c / math.sqrt(c * c + eps), rtol=1e-15)
    x = np.array([3.0, -1.0, 0.0, 2.0])
    np.testing.assert_allclose(O.rmsnorm(x, None), x / math.sqrt(3.5 + 1e-8), rtol=1e-15)
    # mean of squares after the norm is ms / (ms + eps)
    g = np.random.default_rng(6).standard_normal((3, 50)) * 1e-4
    r = O.rmsnorm(g, None)
    ms = np.mean(g * g, axis=-1)
    np.testing.assert_allclose(np.mean(r * r, axis=-1), ms / (ms + 1e-8), rtol=1e-12)


def test_ternarize_codomain_scale_and_statistics():
    W = synth.weight(11, 1000, 1000)
    t, s = O.ternarize(W)
    assert t.dtype == np.int8 and set(np.unique(t).tolist()) <= {-1, 0, 1}
    assert s == np.float32(math.fsum(np.abs(W.astype(np.float64)).ravel().tolist()) / W.size)
    # iid Gaussian: P(t = 0) = P(|z| < 0.5 * sqrt(2/pi)) = erf(0.5 / sqrt(pi)) = 0.3101
    p0 = float(np.mean(t == 0))
    want = math.erf(0.5 / math.sqrt(math.pi))
    assert abs(want - 0.3101) < 1e-4
    assert abs(p0 - want) < 0.005
    assert abs(float(np.mean(t == 1)) - float(np.mean(t == -1))) < 0.005
    # sign symmetry and exact power-of-two scale invariance
    t_neg, s_neg = O.ternarize(-W)
    assert np.array_equal(t_neg, -t) and s_neg == s
    t4, s4 = O.ternarize(W * np.float32(4.0))
    assert np.array_equal(t4, t) and s4 == np.float32(4.0) * s
    # idempotence: more than 2/3 of the codes are non-zero, so t * c re-ternarises to t
    t2, _ = O.ternarize(t.astype(np.float32) * np.float32(0.01))
    assert np.array_equal(t2, t)


def test_ternarize_bruteforce_tiny_and_degenerate():
    W = np.array([[0.3, -0.1, 0.0, 0.5], [-0.6, 0.2, 0.05, -0.05]], dtype=np.float32)
    t, s = O.ternarize(W)
    s_ref = sum(abs(float(v)) for v in W.ravel()) / W.size
    assert abs(float(s) - s_ref) < 1e-7
    for n in range(2):
        for k in range(4):
            v = float(W[n, k]) / s_ref
            want = 0 if abs(v) < 0.5 else (1 if v > 0 else -1)
            assert t[n, k] == want
    tz, sz = O.ternarize(np.zeros((3, 5), np.float32))
    assert np.all(tz == 0) and sz == np.float32(1e-5)


def test_act_quant_invariants():
    g = np.random.default_rng(7)
    r = g.standard_normal((64, 300)) * g.uniform(0.01, 10, (64, 1))
    r[5] = 0.0
    q, deq, v = O.act_quant(r)
    assert q.dtype == np.int8 and q.min() >= -127 and q.max() <= 127
    nz = np.arange(64) != 5
    assert np.all(np.abs(q[nz]).max(axis=1) == 127)
    assert np.all(q[5] == 0)
    # reconstruction error at most half a step (plus the float32 rounding of r)
    r32 = r.astype(np.float32).astype(np.float64)
    err = np.abs(q * deq[:, None] - r32)
    assert np.all(err <= deq[:, None] * 0.5 * (1 + 1e-5) + 1e-12)
    # the step is absmax / 127
    np.testing.assert_allclose(deq[nz], np.abs(r32[nz]).max(axis=1) / 127, rtol=1e-15)
    # power-of-two scale invariance of the codes
    q2, deq2, _ = O.act_quant(r * 8.0)
    assert np.array_equal(q2, q)


# ---------------------------------------------------------------------------------------------
# BitLinear
# ---------------------------------------------------------------------------------------------
def test_bitlinear_handworked():
    gd = _golden("bitlinear_handworked.json")
    W = np.array(gd["W"], dtype=np.float32)
    t, s = O.ternarize(W)
    assert np.array_equal(t, np.array(gd["t"]))
    assert abs(float(s) - gd["s_w"]) < 1e-7
    y, taps = O.bitlinear(np.array([gd["x"]]), np.array(gd["norm_w"]), t, s)
    assert np.array_equal(taps["q"][0], np.array(gd["q"]))
    assert np.array_equal(taps["acc"][0], np.array(gd["acc"]))
    coeff = 3 * float(s) / (127 * math.sqrt(3.5 + 1e-8))
    np.testing.assert_allclose(y[0], np.array(gd["acc"]) * coeff, rtol=1e-6)


def test_bitlinear_bruteforce_conditional_add():
    # integer product equals the conditional add/subtract definition, and the float result equals
    # the dense product of the dequantised operands
    g = np.random.default_rng(8)
    M, K, N = 3, 37, 5
    x = g.standard_normal((M, K))
    nw = 1 + 0.1 * g.standard_normal(K)
    W = synth.weight(9, N, K)
    t, s = O.ternarize(W)
    y, taps = O.bitlinear(x, nw, t, s)
    for m in range(M):
        for n in range(N):
            assert taps["acc"][m, n] == O.ternary_dot_condadd(t[n], taps["q"][m])
    np.testing.assert_allclose(y, O.dense_reference(taps["q"], taps["deq"], t, s), rtol=1e-12, atol=1e-15)
    # the norm gain enters before quantisation: doubling every gain leaves q unchanged
    _, taps2 = O.bitlinear(x, 2 * nw, t, s)
    assert np.array_equal(taps2["q"], taps["q"])


def test_int_product_exact_in_float32_blas():
    # |partial sums| <= 127 * K < 2^24 for K <= 132,000, so float32 BLAS reproduces the integers
    g = np.random.default_rng(10)
    q = g.integers(-127, 128, (16, 2048)).astype(np.int8)
    t = g.integers(-1, 2, (24, 2048)).astype(np.int8)
    acc = O.int_matmul(q, t)
    f32 = q.astype(np.float32) @ t.astype(np.float32).T
    assert np.array_equal(acc, f32.astype(np.int64))


def test_zero_row_gives_zero_output():
    t, s = O.ternarize(synth.weight(12, 8, 32))
    y, taps = O.bitlinear(np.zeros((2, 32)), None, t, s)
    assert np.all(taps["q"] == 0) and np.all(y == 0)


# ---------------------------------------------------------------------------------------------
# packed format
# ---------------------------------------------------------------------------------------------
def test_packed_word_handworked():
    gd = _golden("packed_word_handworked.json")
    words = O.pack_codes(np.array([gd["codes"]]))
    assert words.shape == (1, 4)
    assert int(words[0, 0]) == int(gd["word_hex"], 16)
    assert np.all(words[0, 1:] == 0)


def test_pack_roundtrip_ragged():
    g = np.random.default_rng(13)
    for k in (1, 15, 16, 63, 64, 65, 200):
        t = g.integers(-1, 2, (7, k)).astype(np.int8)
        w = O.pack_codes(t)
        assert w.shape == (7, O.packed_row_words(k)) and (w.shape[1] * 4) % 16 == 0
        assert np.array_equal(O.unpack_codes(w, k), t)
    with pytest.raises(ValueError):
        O.unpack_codes(np.array([[0b10, 0, 0, 0]], dtype=np.uint32), 1)


def test_count_malformed_fields():
    # freshly packed codes (ragged k: the last word of a row holds padding fields) are well formed
    g = np.random.default_rng(17)
    t = g.integers(-1, 2, (5, 70)).astype(np.int8)
    w = O.pack_codes(t)
    assert O.count_malformed_fields(w, 70) == 0
    # the hand-worked word: its sixteen fields are real columns at k = 16 and padding at k = 7
    gd = _golden("packed_word_handworked.json")
    hw = np.array([[int(gd["word_hex"], 16), 0, 0, 0]], dtype=np.uint32)
    assert O.count_malformed_fields(hw, 16) == 0
    assert O.count_malformed_fields(hw, 7) == sum(1 for c in gd["codes"][7:] if c != 0)  # 6 nonzero codes
    # a 10 in a real column counts once; nonzero padding fields count once each, a 10 there too
    bad = w.copy()
    bad[1, 0] = (bad[1, 0] & ~np.uint32(3 << O.code_bit(5))) | np.uint32(2 << O.code_bit(5))
    assert O.count_malformed_fields(bad, 70) == 1
    bad[2, 4] |= np.uint32(1 << O.code_bit(75 - 64))   # column 75: padding, +1
    bad[3, 4] |= np.uint32(2 << O.code_bit(77 - 64))   # column 77: padding, 10
    assert O.count_malformed_fields(bad, 70) == 3
    # a field pattern 11 in a real column is a valid -1
    ok = w.copy()
    ok[0, 0] |= np.uint32(3 << O.code_bit(2))
    assert O.count_malformed_fields(ok, 70) == 0


# ---------------------------------------------------------------------------------------------
# block, decode and stack
# ---------------------------------------------------------------------------------------------
def _tiny_block(seed, d=32, inner=48, random_norms=True):
    sh = synth.BlockShape("t", d, inner, 1)
    return O.quantize_block(synth.block_params(seed, sh, random_norms)), sh


def test_block_prefill_equals_stepwise_decode():
    layers = [_tiny_block(20)[0], _tiny_block(21)[0]]
    x = synth.activations(22, (2, 9, 32))
    # stack of two blocks, prefill
    y1, h1, _ = O.block_forward(x, layers[0])
    y2, h2, _ = O.block_forward(y1, layers[1])
    state = np.zeros((2, 2, 32))
    for t in range(9):
        out, state = O.decode_step(x[:, t, :], layers, state)
        np.testing.assert_allclose(out, y2[:, t, :], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state[0], h1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state[1], h2, rtol=1e-12, atol=1e-12)


def test_block_batch_rows_independent_and_carried_state():
    qp, _ = _tiny_block(23)
    x = synth.activations(24, (3, 6, 32))
    y, hT, _ = O.block_forward(x, qp)
    for b in range(3):
        yb, hb, _ = O.block_forward(x[b:b + 1], qp)
        np.testing.assert_allclose(yb[0], y[b], rtol=1e-13, atol=1e-13)
    # splitting the sequence and carrying h reproduces the whole
    ya, ha, _ = O.block_forward(x[:, :4], qp)
    yb, hb, _ = O.block_forward(x[:, 4:], qp, ha)
    np.testing.assert_allclose(np.concatenate([ya, yb], 1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hb, hT, rtol=1e-12, atol=1e-12)


def test_block_residual_wiring():
    qp, sh = _tiny_block(25)
    x = synth.activations(26, (1, 5, 32))
    zero = {k: (np.zeros_like(v) if k.startswith("t_") else v) for k, v in qp.items()}
    y, _, inter = O.block_forward(x, zero)
    assert np.array_equal(y, x)           # both residual branches vanish with zero weights
    only_mlp_zero = dict(qp, t_gate=np.zeros_like(qp["t_gate"]))
    y2, _, inter2 = O.block_forward(x, only_mlp_zero)
    assert np.array_equal(y2, inter2["x1"])  # SiLU(0) * 0 = 0: the MLP adds nothing
    assert not np.allclose(inter2["x1"], x)


def test_block_gating_and_gnorm_definitions():
    qp, _ = _tiny_block(27)
    x = synth.activations(28, (1, 4, 32))
    _, _, it = O.block_forward(x, qp)
    f = 1 / (1 + np.exp(-it["zf"]))
    np.testing.assert_allclose(it["f"], f, rtol=1e-14)
    np.testing.assert_allclose(it["i"], it["zi"] * (1 / (1 + np.exp(-it["zi"]))) * (1 - f), rtol=1e-13, atol=1e-16)
    h = it["h"]
    rms = np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + 1e-8)
    u = h / rms * qp["gnorm_w"] * it["g"] / (1 + np.exp(-it["g"]))
    np.testing.assert_allclose(it["u"], u, rtol=1e-12, atol=1e-15)


def test_stack_embedding_gather():
    table = synth.embedding(30, 50, 32)
    ids = np.array([[3, 49, 0]])
    layers = [_tiny_block(31)[0]]
    y, st = O.stack_forward(ids, table, layers)
    y_ref, h_ref, _ = O.block_forward(table[ids].astype(np.float64), layers[0])
    np.testing.assert_allclose(y, y_ref, rtol=0, atol=0)
    np.testing.assert_allclose(st[0], h_ref, rtol=0, atol=0)


# ---------------------------------------------------------------------------------------------
# shapes printed on the pages
# ---------------------------------------------------------------------------------------------
def test_printed_layer_shapes():
    # hysenlabs.com: gate_proj out_features 11264 and down_proj in_features 5632 at hidden 2048;
    # default config 32000 vocab, hidden 2048, 24 layers
    sh = synth.B13
    ps = sh.proj_shapes
    assert ps["gate"] == (11264, 2048) and ps["down"] == (2048, 5632)
    assert ps["i"] == ps["f"] == ps["g"] == ps["o"] == (2048, 2048)
    assert sh.n_layers == 24 and synth.VOCAB == 32000
    assert (synth.M370.n_layers, synth.M370.d) == (24, 1024)
    assert (synth.B27.n_layers, synth.B27.d) == (32, 2560)


@pytest.mark.parametrize("shape,name_params", [(synth.M370, 370e6), (synth.B13, 1.3e9), (synth.B27, 2.7e9)])
def test_parameter_counts_match_size_names(shape, name_params):
    tied = O.model_param_count(shape.d, shape.inner, shape.n_layers)
    untied = tied + synth.VOCAB * shape.d
    per_block = 4 * shape.d ** 2 + 3 * shape.d * shape.inner
    assert O.block_param_count(shape.d, shape.inner) == per_block
    # both readings (tied or separate head) land within 10% of the published size name
    assert abs(tied / name_params - 1) < 0.10 and abs(untied / name_params - 1) < 0.10


# ---------------------------------------------------------------------------------------------
# language-model head and greedy generation
# ---------------------------------------------------------------------------------------------
def test_lm_head_hand_worked():
    # x = [3, 4]: mean square 12.5, r = x / sqrt(12.5 + eps); rows [1,0], [0,1], [1,1], [-1,0]
    x = np.array([[3.0, 4.0]])
    table = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [-1.0, 0.0]])
    logits = O.lm_head_logits(x, None, table)
    r = np.array([3.0, 4.0]) / np.sqrt(12.5 + 1e-8)
    np.testing.assert_allclose(logits[0], [r[0], r[1], r[0] + r[1], -r[0]], rtol=1e-12)
    np.testing.assert_allclose(logits[0], [0.848528137, 1.131370850, 1.979898987, -0.848528137], rtol=1e-8)
    assert O.greedy_next(logits)[0] == 2


def test_lm_head_identity_table_and_gain():
    # one-hot table rows: the logits are the normalised input itself, times the gain
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 16))
    w = 1.0 + 0.1 * rng.standard_normal(16)
    logits = O.lm_head_logits(x, w, np.eye(16))
    rms = np.sqrt((x ** 2).mean(axis=1, keepdims=True) + 1e-8)
    np.testing.assert_allclose(logits, x / rms * w, rtol=1e-12)
    assert np.array_equal(O.greedy_next(logits), np.argmax(x / rms * w, axis=1))


def test_lm_head_scale_invariance_and_ties():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 32))
    table = rng.standard_normal((50, 32))
    a = O.lm_head_logits(x, None, table)
    b = O.lm_head_logits(1000.0 * x, None, table)   # RMSNorm removes a positive scale
    np.testing.assert_allclose(a, b, rtol=1e-7)
    # duplicated best row: the lowest index wins
    best = int(O.greedy_next(a[:1])[0])
    table2 = np.concatenate([table[:best], table[best:best + 1], table[best:]], axis=0)
    assert int(O.greedy_next(O.lm_head_logits(x[:1], None, table2))[0]) == best


# ---------------------------------------------------------------------------------------------
# HGRN2 recurrence (state expansion)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("case", _golden("hgrn2_recurrence_handworked.json")["cases"], ids=lambda c: c["name"])
def test_hgrn2_handworked(case):
    q = np.array(case["q"])[None, :, None, :]
    f = np.array(case["f"])[None, :, None, :]
    i = np.array(case["i"])[None, :, None, :]
    S0 = np.array(case["S0"])[None, None]
    o, S = O.hgrn2_recurrence(q, f, i, S0)
    assert np.array_equal(o[0, :, 0], np.array(case["o"]))
    assert np.array_equal(S[0, 0], np.array(case["S"]))


def test_hgrn2_one_key_dimension_is_the_elementwise_recurrence():
    # dk = 1, q = 1: the state is one row and S_t = f_t S_{t-1} + (1 - f_t) i_t channel by
    # channel, which is the pinned element-wise scan with input (1 - f) i
    g = np.random.default_rng(21)
    B, T, H, dv = 2, 13, 3, 4
    f = g.uniform(0, 1, (B, T, H, 1))
    i = g.standard_normal((B, T, H, dv))
    S0 = g.standard_normal((B, H, 1, dv))
    o, S = O.hgrn2_recurrence(np.ones((B, T, H, 1)), f, i, S0)
    fb = np.broadcast_to(f, (B, T, H, dv)).reshape(B, T, H * dv)
    h = O.hgrn_scan(fb, ((1.0 - f) * i).reshape(B, T, H * dv), S0.reshape(B, H * dv))
    np.testing.assert_allclose(o.reshape(B, T, H * dv), h, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S.reshape(B, H * dv), h[:, -1], rtol=1e-12, atol=1e-12)


def test_hgrn2_bruteforce_attention_form():
    # unrolled: o_t[v] = sum_k q_t[k] (prod_{r<=t} f_r[k]) S0[k, v]
    #                  + sum_{s<=t} sum_k q_t[k] (prod_{s<r<=t} f_r[k]) (1 - f_s[k]) i_s[v]
    g = np.random.default_rng(22)
    B, T, H, dk, dv = 1, 6, 2, 3, 2
    q = g.standard_normal((B, T, H, dk))
    f = g.uniform(0, 1, (B, T, H, dk))
    i = g.standard_normal((B, T, H, dv))
    S0 = g.standard_normal((B, H, dk, dv))
    want = np.zeros((B, T, H, dv))
    for hh in range(H):
        for t in range(T):
            for v in range(dv):
                acc = 0.0
                for k in range(dk):
                    decay0 = 1.0
                    for r in range(t + 1):
                        decay0 *= f[0, r, hh, k]
                    acc += q[0, t, hh, k] * decay0 * S0[0, hh, k, v]
                    for s in range(t + 1):
                        w = 1.0 - f[0, s, hh, k]
                        for r in range(s + 1, t + 1):
                            w *= f[0, r, hh, k]
                        acc += q[0, t, hh, k] * w * i[0, s, hh, v]
                want[0, t, hh, v] = acc
    o, _ = O.hgrn2_recurrence(q, f, i, S0)
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-12)


def test_hgrn2_zero_forget_closed_form():
    # f = 0: the state is replaced every step by 1^T i_t, so o_t = (sum_k q_t[k]) i_t
    g = np.random.default_rng(23)
    B, T, H, dk, dv = 2, 5, 2, 4, 3
    q = g.standard_normal((B, T, H, dk))
    i = g.standard_normal((B, T, H, dv))
    o, S = O.hgrn2_recurrence(q, np.zeros((B, T, H, dk)), i, g.standard_normal((B, H, dk, dv)))
    np.testing.assert_allclose(o, q.sum(-1, keepdims=True) * i, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, np.broadcast_to(i[:, -1, :, None, :], (B, H, dk, dv)), rtol=0, atol=0)


def test_hgrn2_state_passing_and_causality():
    g = np.random.default_rng(24)
    B, T, H, dk, dv = 2, 24, 2, 4, 5
    q = g.standard_normal((B, T, H, dk))
    f = g.uniform(0.3, 1.0, (B, T, H, dk))
    i = g.standard_normal((B, T, H, dv))
    o, S = O.hgrn2_recurrence(q, f, i)
    # two halves with the state carried between them give the same outputs and final state
    o1, S1 = O.hgrn2_recurrence(q[:, :10], f[:, :10], i[:, :10])
    o2, S2 = O.hgrn2_recurrence(q[:, 10:], f[:, 10:], i[:, 10:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S2, S, rtol=1e-12, atol=1e-12)
    # a change at step 15 leaves every earlier output as it was and reaches step 15 itself
    i2 = i.copy()
    i2[1, 15, 0, 2] += 1.0
    o3, _ = O.hgrn2_recurrence(q, f, i2)
    assert np.array_equal(o3[:, :15], o[:, :15])
    assert not np.array_equal(o3[1, 15, 0], o[1, 15, 0])
    # heads and sequences are independent
    assert np.array_equal(o3[0], o[0]) and np.array_equal(o3[1, :, 1], o[1, :, 1])


# ---------------------------------------------------------------------------------------------
# backward: every gradient against central finite differences of the forward it differentiates
# ---------------------------------------------------------------------------------------------
def _fd(fun, arr, eps=1e-6):
    """Central differences of the scalar fun() with respect to every element of arr (in place)."""
    grad = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = arr[idx]
        arr[idx] = old + eps
        up = fun()
        arr[idx] = old - eps
        dn = fun()
        arr[idx] = old
        grad[idx] = (up - dn) / (2 * eps)
    return grad


def test_scan_backward_finite_differences():
    g = np.random.default_rng(31)
    B, T, D = 2, 7, 3
    f = g.uniform(0.1, 0.95, (B, T, D))
    i = g.standard_normal((B, T, D))
    h0 = g.standard_normal((B, D))
    c = g.standard_normal((B, T, D))        # L = sum c * h, so dL/dh_t = c_t
    loss = lambda: float(np.sum(c * O.hgrn_scan(f, i, h0)))
    df, di, dh0 = O.hgrn_scan_backward(f, i, c, h0)
    np.testing.assert_allclose(df, _fd(loss, f), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(di, _fd(loss, i), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dh0, _fd(loss, h0), rtol=1e-6, atol=1e-8)
    # an empty sequence: nothing depends on h0
    df0, di0, dh00 = O.hgrn_scan_backward(f[:, :0], i[:, :0], c[:, :0], h0)
    assert df0.shape == (B, 0, D) and di0.shape == (B, 0, D) and np.array_equal(dh00, np.zeros((B, D)))


def test_gates_backward_finite_differences():
    g = np.random.default_rng(32)
    zf = g.standard_normal((3, 5)) * 2
    zi = g.standard_normal((3, 5)) * 2
    a, b = g.standard_normal((3, 5)), g.standard_normal((3, 5))

    def loss():
        f, i = O.hgrn_gates(zf, zi)
        return float(np.sum(a * f + b * i))
    dzf, dzi = O.hgrn_gates_backward(zf, zi, a, b)
    np.testing.assert_allclose(dzf, _fd(loss, zf), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(dzi, _fd(loss, zi), rtol=1e-6, atol=1e-9)


def test_rmsnorm_backward_finite_differences():
    g = np.random.default_rng(33)
    x = g.standard_normal((4, 9))
    w = g.uniform(0.5, 1.5, 9)
    c = g.standard_normal((4, 9))
    loss = lambda: float(np.sum(c * O.rmsnorm(x, w)))
    dx, dw = O.rmsnorm_backward(x, w, c)
    np.testing.assert_allclose(dx, _fd(loss, x), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(dw, _fd(loss, w), rtol=1e-6, atol=1e-9)
    dx1, dw1 = O.rmsnorm_backward(x, None, c)
    loss1 = lambda: float(np.sum(c * O.rmsnorm(x, None)))
    np.testing.assert_allclose(dx1, _fd(loss1, x), rtol=1e-6, atol=1e-9)
    assert dw1 is None


def test_bitlinear_backward_is_straight_through():
    # straight-through: the forward keeps each quantiser's rounding offset (Q(v) - v) frozen and
    # differentiates v itself; finite differences of that surrogate give the gradients
    g = np.random.default_rng(34)
    M, K, N = 3, 16, 5
    x = g.standard_normal((M, K))
    nw = g.uniform(0.5, 1.5, K)
    W = g.standard_normal((N, K)) * 0.05
    dy = g.standard_normal((M, N))
    dx, dnw, dW = O.bitlinear_backward(x, nw, W, dy)
    t, s = O.ternarize(W)
    Wq = t * float(s)
    r0 = O.rmsnorm(x, nw)
    q, deq, _ = O.act_quant(r0)
    off_r = q * deq[:, None] - r0            # frozen activation rounding offset
    x_v, nw_v, W_v = x.copy(), nw.copy(), W.copy()
    loss_act = lambda: float(np.sum(dy * ((O.rmsnorm(x_v, nw_v) + off_r) @ Wq.T)))
    np.testing.assert_allclose(dx, _fd(loss_act, x_v), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(dnw, _fd(loss_act, nw_v), rtol=1e-6, atol=1e-9)
    off_w = Wq - W                           # frozen weight rounding offset
    loss_w = lambda: float(np.sum(dy * ((r0 + off_r) @ (W_v + off_w).T)))
    np.testing.assert_allclose(dW, _fd(loss_w, W_v), rtol=1e-6, atol=1e-9)
    # the forward values themselves are the quantised product (the offsets reproduce it)
    y, _ = O.bitlinear(x, nw, t, s)
    np.testing.assert_allclose((r0 + off_r) @ (W + off_w).T, y, rtol=1e-12, atol=1e-12)


def test_hgrn2_chunked_form_matches_recurrence():
    # the chunk-parallel form a tensor-core kernel evaluates: within a chunk, with
    # B_t = prod_{c0 <= r <= t} f_r (per key row) and the key k_s = 1 - f_s,
    #   o_t = (q_t * B_t) S_start + sum_{c0 <= s <= t} [(q_t * B_t) . (k_s / B_s)] i_s
    #   S_end = diag(B_end) S_start + sum_s (k_s * B_end / B_s)^T i_s
    # i.e. three small matrix products per chunk instead of a step-by-step state update
    g = np.random.default_rng(25)
    B, T, H, dk, dv, C = 2, 32, 2, 4, 3, 8
    q = g.standard_normal((B, T, H, dk))
    f = g.uniform(0.4, 1.0, (B, T, H, dk))
    i = g.standard_normal((B, T, H, dv))
    S0 = g.standard_normal((B, H, dk, dv))
    o_ref, S_ref = O.hgrn2_recurrence(q, f, i, S0)
    o = np.zeros_like(o_ref)
    S = S0.copy()
    for c0 in range(0, T, C):
        qc, fc, ic = q[:, c0:c0 + C], f[:, c0:c0 + C], i[:, c0:c0 + C]
        Bc = np.cumprod(fc, axis=1)                              # [B, C, H, dk]
        qb = qc * Bc
        kb = (1.0 - fc) / Bc
        A = np.einsum("bthk,bshk->bhts", qb, kb) * np.tril(np.ones((C, C)))
        o[:, c0:c0 + C] = np.einsum("bthk,bhkv->bthv", qb, S) + np.einsum("bhts,bshv->bthv", A, ic)
        S = Bc[:, -1][..., :, None] * S + np.einsum("bshk,bshv->bhkv", kb * Bc[:, -1][:, None], ic)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S, S_ref, rtol=1e-10, atol=1e-10)
