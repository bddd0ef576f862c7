"""CPU checks of the arithmetic identities the CUDA kernels are built on (no GPU, no CUDA code):
each restates a kernel's decomposition in numpy and compares it with the oracle's direct form.

* The scan backward in chunks of time, reversed: the total gradient G_t = f_{t+1} G_{t+1} + dh_t
  is affine in what enters a chunk from the later steps, so a chunk folds to (A, B) with
  f_{t0} G_{t0} = A carry + B; a walk over the chunks from the last to the first gives every
  chunk its carry, and replaying each chunk from its carry reproduces the sequential backward.
* The bf16 hi / lo pair of the tensor-core products: hi = bf16(a), lo = bf16(a - hi) carries a
  float32 value to within 2^-17 of its magnitude, and a product with an operand bf16 holds exactly
  (ternary or int8 codes) is then the float32 product up to that bound.
* The chunked form a tensor-core HGRN2 kernel would evaluate (not built: the recurrence kernel is
  the path): the factored chunk form overflows float32 for small gates, while sub-chunks of 16
  steps with every decay taken relative to the sub-chunk (exponents <= 0) reproduce the oracle's
  recurrence in float32 for gates down to 1e-6.
* The packed format's byte-permute expansion: four byte permutes of one constant turn a word of
  16 two-bit codes into four int8 quads, and reproduce the oracle's packed codes column by column.
* The GEMM epilogue's int32 -> float32 step through the mantissa of 1.5 * 2^23: exact for every
  accumulator the library can produce (K <= 32768), checked exhaustively.
* The scan's gates with one reciprocal per channel and exponent arguments clamped at -40: float32-
  accurate against sigmoid and SiLU (1 - f) over saturated arguments, never inf or NaN.
* The activation code with no clamp: a row's maximum maps to exactly 127 (a whole binade of a
  checked), and the low byte of x + 1.5 * 2^23 is rint(x), ties to even.
* The integrity check's word-level bit count equals the oracle's field-by-field definition on
  packed codes, planted faults and random words.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth


def _chunked_scan_backward(f, dh, chunk):
    """G for every step by the fold / reverse carry / replay decomposition ([B, T, D] float64)."""
    b, t, d = f.shape
    nch = (t + chunk - 1) // chunk
    A = np.ones((b, nch, d))
    Bv = np.zeros((b, nch, d))
    for c in range(nch):                       # fold: f_{t0} G_{t0} at carry 0, and the product of f
        t0, t1 = c * chunk, min(c * chunk + chunk, t)
        for s in range(t1 - 1, t0 - 1, -1):
            Bv[:, c] = f[:, s] * (dh[:, s] + Bv[:, c])
            A[:, c] = f[:, s] * A[:, c]
    carry = np.zeros((b, nch, d))
    run = np.zeros((b, d))
    for c in range(nch - 1, -1, -1):            # reverse walk over the chunks
        carry[:, c] = run
        run = A[:, c] * run + Bv[:, c]
    dh0_factor = run                           # = f_0 G_0
    G = np.zeros((b, t, d))
    for c in range(nch):                       # replay every chunk from its carry
        t0, t1 = c * chunk, min(c * chunk + chunk, t)
        cterm = carry[:, c]
        for s in range(t1 - 1, t0 - 1, -1):
            G[:, s] = dh[:, s] + cterm
            cterm = f[:, s] * G[:, s]
    return G, dh0_factor


@pytest.mark.parametrize("t,chunk", [(37, 32), (700, 32), (64, 64), (5, 32), (1, 1), (130, 16)])
def test_chunked_reverse_scan_gradient_matches_the_sequential_one(t, chunk):
    b, d = 2, 6
    zf, zi = synth.scan_inputs(150 + t, b, t, d, long_memory=t > 100)
    f, i = O.hgrn_gates(zf.astype(np.float64), zi.astype(np.float64))
    dh = synth.activations(151 + t, (b, t, d)).astype(np.float64)
    h0 = synth.activations(152 + t, (b, d)).astype(np.float64)
    df, di, dh0 = O.hgrn_scan_backward(f, i, dh, h0)
    G, dh0_c = _chunked_scan_backward(f, dh, chunk)
    # di = G (the oracle's sequential total gradient); dh0 = f_0 G_0
    np.testing.assert_allclose(G, di, rtol=1e-12, atol=1e-12 * np.abs(di).max())
    np.testing.assert_allclose(dh0_c, dh0, rtol=1e-12, atol=1e-12 * max(np.abs(dh0).max(), 1e-300))
    # and df = G h_{t-1} with the forward's states
    h = O.hgrn_scan(f, i, h0)
    hprev = np.concatenate([h0[:, None, :], h[:, :-1, :]], axis=1)
    np.testing.assert_allclose(G * hprev, df, rtol=1e-12, atol=1e-12 * np.abs(df).max())


def _split_bf16(a: np.ndarray):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    hi = t.to(torch.bfloat16)
    lo = (t - hi.float()).to(torch.bfloat16)
    return hi.double().numpy(), lo.double().numpy()


def test_bf16_hi_lo_pair_carries_float32_to_two_to_the_minus_17():
    rng = np.random.default_rng(160)
    a = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    hi, lo = _split_bf16(a)
    err = np.abs(hi + lo - a.astype(np.float64))
    assert np.all(err <= 2.0 ** -17 * np.abs(a.astype(np.float64)))


def test_hi_lo_products_with_exact_codes_stay_float32_accurate():
    # dr = dy . t (ternary) and dW = (dy a/127)^T q (int8): the codes are exact in bf16, so the
    # hi / lo product differs from the float64 product by at most 2^-17 |dy| |codes| per term
    rng = np.random.default_rng(161)
    m, n, k = 64, 96, 80
    dy = rng.standard_normal((m, n)).astype(np.float32)
    t = rng.integers(-1, 2, (n, k)).astype(np.float64)
    q = rng.integers(-127, 128, (m, k)).astype(np.float64)
    hi, lo = _split_bf16(dy)
    assert np.array_equal(torch.from_numpy(t).to(torch.bfloat16).double().numpy(), t)
    assert np.array_equal(torch.from_numpy(q).to(torch.bfloat16).double().numpy(), q)
    exact = dy.astype(np.float64) @ t
    approx = hi @ t + lo @ t
    bound = 2.0 ** -17 * (np.abs(dy.astype(np.float64)) @ np.abs(t))
    assert np.all(np.abs(approx - exact) <= bound + 1e-300)
    exact_w = dy.astype(np.float64).T @ q
    approx_w = hi.T @ q + lo.T @ q
    bound_w = 2.0 ** -17 * (np.abs(dy.astype(np.float64)).T @ np.abs(q))
    assert np.all(np.abs(approx_w - exact_w) <= bound_w + 1e-300)


# ---------------------------------------------------------------------------------------------
# HGRN2: the chunked form for a tensor-core kernel (plan; the recurrence kernel is the built path)
# ---------------------------------------------------------------------------------------------
def _hgrn2_inputs(seed, b, t, h, dk, dv, fmin):
    g = np.random.default_rng(seed)
    q = g.standard_normal((b, t, h, dk))
    f = np.exp(g.uniform(np.log(fmin), 0.0, (b, t, h, dk)))   # forget gates down to fmin
    i = g.standard_normal((b, t, h, dv))
    s0 = g.standard_normal((b, h, dk, dv))
    return q, f, i, s0


def test_hgrn2_factored_chunk_form_overflows_float32_for_small_gates():
    # the factored chunk form needs 1 / prod(f) over the chunk: with gates near 1e-3 it leaves
    # float32 within 16 steps, so a kernel cannot use it as it stands
    f = np.full(16, 1e-3, dtype=np.float32)
    with np.errstate(over="ignore", divide="ignore"):
        inv = np.float32(1.0) / np.cumprod(f)
    assert not np.all(np.isfinite(inv))


def _hgrn2_subchunk(q, f, i, s0, L, dt):
    """The two-level form in precision dt: sub-chunks of L steps in order, the state passed
    between them; inside a sub-chunk every decay is exp(G_t - G_s) <= 1 with G the running sum of
    log f from the sub-chunk's start, so nothing overflows whatever the gates. Per (sequence,
    head), with the state's dv columns as the rows of the products (O^T = S^T Q~^T and
    S^T <- S^T diag(e^G_last) + I^T K~: 128-row operands when dv = 128):
      o_t   = (q_t * e^{G_t}) S_b + sum_{s<=t} [sum_k q_t[k] (1 - f_s[k]) e^{G_t[k] - G_s[k]}] i_s
      S_e   = diag(e^{G_last}) S_b + sum_s ((1 - f_s) * e^{G_last - G_s})^T i_s"""
    q, f, i = q.astype(dt), f.astype(dt), i.astype(dt)
    b, t, h, dk = f.shape
    dv = i.shape[-1]
    S = s0.astype(dt).copy()
    o = np.zeros((b, t, h, dv), dtype=dt)
    for b0 in range(0, t, L):
        e0 = min(b0 + L, t)
        lf = np.log(f[:, b0:e0])                          # [B, l, H, dk], <= 0
        G = np.cumsum(lf, axis=1)                         # inclusive running log-decay
        key = (dt(1) - f[:, b0:e0])
        qc, ic = q[:, b0:e0], i[:, b0:e0]
        inter = np.einsum("bthk,bhkv->bthv", qc * np.exp(G), S)
        diff = G[:, :, None] - G[:, None, :]              # [B, t, s, H, dk] = G_t - G_s
        mask = np.tril(np.ones((e0 - b0, e0 - b0), dtype=bool))[None, :, :, None, None]
        dec = np.where(mask, np.exp(np.where(mask, diff, dt(0))), dt(0))
        P = np.einsum("bthk,bshk,btshk->bhts", qc, key, dec)
        o[:, b0:e0] = inter + np.einsum("bhts,bshv->bthv", P, ic)
        Gl = G[:, -1]                                     # [B, H, dk]
        S = np.exp(Gl)[..., :, None] * S + np.einsum("bshk,bshv->bhkv", key * np.exp(Gl[:, None] - G), ic)
    return o, S


@pytest.mark.parametrize("fmin", [0.5, 1e-3, 1e-6])
def test_hgrn2_subchunk_form_matches_the_recurrence(fmin):
    q, f, i, s0 = _hgrn2_inputs(170, 2, 70, 2, 16, 8, fmin)
    o_ref, S_ref = O.hgrn2_recurrence(q, f, i, s0)
    o64, S64 = _hgrn2_subchunk(q, f, i, s0, 16, np.float64)
    np.testing.assert_allclose(o64, o_ref, rtol=1e-10, atol=1e-10 * np.abs(o_ref).max())
    np.testing.assert_allclose(S64, S_ref, rtol=1e-10, atol=1e-10 * np.abs(S_ref).max())
    # in float32 every intermediate stays finite and the result is float32-accurate
    with np.errstate(over="raise", invalid="raise"):
        o32, S32 = _hgrn2_subchunk(q, f, i, s0, 16, np.float32)
    np.testing.assert_allclose(o32, o_ref, rtol=1e-4, atol=1e-5 * np.abs(o_ref).max())
    np.testing.assert_allclose(S32, S_ref, rtol=1e-4, atol=1e-5 * np.abs(S_ref).max())


# ---------------------------------------------------------------------------------------------
# The packed format's byte-permute expansion (the device helper that turns one 32-bit word of
# 16 codes into four int8 quads), restated with the byte-permute instruction's definition: each
# 4-bit selector picks one byte of the 8-byte pair {y, x} (x = bytes 0-3); result byte i takes
# the byte that selector nibble i names.
# ---------------------------------------------------------------------------------------------
def _byte_perm(x: int, y: int, s: int) -> int:
    pair = (y << 32) | x
    out = 0
    for i in range(4):
        sel = (s >> (4 * i)) & 7
        out |= ((pair >> (8 * sel)) & 0xFF) << (8 * i)
    return out


def _expand_word(w: int) -> list[int]:
    lo = w & 0x33333333
    hi = (w >> 2) & 0x33333333
    table = 0xFF000100                      # bytes 0x00, 0x01, 0x00, 0xFF for fields 00, 01, 10, 11
    quads = [_byte_perm(table, 0, lo & 0xFFFF), _byte_perm(table, 0, hi & 0xFFFF),
             _byte_perm(table, 0, lo >> 16), _byte_perm(table, 0, hi >> 16)]
    codes = []
    for q in quads:                         # lowest column in byte 0, int8 lanes
        codes += [((q >> (8 * b)) & 0xFF) - 256 * (((q >> (8 * b)) & 0xFF) >= 128) for b in range(4)]
    return codes


@pytest.mark.parametrize("n,k", [(3, 16), (5, 65), (2, 200), (4, 1024)])
def test_byte_permute_expansion_recovers_the_oracles_packed_codes(n, k):
    rng = np.random.default_rng(180 + k)
    t = rng.integers(-1, 2, (n, k)).astype(np.int8)
    words = O.pack_codes(t).astype(np.uint32)
    kw = O.packed_row_words(k)
    assert words.shape == (n, kw)
    for r in range(n):
        got = [c for w in words[r] for c in _expand_word(int(w))]
        assert got[:k] == t[r].tolist()
        assert not any(got[k:])             # padding columns expand to zero codes
    # the unused pattern 10 expands to 0 (a malformed field reads as a zero weight)
    assert _expand_word(0xAAAAAAAA) == [0] * 16
    assert _expand_word(0x55555555) == [1] * 16 and _expand_word(0xFFFFFFFF) == [-1] * 16


# ---------------------------------------------------------------------------------------------
# The GEMM epilogue's int32 -> float32 step without a conversion instruction: the bit pattern
# a + 0x4B400000 is the float 1.5 * 2^23 + a (mantissa spacing 1 there), and subtracting 1.5 * 2^23
# is exact, so the result is float(a) exactly for every |a| <= 2^22 -- which covers every
# accumulator of K <= 32768 int8 x ternary products (|acc| <= 127 K < 2^22).
# ---------------------------------------------------------------------------------------------
def _acc_to_float(a: np.ndarray) -> np.ndarray:
    bits = (a.astype(np.int64) + 0x4B400000).astype(np.uint32)
    return bits.view(np.float32) - np.float32(12582912.0)


def test_mantissa_int_to_float_is_exact_over_the_accumulator_range():
    a = np.arange(-(1 << 22), (1 << 22) + 1, dtype=np.int32)       # every value, exhaustively
    got = _acc_to_float(a)
    assert got.dtype == np.float32
    assert np.array_equal(got, a.astype(np.float32))
    assert 127 * 32768 < (1 << 22)                                    # the library's largest K
    # one step outside the range the identity no longer holds: the guard on K is needed
    out = np.array([(1 << 22) + 1, -(1 << 22) - 1], dtype=np.int32)
    assert not np.any(_acc_to_float(out) == out.astype(np.float32))


# ---------------------------------------------------------------------------------------------
# The scan's gate arithmetic with one reciprocal per channel: ef = e^-zf and ez = e^-zi with both
# exponent arguments clamped at -40, r = 1 / ((1 + ef)(1 + ez)), f = (1 + ez) r, i = zi ef r.
# Restated in float32 (exact exponentials and reciprocal; the device's approximate ones add a few
# ulp) against the oracle's sigmoid and SiLU (1 - f) in float64, over saturated arguments too.
# ---------------------------------------------------------------------------------------------
def _gates_one_reciprocal(zf: np.ndarray, zi: np.ndarray):
    f32 = np.float32
    zf, zi = zf.astype(f32), zi.astype(f32)
    nl = f32(-1.4426950408889634)
    ef = np.exp2(np.maximum(zf, f32(-40.0)) * nl, dtype=f32)
    ez = np.exp2(np.maximum(zi, f32(-40.0)) * nl, dtype=f32)
    pz = ez + f32(1.0)
    r = f32(1.0) / ((ef + f32(1.0)) * pz)
    return pz * r, (zi * ef) * r


def test_one_reciprocal_gates_match_sigmoid_and_silu():
    g = np.linspace(-200.0, 200.0, 801)
    zf, zi = np.meshgrid(g, g, indexing="ij")
    rng = np.random.default_rng(190)
    zf = np.concatenate([zf.ravel(), rng.normal(0, 3, 20000), rng.normal(4, 1, 20000)])
    zi = np.concatenate([zi.ravel(), rng.normal(0, 3, 20000), rng.normal(0, 1, 20000)])
    zf = zf.astype(np.float32).astype(np.float64)
    zi = zi.astype(np.float32).astype(np.float64)
    # the definitions in float64 with 1 - f taken as sigmoid(-zf) (no cancellation as f -> 1);
    # they agree with the oracle's f and SiLU(zi) (1 - f) to its own float64 rounding of 1 - f
    with np.errstate(over="ignore"):
        f_ref = 1.0 / (1.0 + np.exp(-zf))
        i_ref = zi / (1.0 + np.exp(-zi)) / (1.0 + np.exp(zf))
    f_o, i_o = O.hgrn_gates(zf, zi)
    assert np.all(np.abs(f_o - f_ref) <= 1e-15)
    assert np.all(np.abs(i_o - i_ref) <= 1e-12 * np.abs(i_ref) + 2.3e-16 * np.abs(zi) / (1.0 + np.exp(-zi)))
    with np.errstate(over="raise", invalid="raise"):
        f, i = _gates_one_reciprocal(zf, zi)
    assert np.all(np.isfinite(f)) and np.all(np.isfinite(i))
    # float32 rounding (the exponent argument's rounding dominates near the clamp), and the clamp
    # itself: sigmoid(-40) < 5e-18 bounds what it moves
    np.testing.assert_array_less(np.abs(f - f_ref), 5e-6 * np.abs(f_ref) + 5e-18)
    np.testing.assert_array_less(np.abs(i - i_ref), 5e-6 * np.abs(i_ref) + 5e-18 * np.abs(zi) + 1e-38)


# ---------------------------------------------------------------------------------------------
# The activation code without a clamp or a conversion instruction: x = r * fl(127 / a) is at most
# fl(a * fl(127 / a)) in magnitude (a = max |r| of the row), which rounds to exactly 127; and the
# low byte of the float32 bits of x + 1.5 * 2^23 is rint(x) (ties to even) for |x| < 127.5 (at
# x = +127.5 the code would be 128, which the bound above keeps out of reach).
# ---------------------------------------------------------------------------------------------
def test_row_maximum_maps_to_code_127_without_a_clamp():
    f32 = np.float32
    one_binade = (np.arange(1 << 23, dtype=np.uint32) | np.uint32(0x3F800000)).view(np.float32)  # [1, 2)
    rng = np.random.default_rng(200)
    spread = np.exp(rng.uniform(np.log(1e-5), np.log(1e30), 2_000_000)).astype(f32)
    for a in (one_binade, spread):
        x = a * (f32(127.0) / a)             # float32 product of float32 operands, each rounded
        assert x.dtype == f32
        assert np.all(np.abs(x - 127.0) <= 2 * np.spacing(f32(127.0)))
        assert np.all(np.rint(x) == 127.0)
    # the dequantisation factor a * fl(1/127) is within 1.5 ulp of a / 127 (scaling by powers of
    # two is exact, so one binade covers every a in the normal range)
    d = one_binade * (f32(1.0) / f32(127.0))
    err = np.abs(d.astype(np.float64) - one_binade.astype(np.float64) / 127.0)
    assert np.all(err <= 1.5 * np.spacing(d).astype(np.float64))


def test_code_byte_from_the_rounding_add_is_rint_ties_to_even():
    f32 = np.float32
    halves = np.arange(-127.5, 128.0, 1.0, dtype=f32)
    near = np.concatenate([halves, np.nextafter(halves, f32(-200)), np.nextafter(halves, f32(200)),
                           np.arange(-127, 128, dtype=f32)])
    rng = np.random.default_rng(201)
    x = np.concatenate([near, rng.uniform(-127.5, 127.5, 2_000_000).astype(f32)])
    x = x[np.abs(x) < 127.5]
    bits = (x + f32(12582912.0)).astype(f32).view(np.uint32)
    code = (bits & 0xFF).astype(np.uint8).view(np.int8)
    assert np.array_equal(code.astype(np.int64), np.rint(x).astype(np.int64))


# ---------------------------------------------------------------------------------------------
# The integrity check's word-level count: with lo / hi the low / high bits of the 16 fields of a
# word and pad the low bits of its padding fields, a word holds popc(hi & ~lo & ~pad) real-column
# 10 fields and popc((lo | hi) & pad) nonzero padding fields (a padding 10 counted once).
# Restated with the field offsets of the oracle's code_bit, against the oracle's definition.
# ---------------------------------------------------------------------------------------------
def _fields_from(jmin: int) -> int:
    m = 0
    for j in range(jmin, 16):
        m |= 1 << O.code_bit(j)
    return m


def _word_level_count(words: np.ndarray, k: int) -> int:
    n, kw = words.shape
    total = 0
    for r in range(n):
        for e in range(kw):
            w = int(words[r, e])
            col0 = e * 16
            lo, hi = w & 0x55555555, (w >> 1) & 0x55555555
            pad = _fields_from(max(k - col0, 0)) if col0 + 16 > k else 0
            total += bin(hi & ~lo & ~pad & 0xFFFFFFFF).count("1") + bin((lo | hi) & pad).count("1")
    return total


@pytest.mark.parametrize("k", [1, 16, 70, 130, 256])
def test_integrity_word_count_equals_the_oracles_definition(k):
    rng = np.random.default_rng(210 + k)
    t = rng.integers(-1, 2, (6, k)).astype(np.int8)
    words = O.pack_codes(t)
    assert _word_level_count(words, k) == O.count_malformed_fields(words, k) == 0
    kw = words.shape[1]
    bad = words.copy()
    bad[1, 0] = (int(bad[1, 0]) & ~(3 << O.code_bit(0))) | (2 << O.code_bit(0))      # real column: 10
    if 16 * kw > k:                                                                  # padding fields
        col = k
        bad[2, col // 16] = int(bad[2, col // 16]) | (1 << O.code_bit(col % 16))      # +1
        col = 16 * kw - 1
        bad[3, col // 16] = int(bad[3, col // 16]) | (2 << O.code_bit(col % 16))      # 10, counted once
    assert _word_level_count(bad, k) == O.count_malformed_fields(bad, k) >= 1
    garbage = rng.integers(0, 1 << 32, (4, kw), dtype=np.uint64).astype(np.uint32)
    assert _word_level_count(garbage, k) == O.count_malformed_fields(garbage, k)
