"""CPU checks of the arithmetic identities the CUDA kernels are built on (no GPU, no CUDA code):
each restates a kernel's decomposition in numpy and compares it with the oracle's direct form.

* The scan backward in chunks of time, reversed: the total gradient G_t = f_{t+1} G_{t+1} + dh_t
  is affine in what enters a chunk from the later steps, so a chunk folds to (A, B) with
  f_{t0} G_{t0} = A carry + B; a walk over the chunks from the last to the first gives every
  chunk its carry, and replaying each chunk from its carry reproduces the sequential backward.
* The bf16 hi / lo pair of the tensor-core products: hi = bf16(a), lo = bf16(a - hi) carries a
  float32 value to within 2^-17 of its magnitude, and a product with an operand bf16 holds exactly
  (ternary or int8 codes) is then the float32 product up to that bound.
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
