"""Kernel sweeps at their full sizes (GPU): BitLinear over (K, N) in {(2048, 2048),
(2048, 11264), (5632, 2048)} and M in {1, 16, 256, 4096, 32768} with N(0,1) bf16 activations, and
the HGRN scan at d = 2048, batch 4, T in {1K, 8K, 64K} with forget pre-activations N(4,1) (long
memory) or N(0,1) and inputs N(0,1), float32.

Each runs in the default engine selection (the launch configuration the library picks for that
size) and is checked against the oracle on sampled outputs the oracle computes one by one:
sampled token rows for BitLinear (exact int32 accumulators, codes equal except at near-ties,
outputs within 1e-3 / 1e-5), sampled channels for the scan (the recurrence is channel-wise).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
RTOL32, ATOL32 = 1e-3, 1e-5


@pytest.fixture(scope="module")
def mmf():
    import ternary_weight_matmul_b200 as m
    m.set_gemm_path(m.MMF_GEMM_AUTO)
    return m


def _to(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV, dtype)


def _ok(mmf):
    assert mmf.sync_status(DEV) == 0


def _near_tie(v, tol=1e-4):
    return np.abs(np.abs(v - np.floor(v)) - 0.5) < tol


@pytest.mark.parametrize("k,n", [(2048, 2048), (2048, 11264), (5632, 2048)])
@pytest.mark.parametrize("m", [1, 16, 256, 4096, 32768])
def test_bitlinear_sweep_sampled_rows(mmf, m, k, n):
    x = synth.activations(900 + m + k, (m, k))
    W = synth.weight(901 + n + k, n, k)
    pt = mmf.pack_ternary(_to(W))
    xb = _to(x, torch.bfloat16)
    y_run = mmf.bitlinear_fwd(xb, None, pt, y_dtype=torch.float32)
    y, q, deq, acc = mmf.bitlinear_fwd(xb, None, pt, y_dtype=torch.float32, debug=True)
    _ok(mmf)
    assert torch.equal(y_run, y)  # the debug taps do not change the product
    rows = np.unique(np.concatenate([np.random.default_rng(902).choice(m, min(m, 20), replace=False), [0, m - 1]]))
    xr = xb[rows].float().cpu().numpy().astype(np.float64)  # the bf16 values the kernels saw
    t, s = O.ternarize(W)
    q_g = q[rows].cpu().numpy()
    assert np.array_equal(acc[rows].cpu().numpy().astype(np.int64), O.int_matmul(q_g, t))
    y_ref, taps = O.bitlinear(xr, None, t, s)
    # codes: equal except where the oracle's value lies within 1e-4 of a half-integer
    mism = q_g != taps["q"]
    assert np.all(_near_tie(taps["v"])[mism])
    # dequantisation factors a/127 to 1e-6
    deq_g = deq[rows].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(deq_g, taps["deq"], rtol=1e-6)
    # every row: its output from its own exact accumulators; rows without a near-tie code: the
    # oracle's output
    y_g = y[rows].cpu().numpy()
    np.testing.assert_allclose(y_g, O.int_matmul(q_g, t) * deq_g[:, None] * float(s), rtol=RTOL32, atol=ATOL32)
    ok = ~mism.any(axis=1)
    np.testing.assert_allclose(y_g[ok], y_ref[ok], rtol=RTOL32, atol=ATOL32)


@pytest.mark.parametrize("t", [1024, 8192, 65536])
@pytest.mark.parametrize("long_memory", [True, False])
def test_scan_sweep_sampled_channels(mmf, t, long_memory):
    b, d = 4, 2048
    zf, zi = synth.scan_inputs(950 + t, b, t, d, long_memory)
    h, hl = mmf.hgrn_scan(_to(zf), _to(zi), None)
    _ok(mmf)
    ch = np.unique(np.concatenate([np.random.default_rng(951).choice(d, 12, replace=False), [0, d - 1]]))
    f, i = O.hgrn_gates(zf[:, :, ch], zi[:, :, ch])
    h_ref = O.hgrn_scan(f, i)
    np.testing.assert_allclose(h[:, :, ch].cpu().numpy(), h_ref, rtol=RTOL32, atol=ATOL32)
    np.testing.assert_allclose(hl[:, ch].cpu().numpy(), h_ref[:, -1], rtol=RTOL32, atol=ATOL32)
