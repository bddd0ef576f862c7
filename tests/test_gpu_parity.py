"""GPU parity of every kernel path against the CPU oracle, through the C ABI.

Tolerances (stated by the build target): integer accumulations bit-exact; float32 outputs within
1e-5 absolute + 1e-3 relative per element; bfloat16 outputs within 2e-2 relative. Quantisation
decisions: the first activation quantisation of a BitLinear sees a correctly rounded float32 r on
both sides, so its codes must match exactly except where the oracle's pre-rounding value lies
within 1e-4 of a half-integer (none are expected); in chained stages a code can flip by one at
such near-ties, which the block-level checks bound instead of forbidding (see the block tests).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_checks import (_close, _codes_match, _near_tie, _np, check_block_end_to_end, check_block_stages,
                           check_chain_end_to_end, check_decode_layer)

pytestmark = pytest.mark.gpu

RTOL32, ATOL32 = 1e-3, 1e-5
RTOL16 = 2e-2


@pytest.fixture(scope="module")
def mmf():
    import ternary_weight_matmul_b200 as m
    from ternary_weight_matmul_b200 import build
    build.build()
    m.lib()
    torch.cuda.set_device(0)
    yield m
    m.set_gemm_path(m.MMF_GEMM_AUTO)


DEV = "cuda:0"


def _to(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV, dtype)


def _bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _ok(mmf):
    assert mmf.sync_status(DEV) == 0


# ---------------------------------------------------------------------------------------------
# K0 pack
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(256, 256), (1408, 256), (256, 704), (37, 100), (3, 1), (5, 64), (7, 65)])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_pack_parity(mmf, n, k, wdt):
    W = synth.weight(100 + n + k, n, k)
    if wdt == "bf16":
        W = _bf16_round(W)
    wt = _to(W, torch.float32 if wdt == "f32" else torch.bfloat16)
    pt = mmf.pack_ternary(wt)
    _ok(mmf)
    t_ref, s_ref = O.ternarize(W)
    assert pt.scale.item() == float(s_ref)
    words = pt.codes.cpu().numpy().view(np.uint32)
    assert np.array_equal(words, O.pack_codes(t_ref))


def test_pack_degenerate_zero_matrix(mmf):
    pt = mmf.pack_ternary(torch.zeros(4, 70, device=DEV))
    _ok(mmf)
    assert pt.scale.item() == np.float32(1e-5)
    assert int(pt.codes.abs().sum()) == 0


# ---------------------------------------------------------------------------------------------
# BitLinear (both integer-product engines)
# ---------------------------------------------------------------------------------------------
BITLINEAR_SHAPES = [(1, 256, 256), (3, 768, 256), (8, 1408, 256), (127, 256, 704), (256, 256, 256),
                    (300, 200, 100), (130, 384, 1024), (9, 64, 2560), (40, 128, 2048), (5, 96, 7040)]


@pytest.mark.parametrize("engine", ["tensor", "simt"])
@pytest.mark.parametrize("m,n,k", BITLINEAR_SHAPES)
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_bitlinear_parity(mmf, engine, m, n, k, xdt):
    mmf.set_gemm_path(mmf.MMF_GEMM_TENSOR if engine == "tensor" else mmf.MMF_GEMM_SIMT)
    try:
        seed = m * 7 + n * 3 + k
        x = synth.activations(seed, (m, k))
        if xdt == "bf16":
            x = _bf16_round(x)
        nw = synth.norm_weight(seed + 1, k, random=True)
        W = synth.weight(seed + 2, n, k)
        pt = mmf.pack_ternary(_to(W))
        y, q, deq, acc = mmf.bitlinear_fwd(_to(x, torch.float32 if xdt == "f32" else torch.bfloat16), _to(nw), pt,
                                            y_dtype=torch.float32, debug=True)
        _ok(mmf)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    t, s = O.ternarize(W)
    y_ref, taps = O.bitlinear(x.astype(np.float64), nw, t, s)
    q_g, acc_g, deq_g, y_g = q.cpu().numpy(), acc.cpu().numpy(), deq.cpu().numpy(), y.cpu().numpy()
    # activation codes: identical except at near-ties of the oracle's float32 value
    mism = q_g != taps["q"]
    assert np.all(np.abs(q_g.astype(int) - taps["q"].astype(int)) <= 1)
    assert np.all(_near_tie(taps["v"])[mism])
    # integer accumulation: bit-exact given the kernel's own codes
    assert np.array_equal(acc_g.astype(np.int64), O.int_matmul(q_g, t))
    np.testing.assert_allclose(deq_g, taps["deq"], rtol=1e-6)
    # epilogue arithmetic on the kernel's own accumulators
    y_from_acc = acc_g.astype(np.float64) * deq_g.astype(np.float64)[:, None] * float(s)
    np.testing.assert_allclose(y_g, y_from_acc, rtol=RTOL32, atol=ATOL32)
    # end to end against the oracle: elementwise where no code flipped
    rows_ok = ~mism.any(axis=1)
    np.testing.assert_allclose(y_g[rows_ok], y_ref[rows_ok], rtol=RTOL32, atol=ATOL32)


def test_bitlinear_zero_rows_and_bf16_output(mmf):
    k, n = 256, 512
    x = synth.activations(5, (20, k))
    x[3] = 0.0
    x[17] = 0.0
    W = synth.weight(6, n, k)
    pt = mmf.pack_ternary(_to(W))
    y = mmf.bitlinear_fwd(_to(x), None, pt, y_dtype=torch.bfloat16)
    _ok(mmf)
    t, s = O.ternarize(W)
    y_ref, _ = O.bitlinear(x.astype(np.float64), None, t, s)
    yg = y.float().cpu().numpy()
    assert np.all(yg[3] == 0) and np.all(yg[17] == 0)
    np.testing.assert_allclose(yg, y_ref, rtol=RTOL16, atol=1e-2 * np.abs(y_ref).max())


@pytest.mark.parametrize("m", [1, 64, 1000])
def test_bitlinear_engines_bit_identical(mmf, m):
    k, n = 1024, 640
    x = _to(synth.activations(40 + m, (m, k)))
    pt = mmf.pack_ternary(_to(synth.weight(41, n, k)))
    outs = []
    for path in (mmf.MMF_GEMM_TENSOR, mmf.MMF_GEMM_SIMT):
        mmf.set_gemm_path(path)
        outs.append(mmf.bitlinear_fwd(x, None, pt, debug=True))
    mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    _ok(mmf)
    assert torch.equal(outs[0][3], outs[1][3])   # accumulators
    assert torch.equal(outs[0][0], outs[1][0])   # rescaled outputs


@pytest.mark.parametrize("m,n,k", [(4096, 9472, 1024), (4096, 2048, 2816)])
def test_bitlinear_large_sampled_rows(mmf, m, n, k):
    # enough weight tiles that the tensor-core engine groups several of them per resident
    # activation block (K <= 1024) or streams (K > 1024); checked on sampled rows
    mmf.set_gemm_path(mmf.MMF_GEMM_TENSOR)
    try:
        x = synth.activations(70 + k, (m, k))
        W = synth.weight(71 + k, n, k)
        pt = mmf.pack_ternary(_to(W))
        y, q, deq, acc = mmf.bitlinear_fwd(_to(x), None, pt, debug=True)
        _ok(mmf)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    rows = np.random.default_rng(72).choice(m, 48, replace=False)
    rows = np.concatenate([rows, [0, 127, 128, m - 1]])
    t, s = O.ternarize(W)
    q_g = q[rows].cpu().numpy()
    acc_g = acc[rows].cpu().numpy()
    assert np.array_equal(acc_g.astype(np.int64), O.int_matmul(q_g, t))
    y_ref, taps = O.bitlinear(x[rows].astype(np.float64), None, t, s)
    mism = q_g != taps["q"]
    assert np.all(_near_tie(taps["v"])[mism])
    ok = ~mism.any(axis=1)
    np.testing.assert_allclose(y[rows].cpu().numpy()[ok], y_ref[ok], rtol=RTOL32, atol=ATOL32)


# ---------------------------------------------------------------------------------------------
# HGRN scan
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("b,t,d", [(1, 1, 32), (2, 7, 96), (3, 128, 100), (1, 129, 64), (2, 1000, 32), (1, 300, 2048)])
@pytest.mark.parametrize("long_memory", [False, True])
@pytest.mark.parametrize("with_h0", [False, True])
def test_scan_parity_f32(mmf, b, t, d, long_memory, with_h0):
    zf, zi = synth.scan_inputs(b * t + d, b, t, d, long_memory)
    h0 = synth.activations(9, (b, d)) if with_h0 else None
    h, hl = mmf.hgrn_scan(_to(zf), _to(zi), _to(h0) if with_h0 else None)
    _ok(mmf)
    f, i = O.hgrn_gates(zf, zi)
    h_ref = O.hgrn_scan(f, i, h0)
    np.testing.assert_allclose(h.cpu().numpy(), h_ref, rtol=RTOL32, atol=ATOL32)
    np.testing.assert_allclose(hl.cpu().numpy(), h_ref[:, -1], rtol=RTOL32, atol=ATOL32)


def test_scan_parity_bf16_strided(mmf):
    b, t, d = 2, 333, 256
    z = synth.activations(11, (b, t, 3 * d))
    z = _bf16_round(z)
    zt = _to(z, torch.bfloat16)
    zi_v, zf_v = zt[:, :, :d], zt[:, :, d:2 * d]
    h, hl = mmf.hgrn_scan(zf_v, zi_v, None, h_dtype=torch.bfloat16)
    _ok(mmf)
    f, i = O.hgrn_gates(z[:, :, d:2 * d], z[:, :, :d])
    h_ref = O.hgrn_scan(f, i)
    np.testing.assert_allclose(h.float().cpu().numpy(), h_ref, rtol=RTOL16, atol=RTOL16 * 0.1)


@pytest.mark.parametrize("b,t,d", [(2, 50, 33), (1, 300, 31), (2, 70, 34), (3, 129, 6)])
def test_scan_parity_unaligned_channels(mmf, b, t, d):
    # rows that are not 16-byte multiples take the three-pass kernels (paired for even d)
    zf, zi = synth.scan_inputs(b * t + d, b, t, d, False)
    h0 = synth.activations(5, (b, d))
    h, hl = mmf.hgrn_scan(_to(zf), _to(zi), _to(h0))
    _ok(mmf)
    h_ref = O.hgrn_scan(*O.hgrn_gates(zf, zi), h0)
    np.testing.assert_allclose(h.cpu().numpy(), h_ref, rtol=RTOL32, atol=ATOL32)
    np.testing.assert_allclose(hl.cpu().numpy(), h_ref[:, -1], rtol=RTOL32, atol=ATOL32)


def test_scan_parity_bf16_full_size(mmf):
    # the prefill step's scan: 8 sequences of 2048 steps, 1024 channels, gates read in place from
    # the [i | f | g] projection output (row stride 3d), float32 states; every element checked
    b, t, d = 8, 2048, 1024
    z = _bf16_round(synth.activations(17, (b, t, 3 * d)))
    z[:, :, d:2 * d] += 3.0  # forget gates near 0.95: long memory across chunks
    z = _bf16_round(z)
    zt = _to(z, torch.bfloat16)
    h0 = synth.activations(19, (b, d))
    h, hl = mmf.hgrn_scan(zt[:, :, d:2 * d], zt[:, :, :d], _to(h0), h_dtype=torch.float32)
    _ok(mmf)
    h_ref = O.hgrn_scan(*O.hgrn_gates(z[:, :, d:2 * d], z[:, :, :d]), h0)
    np.testing.assert_allclose(h.cpu().numpy(), h_ref, rtol=RTOL32, atol=ATOL32)
    np.testing.assert_allclose(hl.cpu().numpy(), h_ref[:, -1], rtol=RTOL32, atol=ATOL32)


def test_scan_long_sequence_closed_form(mmf):
    # constant gates: h_t = SiLU(zi) (1 - f^t); T = 65536 with f = sigmoid(4) checks carry drift
    b, t, d = 1, 65536, 64
    zf = np.full((b, t, d), 4.0, np.float32)
    zi = np.tile(np.linspace(-2, 2, d, dtype=np.float32), (b, t, 1))
    h, hl = mmf.hgrn_scan(_to(zf), _to(zi))
    _ok(mmf)
    f = 1 / (1 + np.exp(-4.0))
    silu = zi[0, 0].astype(np.float64) / (1 + np.exp(-zi[0, 0].astype(np.float64)))
    ts = np.array([1, 2, 10, 100, 1000, 30000, 65536])
    want = silu[None, :] * (1 - f ** ts[:, None])
    np.testing.assert_allclose(h[0, ts - 1].cpu().numpy(), want, rtol=RTOL32, atol=ATOL32)


def test_scan_empty_sequence_returns_h0(mmf):
    h0 = _to(synth.activations(3, (2, 64)))
    zf = torch.zeros(2, 0, 64, device=DEV)
    h, hl = mmf.hgrn_scan(zf, zf, h0)
    _ok(mmf)
    assert h.numel() == 0 and torch.equal(hl, h0)


# ---------------------------------------------------------------------------------------------
# block, decode, stack
# ---------------------------------------------------------------------------------------------
def _block_case(mmf, seed, d, inner, random_norms=True):
    shape = synth.BlockShape("case", d, inner, 1)
    params = synth.block_params(seed, shape, random_norms)
    return params, O.quantize_block(params), mmf.make_block(params, DEV)


@pytest.mark.parametrize("engine", ["auto", "tensor", "simt"])
def test_block_parity_tiny_config_f32(mmf, engine):
    # one HGRNBit block, fp32, d=256, I=704, x ~ N(0,1) [2, 128, 256]
    mmf.set_gemm_path({"auto": 0, "tensor": 1, "simt": 2}[engine])
    try:
        params, qp, blk = _block_case(mmf, 1, 256, 704, random_norms=False)
        x = synth.activations(2, (2, 128, 256))
        y, hl, taps = mmf.block_fwd_taps(blk, _to(x))
        y2, hl2 = mmf.block_fwd(blk, _to(x))
        _ok(mmf)
        fused = mmf.glu_fused(2 * 128, 704)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    assert fused == (engine != "simt")
    assert torch.equal(y, y2) and torch.equal(hl, hl2)   # taps variant runs the same path
    check_block_stages(x, qp, taps, y.cpu().numpy(), hl.cpu().numpy(), None, bf16=False, glu_fused=fused)
    y_ref, h_ref, inter = O.block_forward(x.astype(np.float64), qp)
    check_block_end_to_end(y.cpu().numpy(), y_ref, inter, qp, bf16=False, taps=taps, x=x)
    np.testing.assert_allclose(hl.cpu().numpy(), h_ref, rtol=RTOL32, atol=ATOL32 * 10)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_parity_ragged_with_state(mmf, dtype):
    bf16 = dtype == "bf16"
    params, qp, blk = _block_case(mmf, 3, 256, 704)
    x = synth.activations(4, (3, 37, 256))
    if bf16:
        x = _bf16_round(x)
    h0 = synth.activations(5, (3, 256))
    y, hl, taps = mmf.block_fwd_taps(blk, _to(x, torch.bfloat16 if bf16 else torch.float32), _to(h0))
    _ok(mmf)
    yg = _np(y)
    check_block_stages(x, qp, taps, yg, hl.cpu().numpy(), h0, bf16=bf16, glu_fused=mmf.glu_fused(3 * 37, 704))
    y_ref, h_ref, inter = O.block_forward(x.astype(np.float64), qp, h0)
    check_block_end_to_end(yg, y_ref, inter, qp, bf16=bf16, taps=taps, x=x)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_parity_inner_not_multiple_of_64(mmf, dtype):
    # I = 720 does not split into 64-row gate/up halves: gate_proj stores [gate | up] and the
    # GLU is formed by down_proj's norm kernel, on the tensor-core engine as well
    bf16 = dtype == "bf16"
    params, qp, blk = _block_case(mmf, 13, 256, 720)
    x = synth.activations(14, (2, 50, 256))
    if bf16:
        x = _bf16_round(x)
    assert not mmf.glu_fused(100, 720)
    y, hl, taps = mmf.block_fwd_taps(blk, _to(x, torch.bfloat16 if bf16 else torch.float32))
    _ok(mmf)
    yg = _np(y)
    check_block_stages(x, qp, taps, yg, hl.cpu().numpy(), None, bf16=bf16, glu_fused=False)
    y_ref, h_ref, inter = O.block_forward(x.astype(np.float64), qp)
    check_block_end_to_end(yg, y_ref, inter, qp, bf16=bf16, taps=taps, x=x)


def test_block_prefill_equals_stepwise_decode_on_gpu(mmf):
    params, qp, blk = _block_case(mmf, 6, 256, 704)
    params2, qp2, blk2 = _block_case(mmf, 7, 256, 704)
    x = synth.activations(8, (2, 12, 256))
    xt = _to(x)
    y1, h1 = mmf.block_fwd(blk, xt)
    y2, h2 = mmf.block_fwd(blk2, y1)
    state = torch.zeros(2, 2, 256, device=DEV)
    outs = []
    for t in range(12):
        outs.append(mmf.decode_step([blk, blk2], xt[:, t].contiguous(), state))
    _ok(mmf)
    yd = torch.stack(outs, 1).cpu().numpy()
    rel = np.linalg.norm(yd - y2.cpu().numpy()) / np.linalg.norm(y2.cpu().numpy())
    assert rel < 1e-3, rel
    np.testing.assert_allclose(state[0].cpu().numpy(), h1.cpu().numpy(), rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(state[1].cpu().numpy(), h2.cpu().numpy(), rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("b", [1, 2, 3, 4, 8, 64])
def test_decode_step_parity(mmf, b):
    # every stage of both layers against the oracle's definition on the kernel's own inputs to it
    # (elementwise), then the step end to end against the oracle's own chain
    layers = [_block_case(mmf, 20 + l, 256, 704) for l in range(2)]
    x = synth.activations(30 + b, (b, 256))
    state0 = synth.activations(31 + b, (2, b, 256)) * 0.5
    st = _to(state0)
    y, taps = mmf.decode_step_taps([c[2] for c in layers], _to(x), st)
    _ok(mmf)
    st_g = st.cpu().numpy()
    x_in = x.astype(np.float64)
    for l in range(2):
        x_in = check_decode_layer(x_in, state0[l], st_g[l], layers[l][1], taps[l], False, z_rounded=False)
    # end to end against the oracle's own two-layer chain: rows whose code decisions all match
    # the oracle's elementwise, every other row's first differing code a near-tie
    rel, frac = check_chain_end_to_end(x[:, None, :], [c[1] for c in layers], taps, _np(y), st_g,
                                       h0s=state0.astype(np.float64))
    print(f"decode d=256 b={b}: rel L2 y {rel:.3e}, clean rows {frac:.2f}")
    # the first layer's state depends only on exactly quantised inputs: elementwise
    y_ref, st_ref = O.decode_step(x.astype(np.float64), [c[1] for c in layers], state0.astype(np.float64))
    np.testing.assert_allclose(st_g[0], st_ref[0], rtol=RTOL32, atol=ATOL32)


@pytest.mark.parametrize("b", [1, 2, 4, 8])
def test_decode_fused_matches_unfused(mmf, b):
    # on the CUDA-core engine 1, 2, 4 or 8 rows take the fused four-launch decode (inputs staged
    # in shared memory up to two rows, read in place beyond; the automatic choice takes it for 1,
    # 2 and 4 rows); forcing the tensor-core engine takes the nine-launch block path instead. Same
    # quantisation arithmetic: states agree closely and the outputs within the chained-
    # quantisation tolerance.
    layers = [_block_case(mmf, 40 + l, 256, 704) for l in range(2)]
    x = _to(synth.activations(41 + b, (b, 256)))
    state0 = _to(synth.activations(42 + b, (2, b, 256)) * 0.5)
    st_f, st_u = state0.clone(), state0.clone()
    try:
        mmf.set_gemm_path(mmf.MMF_GEMM_SIMT)
        y_f = mmf.decode_step([c[2] for c in layers], x, st_f)
        mmf.set_gemm_path(mmf.MMF_GEMM_TENSOR)
        y_u = mmf.decode_step([c[2] for c in layers], x, st_u)
        _ok(mmf)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    np.testing.assert_allclose(st_f[0].cpu().numpy(), st_u[0].cpu().numpy(), rtol=RTOL32, atol=ATOL32)
    rel = float(torch.linalg.norm(y_f - y_u) / torch.linalg.norm(y_u))
    assert rel < 1e-3, rel


def test_decode_wait_cap_ends_and_recovers(mmf):
    # with a 1 us cap on every in-kernel wait the fused decode's waits for its bulk copies run
    # out: every launch must still end (the CTA drains its copies and leaves as a whole), report
    # MMF_ERR_TIMEOUT (or, if no wait ran out, be right), and leave the context usable for the
    # next step at the default cap
    layers = [_block_case(mmf, 70 + l, 256, 704) for l in range(2)]
    blocks = [c[2] for c in layers]
    x = _to(synth.activations(71, (1, 256)))
    state0 = _to(synth.activations(72, (2, 1, 256)) * 0.5)
    y_ref, st_ref = O.decode_step(_np(x).astype(np.float64), [c[1] for c in layers], _np(state0).astype(np.float64))
    st = state0.clone()
    mmf.set_wait_limit(1)
    try:
        y = mmf.decode_step(blocks, x, st)
        status = mmf.sync_status(DEV)
    finally:
        mmf.set_wait_limit(0)
    assert status in (mmf.MMF_OK, mmf.MMF_ERR_TIMEOUT)
    if status == mmf.MMF_OK:
        assert np.linalg.norm(_np(y) - y_ref) / np.linalg.norm(y_ref) < 1e-3
    st = state0.clone()
    y = mmf.decode_step(blocks, x, st)
    _ok(mmf)
    assert np.linalg.norm(_np(y) - y_ref) / np.linalg.norm(y_ref) < 1e-3
    np.testing.assert_allclose(_np(st)[0], st_ref[0], rtol=RTOL32, atol=ATOL32)


def test_gemm_wait_cap_ends_and_recovers(mmf):
    # the tensor-core GEMM under a 1 us cap on every in-kernel wait: the launch must end (each CTA
    # drains its TMA copies and MMAs, releases its tensor memory and leaves), report
    # MMF_ERR_TIMEOUT (or, if no wait ran out, be right), and the next call at the default cap must
    # be right
    m, n, k = 512, 2048, 2048
    x = _to(synth.activations(120, (m, k)))
    W = synth.weight(121, n, k)
    pt = mmf.pack_ternary(_to(W))
    _ok(mmf)
    mmf.set_gemm_path(mmf.MMF_GEMM_TENSOR)
    try:
        mmf.set_wait_limit(1)
        try:
            y, q, deq, acc = mmf.bitlinear_fwd(x, None, pt, debug=True)
            status = mmf.sync_status(DEV)
        finally:
            mmf.set_wait_limit(0)
        assert status in (mmf.MMF_OK, mmf.MMF_ERR_TIMEOUT)
        t, s = O.ternarize(W)
        if status == mmf.MMF_OK:
            assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_matmul(q.cpu().numpy(), t))
        y, q, deq, acc = mmf.bitlinear_fwd(x, None, pt, debug=True)
        _ok(mmf)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_matmul(q.cpu().numpy(), t))


def test_backward_products_wait_cap_ends_and_recovers(mmf):
    # the BitLinear backward's bf16 tensor-core products under a 1 us cap on every in-kernel wait:
    # the launches must end (each CTA drains its TMA copies and MMAs, releases its tensor memory and
    # leaves), report MMF_ERR_TIMEOUT (or, if no wait ran out, be right), and the next call at the
    # default cap must be right
    m, n, k = 512, 512, 1024
    x = _to(synth.activations(140, (m, k)))
    Wl = synth.weight(141, n, k)
    w = mmf.pack_ternary(_to(Wl))
    dy = _to(synth.activations(142, (m, n)))
    _, q, deq, _ = mmf.bitlinear_fwd(x, None, w, y_dtype=torch.float32, debug=True)
    _ok(mmf)
    dW_ref = _np(dy).astype(np.float64).T @ (q.cpu().numpy().astype(np.float64) * deq.cpu().numpy()[:, None])
    scale = np.abs(dW_ref).max()
    mmf.set_gemm_path(mmf.MMF_GEMM_TENSOR)
    try:
        mmf.set_wait_limit(1)
        try:
            dx, dnw, dW = mmf.bitlinear_backward(x, None, w, q, deq, dy)
            status = mmf.sync_status(DEV)
        finally:
            mmf.set_wait_limit(0)
        assert status in (mmf.MMF_OK, mmf.MMF_ERR_TIMEOUT)
        if status == mmf.MMF_OK:
            np.testing.assert_allclose(dW.cpu().numpy(), dW_ref, rtol=1e-4, atol=1e-4 * scale)
        dx, dnw, dW = mmf.bitlinear_backward(x, None, w, q, deq, dy)
        _ok(mmf)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    np.testing.assert_allclose(dW.cpu().numpy(), dW_ref, rtol=1e-4, atol=1e-4 * scale)


def test_head_wait_cap_ends_and_recovers(mmf):
    # the tensor-core head under a 1 us cap: ends, reports MMF_ERR_TIMEOUT or is right, and the
    # next call at the default cap is right
    b, d, vocab = 8, 2560, 32000
    x = _to(synth.activations(130, (b, d)), torch.bfloat16)
    table = _to(synth.embedding(131, vocab, d), torch.bfloat16)
    ref = O.lm_head_logits(_np(x).astype(np.float64), None, _np(table).astype(np.float64))
    mmf.set_wait_limit(1)
    try:
        ids, logits = mmf.lm_head_argmax(x, None, table, want_logits=True)
        status = mmf.sync_status(DEV)
    finally:
        mmf.set_wait_limit(0)
    assert status in (mmf.MMF_OK, mmf.MMF_ERR_TIMEOUT)
    scale = np.abs(ref).max()
    if status == mmf.MMF_OK:
        np.testing.assert_allclose(logits.cpu().numpy(), ref, rtol=1e-4, atol=1e-4 * scale)
    ids, logits = mmf.lm_head_argmax(x, None, table, want_logits=True)
    _ok(mmf)
    np.testing.assert_allclose(logits.cpu().numpy(), ref, rtol=1e-4, atol=1e-4 * scale)


def test_decode_skinny_wait_cap_ends_and_recovers(mmf):
    # the skinny tensor-core decode (8 rows: cluster split-K products and row stages) under a 1 us
    # cap on every in-kernel wait: every launch ends (an abandoned CTA still joins its cluster's
    # barriers), the step reports MMF_ERR_TIMEOUT or is right, and the next step at the default
    # cap is right
    layers = [_block_case(mmf, 75 + l, 256, 704) for l in range(2)]
    blocks = [c[2] for c in layers]
    x = _to(synth.activations(76, (8, 256)))
    state0 = _to(synth.activations(77, (2, 8, 256)) * 0.5)
    y_ref, st_ref = O.decode_step(_np(x).astype(np.float64), [c[1] for c in layers], _np(state0).astype(np.float64))
    mmf.set_decode_path(mmf.MMF_DECODE_SKINNY)
    try:
        st = state0.clone()
        mmf.set_wait_limit(1)
        try:
            y = mmf.decode_step(blocks, x, st)
            status = mmf.sync_status(DEV)
        finally:
            mmf.set_wait_limit(0)
        assert status in (mmf.MMF_OK, mmf.MMF_ERR_TIMEOUT)
        if status == mmf.MMF_OK:
            assert np.linalg.norm(_np(y) - y_ref) / np.linalg.norm(y_ref) < 1e-3
        st = state0.clone()
        y = mmf.decode_step(blocks, x, st)
        _ok(mmf)
    finally:
        mmf.set_decode_path(mmf.MMF_DECODE_AUTO)
    assert np.linalg.norm(_np(y) - y_ref) / np.linalg.norm(y_ref) < 1e-3
    np.testing.assert_allclose(_np(st)[0], st_ref[0], rtol=RTOL32, atol=ATOL32)


# CUDA-core form: float32 table, or one row; tensor-core form: bf16 table and b >= 2 (ragged d and
# vocabulary tails, two passes at b = 130)
@pytest.mark.parametrize("b,d,vocab,xdt,tdt", [(1, 256, 1000, "f32", "f32"), (5, 264, 900, "bf16", "f32"),
                                                (1, 2560, 32000, "bf16", "bf16"), (2, 256, 777, "bf16", "bf16"),
                                                (11, 264, 1200, "f32", "bf16"), (8, 2560, 32000, "bf16", "bf16"),
                                                (64, 2560, 32000, "bf16", "bf16"), (130, 200, 1000, "bf16", "bf16")])
def test_lm_head_argmax_parity(mmf, b, d, vocab, xdt, tdt):
    # final RMSNorm + tied head + greedy next token against the oracle on the same (dtype-
    # rounded) inputs: logits within 1e-4 (float32 accumulation of d products; the tensor-core
    # form's bf16 hi + lo split of the normalised rows adds ~2^-17 relative); the ids are the
    # first argmax of the kernel's own logits, and the oracle's argmax except at near-ties
    dts = {"f32": torch.float32, "bf16": torch.bfloat16}
    x = _to(synth.activations(80 + b, (b, d)), dts[xdt])
    w = synth.norm_weight(81, d, random=True)
    table = _to(synth.embedding(82, vocab, d), dts[tdt])
    ids, logits = mmf.lm_head_argmax(x, _to(w), table, want_logits=True)
    ids2 = mmf.lm_head_argmax(x, _to(w), table)
    _ok(mmf)
    lg = logits.cpu().numpy()
    ref = O.lm_head_logits(_np(x).astype(np.float64), w, _np(table).astype(np.float64))
    scale = np.abs(ref).max()
    np.testing.assert_allclose(lg, ref, rtol=1e-4, atol=1e-4 * scale)
    got = ids.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, ids2.cpu().numpy())
    assert np.array_equal(got, np.argmax(lg, axis=1))
    want = O.greedy_next(ref)
    for r in np.nonzero(got != want)[0]:
        assert ref[r, got[r]] >= ref[r].max() - 2e-4 * scale  # a near-tie


def test_embed_gather(mmf):
    table = synth.embedding(50, 1000, 256)
    ids = synth.token_ids(51, (3, 17), vocab=1000)
    ids[0, 0] = -1
    ids[2, 5] = 1000
    out = mmf.embed_gather(_to(ids, torch.int32), _to(table))
    _ok(mmf)
    o = out.cpu().numpy()
    ok = (ids >= 0) & (ids < 1000)
    assert np.array_equal(o[ok], table[ids[ok]])
    assert np.all(o[~ok] == 0)


def test_stack_parity_two_layers(mmf):
    layers = [_block_case(mmf, 60 + l, 256, 704) for l in range(2)]
    table = synth.embedding(62, 500, 256)
    ids = synth.token_ids(63, (2, 50), vocab=500)
    y, hl = mmf.stack_fwd([c[2] for c in layers], _to(ids, torch.int32), _to(table), want_state=True)
    _ok(mmf)
    # the stack is the embedding gather followed by the block forward of each layer: same kernels,
    # same inputs, so it reproduces the per-layer calls bit for bit (each block is checked against
    # the oracle stage by stage above)
    x0 = mmf.embed_gather(_to(ids, torch.int32), _to(table))
    y1, h1 = mmf.block_fwd(layers[0][2], x0)
    y2, h2 = mmf.block_fwd(layers[1][2], y1)
    _ok(mmf)
    assert torch.equal(y, y2) and torch.equal(hl[0], h1) and torch.equal(hl[1], h2)
    # every stage of each layer against the oracle on the kernel's own inputs to it (elementwise)
    x_in = x0
    tap_list = []
    for l in range(2):
        yl, hll, taps = mmf.block_fwd_taps(layers[l][2], x_in)
        _ok(mmf)
        check_block_stages(_np(x_in), layers[l][1], taps, _np(yl), hll.cpu().numpy(), None, bf16=False,
                           glu_fused=mmf.glu_fused(100, 704))
        tap_list.append(taps)
        x_in = yl
    # end to end against the oracle's own chain: every divergence starts at a near-tie code (the
    # second layer's first quantisation is a chained one, and the recurrence carries a change to
    # later tokens), rows without one elementwise
    x_emb = O.embed(ids, table)
    rel, frac = check_chain_end_to_end(x_emb, [c[1] for c in layers], tap_list, _np(y), hl.cpu().numpy())
    print(f"stack two layers d=256: rel L2 y {rel:.3e}, clean rows {frac:.2f}")
    y_ref, st_ref = O.stack_forward(ids, table, [c[1] for c in layers])
    # first layer: exactly quantised inputs, so its state matches elementwise
    np.testing.assert_allclose(hl.cpu().numpy()[0], st_ref[0], rtol=RTOL32, atol=ATOL32)


# HGRN2 state expansion against the oracle's step-by-step recurrence: ragged dk and dv (padding
# rows and partial column blocks), long and empty sequences, a carried state. float32: outputs
# within 1e-4 of the largest (float32 state over up to 300 steps); bf16: the same on inputs
# rounded to bf16, with the bf16 rounding of the output (2^-9 relative) inside 1e-2.
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("b,t,heads,dk,dv", [(2, 50, 3, 40, 33), (1, 300, 2, 128, 130), (3, 17, 1, 16, 8),
                                             (1, 0, 2, 8, 5)])
def test_hgrn2_recurrence_parity(mmf, dt, b, t, heads, dk, dv):
    dts = {"f32": torch.float32, "bf16": torch.bfloat16}
    q = _to(synth.activations(90, (b, t, heads, dk)), dts[dt])
    f = _to(O.sigmoid(synth.activations(91, (b, t, heads, dk)) + 2.0), dts[dt])
    i = _to(synth.activations(92, (b, t, heads, dv)), dts[dt])
    s0 = _to(synth.activations(93, (b, heads, dk, dv)) * 0.5)
    o, s = mmf.hgrn2_recurrence(q, f, i, s0, want_state=True)
    _ok(mmf)
    o_ref, s_ref = O.hgrn2_recurrence(_np(q).astype(np.float64), _np(f).astype(np.float64),
                                      _np(i).astype(np.float64), _np(s0).astype(np.float64))
    tol = 1e-4 if dt == "f32" else 1e-2
    if t:
        np.testing.assert_allclose(_np(o), o_ref, rtol=tol, atol=tol * np.abs(o_ref).max())
    np.testing.assert_allclose(_np(s), s_ref, rtol=1e-4, atol=1e-4 * np.abs(s_ref).max())


# Gradients of the scan with its gates against the oracle's chain (gates -> scan backward -> gate
# backward) on the oracle's own forward states, rounded to the kernel's dtype; one chunk (up to 32
# steps), two chunks with a ragged last one, many chunks (700 steps, and 5000 steps in chunks of
# 48), odd d (one channel per thread) and even d (channel pairs), a carried initial state, long
# memory, an empty sequence. float32 within 1e-4 of the largest gradient (float32 accumulation
# over up to 5000 steps of G); bf16 inputs, states and outputs within 2e-2.
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("b,t,d,long_memory", [(2, 37, 100, False), (1, 700, 64, True), (2, 0, 16, False),
                                               (3, 20, 6, False), (3, 33, 7, True), (1, 5000, 10, True)])
def test_scan_backward_parity(mmf, dt, b, t, d, long_memory):
    dts = {"f32": torch.float32, "bf16": torch.bfloat16}
    zf, zi = synth.scan_inputs(95, b, t, d, long_memory)
    zf_g, zi_g = _to(zf, dts[dt]), _to(zi, dts[dt])
    zf64, zi64 = _np(zf_g).astype(np.float64), _np(zi_g).astype(np.float64)
    h0 = synth.activations(96, (b, d)) * 0.5
    f, i = O.hgrn_gates(zf64, zi64)
    h = O.hgrn_scan(f, i, h0)
    dh = synth.activations(97, (b, t, d))
    h_g, dh_g = _to(h, dts[dt]), _to(dh, dts[dt])
    dzf, dzi, dh0 = mmf.hgrn_scan_backward(zf_g, zi_g, h_g, dh_g, _to(h0))
    _ok(mmf)
    df, di, dh0_ref = O.hgrn_scan_backward(f, i, _np(dh_g).astype(np.float64), h0)
    dzf_ref, dzi_ref = O.hgrn_gates_backward(zf64, zi64, df, di)
    tol = 1e-4 if dt == "f32" else 2e-2
    if t:
        np.testing.assert_allclose(_np(dzf), dzf_ref, rtol=tol, atol=tol * np.abs(dzf_ref).max())
        np.testing.assert_allclose(_np(dzi), dzi_ref, rtol=tol, atol=tol * np.abs(dzi_ref).max())
    np.testing.assert_allclose(dh0.cpu().numpy(), dh0_ref, rtol=tol, atol=tol * max(np.abs(dh0_ref).max(), 1e-30))


# BitLinear gradients with the straight-through estimator against the oracle, on the forward's own
# activation codes (the kernel backward takes them from mmf_bitlinear_fwd, whose codes the forward
# parity tests check against the oracle's): dx and the gain's gradient against the oracle's RMSNorm
# backward of dr = dy (t s), dW against dy^T (q a/127) with the forward's q and a/127. On the
# tensor cores dy enters as bf16 hi / lo pairs (about 2^-17 relative per term) and the codes are
# exact; on the CUDA cores everything is float32. float32 accumulation over n (dr) or m (dW):
# within 1e-4 of the largest value either way. Shapes: ragged n and k (scalar epilogue stores,
# split dy rows), n a multiple of 8 (bf16 dy used in place), m large enough for a K split of dW
# (the partials added by the reduction kernel), m = 0.
@pytest.mark.parametrize("engine", ["tensor", "simt"])
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
@pytest.mark.parametrize("m,n,k", [(5, 33, 200), (64, 128, 256), (0, 16, 64), (300, 640, 1024), (2000, 72, 88)])
def test_bitlinear_backward_parity(mmf, engine, xdt, m, n, k):
    dts = {"f32": torch.float32, "bf16": torch.bfloat16}
    x = _to(synth.activations(100, (m, k)), dts[xdt])
    nw = synth.norm_weight(101, k, random=True)
    Wl = synth.weight(102, n, k)
    w = mmf.pack_ternary(_to(Wl))
    dy = _to(synth.activations(103, (m, n)), dts[xdt])
    _, q, deq, _ = mmf.bitlinear_fwd(x, _to(nw), w, y_dtype=torch.float32, debug=True)
    mmf.set_gemm_path(mmf.MMF_GEMM_SIMT if engine == "simt" else mmf.MMF_GEMM_TENSOR)
    try:
        dx, dnw, dW = mmf.bitlinear_backward(x, _to(nw), w, q, deq, dy)
        _ok(mmf)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)
    t, s = O.ternarize(Wl)
    x64, dy64 = _np(x).astype(np.float64), _np(dy).astype(np.float64)
    dr = dy64 @ (t.astype(np.float64) * float(s))
    dx_ref, dnw_ref = O.rmsnorm_backward(x64, nw, dr)
    dW_ref = dy64.T @ (q.cpu().numpy().astype(np.float64) * deq.cpu().numpy().astype(np.float64)[:, None])
    if m:
        np.testing.assert_allclose(dx.cpu().numpy(), dx_ref, rtol=1e-4, atol=1e-4 * np.abs(dx_ref).max())
    scale_nw = max(np.abs(dnw_ref).max(), 1e-30)
    np.testing.assert_allclose(dnw.cpu().numpy(), dnw_ref, rtol=1e-4, atol=1e-4 * scale_nw)
    scale_w = max(np.abs(dW_ref).max(), 1e-30)
    np.testing.assert_allclose(dW.cpu().numpy(), dW_ref, rtol=1e-4, atol=1e-4 * scale_w)


# The packed-code integrity check: a freshly packed matrix (ragged k, so the last word of each row
# has padding fields) has no malformed field; a planted 10 field in the codes and a nonzero padding
# field are each counted once (positions from the oracle's bit layout).
def test_validate_packed_counts_planted_faults(mmf):
    n, k = 9, 70
    w = mmf.pack_ternary(_to(synth.weight(110, n, k)))
    assert mmf.validate_packed(w) == 0
    codes = w.codes.clone()
    w2 = mmf.PackedTernary(codes, w.scale, n, k)

    def plant(row, col, field):
        b = O.code_bit(col % 16)
        word = int(codes[row, col // 16].item()) & 0xFFFFFFFF
        word = (word & ~(3 << b)) | (field << b)
        codes[row, col // 16] = word - (1 << 32) if word >= 1 << 31 else word

    plant(3, 5, 0b10)    # real column: the unused pattern 10
    assert mmf.validate_packed(w2) == 1
    plant(7, 75, 0b01)   # padding column (k = 70) holding +1
    assert mmf.validate_packed(w2) == 2
    plant(8, 77, 0b10)   # padding column holding 10: one malformed field, counted once
    assert mmf.validate_packed(w2) == 3
    assert mmf.validate_packed(w2) == O.count_malformed_fields(codes.cpu().numpy().view(np.uint32), k)
    # random corruption of a larger matrix against the oracle's definition of the count
    n, k = 300, 1000
    w = mmf.pack_ternary(_to(synth.weight(111, n, k)))
    words = w.codes.cpu().numpy().view(np.uint32).copy()
    g = np.random.default_rng(112)
    for _ in range(40):
        r, c = int(g.integers(0, n)), int(g.integers(0, words.shape[1] * 16))
        b = O.code_bit(c % 16)
        words[r, c // 16] = (words[r, c // 16] & ~np.uint32(3 << b)) | np.uint32(int(g.integers(0, 4)) << b)
    w3 = mmf.PackedTernary(_to(words.view(np.int32), torch.int32), w.scale, n, k)
    assert mmf.validate_packed(w3) == O.count_malformed_fields(words, k) > 0
