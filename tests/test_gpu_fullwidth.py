"""GPU parity at the model widths the measurements run (the pages' model table: 370M d 1024 /
I 2816, 1.3B d 2048 / I 5632, 2.7B d 2560 / I 7040), through the C ABI.

* Decode: two layers of the 2.7B width at batch 1 to 64 on each decode path (the fused CUDA-core
  launches, the skinny tensor-core products with their row stages, the block path), float32 and
  bf16: every stage of every layer against the oracle's definition
  applied to the kernel's own inputs to that stage (mmf_decode_step_taps), the second layer fed
  the first layer's output as the kernels produced it; then the whole step against the oracle's
  own two-layer step.
* Block: mmf_block_fwd_taps at the 370M and 1.3B widths on a few hundred tokens, stage by stage,
  then end to end.

End to end, the oracle's own chain differs from the kernels' only where a float32 code decision
sits at a near-tie (both sides decide in float32, so only a value within rounding of a
half-integer can round the other way); after such a flip the row's later
quantisations see different inputs and differ in numbers. In float32 the end-to-end check follows
every row's chain of code decisions: the first difference must be a near-tie, and rows without one
match elementwise. In bf16 the kernels store every intermediate in bf16 and the oracle
none, so end to end only a sanity bound holds; the stage checks carry the elementwise claim.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_checks import _np, check_block_end_to_end, check_block_stages, check_chain_end_to_end, check_decode_layer

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def mmf():
    import ternary_weight_matmul_b200 as m
    from ternary_weight_matmul_b200 import build
    build.build()
    m.lib()
    torch.cuda.set_device(0)
    m.set_gemm_path(m.MMF_GEMM_AUTO)
    yield m
    m.set_gemm_path(m.MMF_GEMM_AUTO)


def _to(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV, dtype)


def _ok(mmf):
    assert mmf.sync_status(DEV) == 0


def _bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


_LAYERS = {}


def _layers(mmf, d, inner, n, seed):
    key = (d, inner, n, seed)
    if key not in _LAYERS:
        out = []
        for l in range(n):
            params = synth.block_params(seed + l, synth.BlockShape("w", d, inner, 1), True)
            out.append((O.quantize_block(params), mmf.make_block(params, DEV)))
        _LAYERS[key] = out
    return _LAYERS[key]


PATHS = {"auto": 0, "fused": 1, "skinny": 2, "block": 3}
DECODE_CASES = [(1, "f32", "auto"), (1, "bf16", "auto"), (2, "f32", "auto"), (4, "bf16", "auto"), (8, "f32", "auto"),
                (64, "f32", "auto"), (1, "f32", "skinny"), (3, "bf16", "skinny"), (17, "f32", "skinny"),
                (33, "bf16", "skinny"), (8, "bf16", "block"), (64, "f32", "block")]


@pytest.mark.parametrize("b,dtype,path", DECODE_CASES)
def test_decode_step_full_width_stages(mmf, b, dtype, path):
    d, inner = 2560, 7040
    bf16 = dtype == "bf16"
    tdt = torch.bfloat16 if bf16 else torch.float32
    layers = _layers(mmf, d, inner, 2, 500)
    x = synth.activations(510 + b, (b, d))
    if bf16:
        x = _bf16_round(x)
    state0 = synth.activations(511 + b, (2, b, d)) * 0.5
    mmf.set_decode_path(PATHS[path])
    try:
        taken = mmf.decode_path(b, d, inner)
        st = _to(state0)
        y, taps = mmf.decode_step_taps([c[1] for c in layers], _to(x, tdt), st)
        _ok(mmf)
        # the step without taps runs the same kernels: bit-identical output and state
        st2 = _to(state0)
        y2 = mmf.decode_step([c[1] for c in layers], _to(x, tdt), st2)
        _ok(mmf)
    finally:
        mmf.set_decode_path(mmf.MMF_DECODE_AUTO)
    if path == "auto":
        assert taken == (mmf.MMF_DECODE_FUSED if b in (1, 2) else mmf.MMF_DECODE_SKINNY)
    else:
        assert taken == PATHS[path]
    assert torch.equal(y, y2) and torch.equal(st, st2)
    st_g = st.cpu().numpy()
    x_in = x.astype(np.float64)
    for l, (qp, _) in enumerate(layers):
        # the block path stores z and h in the activation dtype; the others keep them in float32
        y_l = check_decode_layer(x_in, state0[l], st_g[l], qp, taps[l], bf16,
                                 z_rounded=bf16 and taken == mmf.MMF_DECODE_BLOCK)
        x_in = y_l
    assert np.array_equal(_np(taps[-1]["y"]), _np(y))
    # end to end against the oracle's own two-layer step. float32: rows whose code decisions all
    # match the oracle's elementwise (output and both states), every other row's first differing
    # code a near-tie. bf16: the kernels store every intermediate in bf16 and the oracle none, so
    # the whole-output error is reported under a sanity bound (the stages above carry the claim)
    if bf16:
        y_ref, _ = O.decode_step(x.astype(np.float64), [c[0] for c in layers], state0.astype(np.float64))
        rel = np.linalg.norm(_np(y) - y_ref) / np.linalg.norm(y_ref)
        assert rel < 5e-2 * np.sqrt(2), rel
        frac = float("nan")
    else:
        rel, frac = check_chain_end_to_end(x[:, None, :], [c[0] for c in layers], taps, _np(y), st_g,
                                           h0s=state0.astype(np.float64))
    print(f"decode full width b={b} {dtype} path={taken}: rel L2 y {rel:.3e}, clean rows {frac:.2f}")


@pytest.mark.parametrize("d,inner,b,t,dtype", [(1024, 2816, 2, 96, "f32"), (1024, 2816, 2, 96, "bf16"),
                                               (2048, 5632, 1, 160, "bf16")])
def test_block_full_width_stages(mmf, d, inner, b, t, dtype):
    bf16 = dtype == "bf16"
    qp, blk = _layers(mmf, d, inner, 1, 600 + d)[0]
    x = synth.activations(601 + d, (b, t, d))
    if bf16:
        x = _bf16_round(x)
    h0 = synth.activations(602 + d, (b, d)) * 0.5
    y, hl, taps = mmf.block_fwd_taps(blk, _to(x, torch.bfloat16 if bf16 else torch.float32), _to(h0))
    _ok(mmf)
    assert mmf.glu_fused(b * t, inner)
    yg = _np(y)
    check_block_stages(x, qp, taps, yg, hl.cpu().numpy(), h0, bf16=bf16, glu_fused=True)
    y_ref, h_ref, inter = O.block_forward(x.astype(np.float64), qp, h0)
    rel, clean = check_block_end_to_end(yg, y_ref, inter, qp, bf16=bf16, taps=taps, x=x)
    frac = float("nan") if clean is None else float(clean.mean())
    print(f"block full width d={d} I={inner} {b}x{t} {dtype}: rel L2 y {rel:.3e}, clean rows {frac:.2f}")
