"""The allocation-free BitLinear entry point (mmf_bitlinear_fwd_noalloc).

It exists for callers that cannot allocate device memory or pass a workspace (a custom-op
interface that only hands over inputs and outputs, a runtime whose memory pool owns the device,
a loop where cudaMalloc's implicit synchronisation is not allowed). Its scratch is a static
device array inside the library. These tests call it through the C ABI, twice in a row with
different shapes and dtypes (so the second call runs over the first one's leftovers in the
shared array), and compare each result with the workspace entry point mmf_bitlinear_fwd on the
same inputs, within the float32 tolerance the parity tests use. The file is named to be
collected last; it passes on its own in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
RTOL, ATOL = 1e-3, 1e-5


@pytest.fixture(scope="module")
def mmf():
    import ternary_weight_matmul_b200 as m
    from ternary_weight_matmul_b200 import build
    build.build()
    m.lib()
    torch.cuda.set_device(0)
    return m


def _noalloc(mmf, x, norm_w, w, y_dtype):
    L = mmf.lib()
    m = x.numel() // w.k
    y = torch.empty(m, w.n, dtype=y_dtype, device=DEV)
    tw = w.c()
    st = L.mmf_bitlinear_fwd_noalloc(x.data_ptr(), mmf._dt(x.dtype), m, norm_w.data_ptr() if norm_w is not None else None,
                                     ctypes.byref(tw), y.data_ptr(), mmf._dt(y_dtype),
                                     torch.cuda.current_stream().cuda_stream)
    assert st == mmf.MMF_OK, L.mmf_last_error()
    return y


@pytest.mark.parametrize("engine", ["auto", "tensor", "simt"])
def test_noalloc_matches_workspace_entry_point_twice_in_a_row(mmf, engine):
    mmf.set_gemm_path({"auto": mmf.MMF_GEMM_AUTO, "tensor": mmf.MMF_GEMM_TENSOR, "simt": mmf.MMF_GEMM_SIMT}[engine])
    try:
        cases = [(300, 640, 1024, torch.float32), (77, 256, 704, torch.bfloat16)]
        for i, (m, n, k, xdt) in enumerate(cases):
            x = torch.from_numpy(synth.activations(900 + i, (m, k))).to(DEV, xdt)
            nw = torch.from_numpy(synth.norm_weight(910 + i, k, random=True)).to(DEV)
            w = mmf.pack_ternary(torch.from_numpy(synth.weight(920 + i, n, k)).to(DEV))
            y_na = _noalloc(mmf, x, nw, w, torch.float32)
            y_ws = mmf.bitlinear_fwd(x, nw, w, y_dtype=torch.float32)
            assert mmf.sync_status(DEV) == mmf.MMF_OK
            np.testing.assert_allclose(y_na.cpu().numpy(), y_ws.cpu().numpy(), rtol=RTOL, atol=ATOL)
    finally:
        mmf.set_gemm_path(mmf.MMF_GEMM_AUTO)


def test_noalloc_rejects_requests_beyond_the_static_array(mmf):
    L = mmf.lib()
    k, n = 2048, 64
    w = mmf.pack_ternary(torch.from_numpy(synth.weight(930, n, k)).to(DEV))
    m = mmf.NOALLOC_SCRATCH_BYTES // k + 1  # int8 codes alone exceed the array
    tw = w.c()
    st = L.mmf_bitlinear_fwd_noalloc(None, mmf.MMF_F32, m, None, ctypes.byref(tw), None, mmf.MMF_F32, None)
    assert st == mmf.MMF_ERR_WORKSPACE
    assert b"static array" in L.mmf_last_error()
    assert mmf.sync_status(DEV) == mmf.MMF_OK
