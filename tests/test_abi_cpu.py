"""Host-side checks of the C ABI that need no GPU: the library loads, exports every symbol
include/mmf.h declares, reports sizes, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import ternary_weight_matmul_b200 as mmf
from ternary_weight_matmul_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mmf.h")


@pytest.fixture(scope="module")
def L():
    mbuild.build()
    return mmf.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mmf_[a-z_0-9]+)\s*\(", text)))


def test_header_declarations_exported(L):
    names = _declared()
    assert len(names) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", mbuild.OUT], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (mmf_[a-z_0-9]+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(names) == set(mmf.EXPORTED)
    for n in names:
        assert getattr(L, n) is not None


def test_sizes(L):
    for k, w in [(1, 4), (16, 4), (63, 4), (64, 4), (65, 8), (256, 16), (704, 44), (7040, 440)]:
        assert L.mmf_packed_row_words(k) == w
    assert L.mmf_packed_words(3, 65) == 24
    assert L.mmf_packed_words(0, 65) == 0
    assert L.mmf_workspace_bytes(mmf.MMF_OP_PACK, 10, 0, 0, 0) >= 296 * 8
    b1 = L.mmf_workspace_bytes(mmf.MMF_OP_BLOCK, 256, 256, 704, 1)
    b2 = L.mmf_workspace_bytes(mmf.MMF_OP_BLOCK, 512, 256, 704, 1)
    assert 0 < b1 < b2
    assert L.mmf_workspace_bytes(mmf.MMF_OP_STACK, 256, 256, 704, 2) > b1
    assert L.mmf_workspace_bytes(mmf.MMF_OP_BITLINEAR, 5, 100, 7, 0) >= 5 * 128 + 5 * 4
    # chunked scan: three float arrays of b * nchunk * d with b * nchunk <= ceil(m / 8)
    assert L.mmf_workspace_bytes(mmf.MMF_OP_SCAN, 8 * 2048, 1024, 0, 0) >= 3 * 1024 * 4 * 8 * 128


def test_status_strings(L):
    for s in range(6):
        assert L.mmf_status_string(s)
    assert L.mmf_status_string(99) == b"unknown status"


def test_invalid_arguments_rejected_on_host(L):
    # every one of these fails validation before any CUDA call
    assert L.mmf_pack_ternary(None, 0, 4, 4, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_pack_ternary(None, 7, 4, 4, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_pack_ternary(None, 0, 0, 4, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert b"pack" in L.mmf_last_error()
    t = mmf.Ternary(None, None, 8, 16)
    assert L.mmf_bitlinear_fwd(None, 0, 4, None, ctypes.byref(t), None, 0, None, None, None, None, 0,
                               None) == mmf.MMF_ERR_INVALID_ARG
    t = mmf.Ternary(16, 32, 8, 16)  # misaligned codes pointer (16 is aligned; 20 is not)
    t.codes = 20
    assert L.mmf_bitlinear_fwd(None, 0, 4, None, ctypes.byref(t), None, 0, None, None, None, None, 0,
                               None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_hgrn_scan(None, None, 0, 2, 1, 4, 4, None, None, 0, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_hgrn_scan(None, None, 5, 4, 1, 4, 4, None, None, 0, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    # a long sequence needs scratch: too little is reported before anything runs
    assert L.mmf_hgrn_scan(16, 16, 0, 4, 1, 1000, 4, None, 16, 0, None, None, 0, None) == mmf.MMF_ERR_WORKSPACE
    bw = mmf.BlockWeightsC(d=0, inner=4)
    assert L.mmf_block_fwd(ctypes.byref(bw), None, 0, 1, 1, None, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_decode_step(None, 0, None, 0, 1, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_stack_fwd(None, 0, None, 1, 1, None, 10, 0, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_embed_gather(None, 4, None, 0, 0, 4, None, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_set_gemm_path(9) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_set_gemm_path(mmf.MMF_GEMM_AUTO) == mmf.MMF_OK
    assert L.mmf_set_wait_limit(0) == mmf.MMF_OK


def test_head_arguments_and_workspace_on_host(L):
    # mmf_lm_head_argmax(x, x_dtype, b, d, norm_w, eps, table, table_dtype, vocab, ids, logits, ws,
    # ws_bytes, stream): validation, alignment and workspace size are checked before any CUDA call
    head = L.mmf_lm_head_argmax
    assert head(16, 0, 2, 12, None, 1e-8, 16, 1, 100, 16, None, 16, 1 << 30, None) == mmf.MMF_ERR_INVALID_ARG  # d % 8
    assert head(16, 0, 2, 16, None, 1e-8, 16, 1, 0, 16, None, 16, 1 << 30, None) == mmf.MMF_ERR_INVALID_ARG  # vocab
    assert head(None, 0, 2, 16, None, 1e-8, 16, 1, 100, 16, None, 16, 1 << 30, None) == mmf.MMF_ERR_INVALID_ARG
    assert head(24, 0, 2, 16, None, 1e-8, 16, 1, 100, 16, None, 16, 1 << 30, None) == mmf.MMF_ERR_INVALID_ARG  # x align
    assert head(16, 0, 0, 16, None, 1e-8, None, 1, 100, None, None, None, 0, None) == mmf.MMF_OK  # b = 0: nothing
    need = L.mmf_workspace_bytes(mmf.MMF_OP_HEAD, 0, 2560, 32000, 0)
    assert head(16, 1, 8, 2560, None, 1e-8, 16, 1, 32000, 16, None, 16, need - 1, None) == mmf.MMF_ERR_WORKSPACE
    # the tensor-core form keeps 2 x 128 bf16 token rows of d values in the workspace
    assert need - L.mmf_workspace_bytes(mmf.MMF_OP_HEAD, 0, 0, 32000, 0) == 2 * 128 * 2560 * 2
    assert L.mmf_workspace_bytes(mmf.MMF_OP_HEAD, 0, 2560, 0, 0) == 0


def test_hgrn2_arguments_on_host(L):
    # mmf_hgrn2_recurrence(q, f, i, dtype, b, t, heads, dk, dv, s0, s_out, o, stream)
    h2 = L.mmf_hgrn2_recurrence
    assert h2(16, 16, 16, 0, 1, 4, 1, 0, 4, None, None, 16, None) == mmf.MMF_ERR_INVALID_ARG    # dk = 0
    assert h2(16, 16, 16, 0, 1, 4, 1, 129, 4, None, None, 16, None) == mmf.MMF_ERR_INVALID_ARG  # dk > 128
    assert h2(16, 16, 16, 5, 1, 4, 1, 8, 4, None, None, 16, None) == mmf.MMF_ERR_INVALID_ARG    # dtype
    assert h2(None, 16, 16, 0, 1, 4, 1, 8, 4, None, None, 16, None) == mmf.MMF_ERR_INVALID_ARG  # null q
    assert h2(16, 16, 16, 0, -1, 4, 1, 8, 4, None, None, 16, None) == mmf.MMF_ERR_INVALID_ARG   # b < 0
    assert h2(16, 16, 16, 0, 70000, 4, 1, 8, 4, None, None, 16, None) == mmf.MMF_ERR_INVALID_ARG
    assert h2(None, None, None, 0, 0, 4, 1, 8, 4, None, None, None, None) == mmf.MMF_OK          # b = 0


def test_scan_backward_arguments_on_host(L):
    # mmf_hgrn_scan_backward(zf, zi, h, dh, dtype, b, t, d, h0, dzf, dzi, dh0, ws, ws_bytes, stream)
    sb = L.mmf_hgrn_scan_backward
    assert sb(16, 16, 16, 16, 0, -1, 4, 8, None, 16, 16, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG  # b < 0
    assert sb(16, 16, 16, 16, 3, 1, 4, 8, None, 16, 16, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG   # dtype
    assert sb(16, 16, None, 16, 0, 1, 4, 8, None, 16, 16, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG  # null h
    assert sb(None, None, None, None, 0, 0, 4, 8, None, None, None, None, None, 0, None) == mmf.MMF_OK     # b = 0
    # past 32 steps the chunked backward needs the scan's workspace, 256-byte aligned
    need = mmf.workspace_bytes(mmf.MMF_OP_SCAN, 2 * 64, 8, 0, 0)
    assert need > 0
    assert sb(16, 16, 16, 16, 0, 2, 64, 8, None, 16, 16, None, None, 0, None) == mmf.MMF_ERR_WORKSPACE
    assert sb(16, 16, 16, 16, 0, 2, 64, 8, None, 16, 16, None, 256, need - 1, None) == mmf.MMF_ERR_WORKSPACE
    assert sb(16, 16, 16, 16, 0, 2, 64, 8, None, 16, 16, None, 272, need, None) == mmf.MMF_ERR_WORKSPACE


def test_bitlinear_backward_arguments_on_host(L):
    # mmf_bitlinear_backward(x, x_dtype, m, norm_w, eps, w, q, deq, dy, dy_dtype, dx, dnorm_w, dW,
    # ws, ws_bytes, stream)
    bb = L.mmf_bitlinear_backward
    ok_w = mmf.Ternary(16, 32, 8, 64)
    assert bb(16, 0, 4, None, 1e-8, None, 16, 16, 16, 0, 16, None, None, 256, 1 << 20, None) == mmf.MMF_ERR_INVALID_ARG
    big = mmf.Ternary(16, 32, 70000, 64)
    assert bb(16, 0, 4, None, 1e-8, ctypes.byref(big), 16, 16, 16, 0, 16, None, None, 256, 1 << 20,
              None) == mmf.MMF_ERR_INVALID_ARG                                                     # n > 65535
    assert bb(16, 0, -1, None, 1e-8, ctypes.byref(ok_w), 16, 16, 16, 0, 16, None, None, 256, 1 << 20,
              None) == mmf.MMF_ERR_INVALID_ARG                                                     # m < 0
    assert bb(16, 4, 4, None, 1e-8, ctypes.byref(ok_w), 16, 16, 16, 0, 16, None, None, 256, 1 << 20,
              None) == mmf.MMF_ERR_INVALID_ARG                                                     # dtype
    assert bb(16, 0, 4, None, 1e-8, ctypes.byref(ok_w), None, 16, 16, 0, 16, None, None, 256, 1 << 20,
              None) == mmf.MMF_ERR_INVALID_ARG                                                     # null q
    assert bb(16, 0, 1000, None, 1e-8, ctypes.byref(ok_w), 16, 16, 16, 0, 16, None, None, 256, 1024,
              None) == mmf.MMF_ERR_WORKSPACE                                                       # 4 KB needed
    # the workspace holds rho and the bf16 operands of the tensor-core products (dr's dy hi / lo
    # [m][n] and t^T [k][n]; dW's scaled dy^T hi / lo [n][m] and q^T [k][m], sharing the space)
    m, k, n = 1000, 64, 8
    need = mmf.workspace_bytes(mmf.MMF_OP_BITLINEAR_BWD, m, k, n, 0)
    assert need >= 4 * m + max(2 * m * n * 2 + k * n * 2, 2 * n * m * 2 + k * m * 2)
    assert bb(16, 0, m, None, 1e-8, ctypes.byref(ok_w), 16, 16, 16, 0, 16, None, None, 256, need - 1,
              None) == mmf.MMF_ERR_WORKSPACE
    assert mmf.workspace_bytes(mmf.MMF_OP_BITLINEAR_BWD, 0, k, n, 0) == 0 or m > 0


def test_block_shape_mismatch_rejected(L):
    z = mmf.Ternary(256, 256, 64, 64)
    bw = mmf.BlockWeightsC(d=64, inner=32, eps=1e-8, i=z, f=z, g=z, o=z,
                           gate=mmf.Ternary(256, 256, 64, 64),  # should be [64][64] -> [2*32][64] ok
                           down=mmf.Ternary(256, 256, 64, 64))  # should be [64][32]: wrong
    assert L.mmf_block_fwd(ctypes.byref(bw), None, 0, 1, 1, None, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert b"down_proj" in L.mmf_last_error()


def test_binding_refuses_cpu_tensors(L):
    import torch
    with pytest.raises(ValueError):
        mmf.pack_ternary(torch.zeros(4, 4))


def test_new_bindings_refuse_cpu_tensors(L):
    # the training-gradient and HGRN2 wrappers reject host tensors before any library call
    import torch
    z = torch.zeros(1, 4, 2, 8)
    with pytest.raises(ValueError):
        mmf.hgrn2_recurrence(z, z, z)
    z3 = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        mmf.hgrn_scan_backward(z3, z3, z3, z3)
    w = mmf.PackedTernary.__new__(mmf.PackedTernary)
    w.n, w.k = 4, 8
    with pytest.raises(ValueError):
        mmf.bitlinear_backward(torch.zeros(2, 8), None, w, torch.zeros(2, 8, dtype=torch.int8),
                               torch.zeros(2), torch.zeros(2, 4))


def test_validate_packed_arguments_on_host(L):
    assert L.mmf_validate_packed(None, 16, None) == mmf.MMF_ERR_INVALID_ARG
    t = mmf.Ternary(16, 32, 4, 64)
    assert L.mmf_validate_packed(ctypes.byref(t), None, None) == mmf.MMF_ERR_INVALID_ARG
    neg = mmf.Ternary(16, 32, -1, 64)
    assert L.mmf_validate_packed(ctypes.byref(neg), 16, None) == mmf.MMF_ERR_INVALID_ARG


def test_validate_packed_alignment_on_host(L):
    # misaligned codes (not 16 bytes) or counter (not 8 bytes) are refused before any CUDA call
    good = ctypes.c_void_p(4096)
    t = mmf.Ternary(4096 + 4, 32, 4, 64)
    assert L.mmf_validate_packed(ctypes.byref(t), good, None) == mmf.MMF_ERR_INVALID_ARG
    t = mmf.Ternary(4096, 32, 4, 64)
    assert L.mmf_validate_packed(ctypes.byref(t), ctypes.c_void_p(4096 + 4), None) == mmf.MMF_ERR_INVALID_ARG


def test_decode_taps_arguments_on_host(L):
    assert L.mmf_decode_step_taps(None, 1, None, 0, 1, None, None, None, None, 0, None) == mmf.MMF_ERR_INVALID_ARG
    bw = mmf.BlockWeightsC()
    assert L.mmf_decode_step_taps(ctypes.byref(bw), 1, None, 0, 1, None, None, None, None, 0, None) == \
        mmf.MMF_ERR_INVALID_ARG


def test_header_is_plain_c_and_links_from_c(tmp_path):
    # the boundary is a C ABI: the header compiles as C99, and a C program linked against the
    # library calls its host-only entry points (sizes, status strings) with no C++ or torch
    import shutil

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "mmf.h"
int main(void) {
  if (mmf_packed_row_words(65) != 8) return 1;
  if (mmf_packed_words(3, 65) != 24) return 2;
  if (mmf_workspace_bytes(MMF_OP_SCAN, 8 * 2048, 1024, 0, 0) < (size_t)3 * 1024 * 4 * 8 * 128) return 3;
  if (mmf_workspace_bytes(MMF_OP_BITLINEAR_BWD, 1000, 64, 8, 0) == 0) return 4;
  if (strlen(mmf_status_string(MMF_ERR_WORKSPACE)) == 0) return 5;
  /* argument validation happens on the host before any device work */
  if (mmf_hgrn_scan_backward(NULL, NULL, NULL, NULL, MMF_F32, -1, 4, 8, NULL, NULL, NULL, NULL, NULL, 0, NULL)
      != MMF_ERR_INVALID_ARG) return 6;
  printf("ok\n");
  return 0;
}
''')
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(mbuild.OUT)
    res = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                          str(src), "-L", lib_dir, "-lmmf", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)


def test_decode_path_choice_on_host(L):
    # the automatic choice (fused CUDA-core launches for 1 or 2 rows, skinny tensor-core products
    # for 3 to 64 rows, the block path beyond), the engine setting's precedence and the forced
    # paths that fall back to the block path where their kernel cannot serve the shape
    F, S, B = mmf.MMF_DECODE_FUSED, mmf.MMF_DECODE_SKINNY, mmf.MMF_DECODE_BLOCK
    pf = L.mmf_decode_path_for
    try:
        assert L.mmf_set_decode_path(7) == mmf.MMF_ERR_INVALID_ARG
        assert L.mmf_set_decode_path(mmf.MMF_DECODE_AUTO) == mmf.MMF_OK
        assert pf(0, 2560, 7040) == -1 and pf(1, 0, 7040) == -1 and pf(1, 2560, -1) == -1
        assert [pf(b, 2560, 7040) for b in (1, 2, 3, 4, 8, 17, 64, 65, 256)] == [F, F, S, S, S, S, S, B, B]
        assert pf(1, 2564, 7040) == B                               # d % 8 != 0: neither fused nor skinny
        assert pf(8, 8200, 7040) == B                               # a row stage holds K <= 8192
        assert L.mmf_set_gemm_path(mmf.MMF_GEMM_SIMT) == mmf.MMF_OK
        assert [pf(b, 2560, 7040) for b in (1, 2, 3, 4, 8, 16)] == [F, F, B, F, F, B]
        assert L.mmf_set_gemm_path(mmf.MMF_GEMM_TENSOR) == mmf.MMF_OK
        assert [pf(b, 2560, 7040) for b in (1, 8, 64)] == [B, B, B]
        assert L.mmf_set_gemm_path(mmf.MMF_GEMM_AUTO) == mmf.MMF_OK
        assert L.mmf_set_decode_path(mmf.MMF_DECODE_FUSED) == mmf.MMF_OK
        assert [pf(b, 2560, 7040) for b in (1, 2, 3, 4, 8, 9)] == [F, F, B, F, F, B]
        assert L.mmf_set_decode_path(mmf.MMF_DECODE_SKINNY) == mmf.MMF_OK
        assert [pf(b, 2560, 7040) for b in (1, 64, 65)] == [S, S, B]
        assert L.mmf_set_decode_path(mmf.MMF_DECODE_BLOCK) == mmf.MMF_OK
        assert [pf(b, 2560, 7040) for b in (1, 8, 64)] == [B, B, B]
    finally:
        L.mmf_set_decode_path(mmf.MMF_DECODE_AUTO)
        L.mmf_set_gemm_path(mmf.MMF_GEMM_AUTO)


def test_noalloc_and_taps_arguments_on_host(L):
    # the allocation-free BitLinear refuses, before any CUDA call, a request whose scratch exceeds
    # its static array; the block taps refuse a null taps struct
    w = mmf.Ternary(4096, 32, 2048, 2048)
    # the codes (m x K bytes) plus per-row factors and padding: 4088 rows fit at K = 2048, 4096 not
    assert L.mmf_workspace_bytes(mmf.MMF_OP_BITLINEAR, 4088, 2048, 2048, 0) <= 8 << 20
    assert L.mmf_workspace_bytes(mmf.MMF_OP_BITLINEAR, 4096, 2048, 2048, 0) > 8 << 20
    m_big = 4096
    assert L.mmf_bitlinear_fwd_noalloc(16, 0, m_big, None, ctypes.byref(w), 16, 0, None) == mmf.MMF_ERR_WORKSPACE
    assert b"static array" in L.mmf_last_error()
    assert L.mmf_bitlinear_fwd_noalloc(16, 0, -1, None, ctypes.byref(w), 16, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_bitlinear_fwd_noalloc(16, 0, 4, None, None, 16, 0, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_bitlinear_fwd_noalloc(16, 0, 0, None, ctypes.byref(w), 16, 0, None) == mmf.MMF_OK  # nothing to do
    bw = mmf.BlockWeightsC()
    assert L.mmf_block_fwd_taps(ctypes.byref(bw), None, 0, 1, 1, None, None, None, None, None, 0,
                                None) == mmf.MMF_ERR_INVALID_ARG
    assert b"taps" in L.mmf_last_error()


def test_instrumentation_on_host(L):
    # the launch counter and the per-class timing records need no device while nothing launches
    n0 = L.mmf_launch_count()
    assert L.mmf_timing_enable(1) == mmf.MMF_OK
    assert L.mmf_timing_enable(0) == mmf.MMF_OK
    launches, ms, work = ctypes.c_int64(-1), ctypes.c_double(-1.0), ctypes.c_double(-1.0)
    assert L.mmf_timing_read(0, ctypes.byref(launches), ctypes.byref(ms), ctypes.byref(work)) == mmf.MMF_OK
    assert (launches.value, ms.value, work.value) == (0, 0.0, 0.0)
    assert L.mmf_timing_read(-1, None, None, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_timing_read(99, None, None, None) == mmf.MMF_ERR_INVALID_ARG
    assert L.mmf_launch_count() == n0


def test_bitlinear_limits_on_host(L):
    # the documented limits of mmf_bitlinear_fwd: K in [1, 32768], codes 16-byte aligned, codes and
    # scale present, x and y 16-byte aligned; each refused before any CUDA call
    ws = 1 << 30

    def call(w, x=16, y=16, m=4):
        return L.mmf_bitlinear_fwd(x, 0, m, None, ctypes.byref(w), y, 0, None, None, None, 256, ws, None)

    assert call(mmf.Ternary(16, 32, 8, 32769)) == mmf.MMF_ERR_INVALID_ARG
    assert call(mmf.Ternary(16, 32, 0, 64)) == mmf.MMF_ERR_INVALID_ARG
    assert call(mmf.Ternary(16, None, 8, 64)) == mmf.MMF_ERR_INVALID_ARG
    assert call(mmf.Ternary(16, 32, 8, 64), x=24) == mmf.MMF_ERR_INVALID_ARG
    assert call(mmf.Ternary(16, 32, 8, 64), y=None) == mmf.MMF_ERR_INVALID_ARG
    assert call(mmf.Ternary(16, 32, 8, 64), m=-1) == mmf.MMF_ERR_INVALID_ARG
    assert call(mmf.Ternary(16, 32, 8, 64), m=0) == mmf.MMF_OK
    # a workspace one byte short is refused, naming the size it needs
    need = L.mmf_workspace_bytes(mmf.MMF_OP_BITLINEAR, 4, 64, 8, 0)
    w = mmf.Ternary(16, 32, 8, 64)
    assert L.mmf_bitlinear_fwd(16, 0, 4, None, ctypes.byref(w), 16, 0, None, None, None, 256, need - 1,
                               None) == mmf.MMF_ERR_WORKSPACE


def test_block_and_backward_limits_on_host(L):
    # block sizes are 1 to 32768 with eps >= 0; the backward takes at most 2^31 - 1 rows
    for d, inner, eps in ((32776, 64, 1e-8), (64, 32776, 1e-8), (64, 64, -1.0)):
        bw = mmf.BlockWeightsC(d=d, inner=inner, eps=eps)
        assert L.mmf_block_fwd(ctypes.byref(bw), None, 0, 1, 1, None, None, None, None, 0,
                               None) == mmf.MMF_ERR_INVALID_ARG
    w = mmf.Ternary(16, 32, 8, 64)
    assert L.mmf_bitlinear_backward(16, 0, 1 << 31, None, 1e-8, ctypes.byref(w), 16, 16, 16, 0, 16, None,
                                    None, 256, 1 << 40, None) == mmf.MMF_ERR_INVALID_ARG
