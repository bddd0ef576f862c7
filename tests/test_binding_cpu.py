"""The Python binding's marshalling and argument checks, on the CPU: the library's compute entry
points are replaced by a recorder (the size queries stay the real library's), host tensors stand
in for device tensors, and each wrapper's call is checked argument by argument against the C
signature in include/mmf.h. Bad shapes and dtypes must raise before anything reaches the library."""
import ctypes

import pytest
import torch

import ternary_weight_matmul_b200 as mmf
from ternary_weight_matmul_b200 import build as mbuild


class _Recorder:
    """Stands in for libmmf: size queries go to the real library, every other mmf_* call is
    recorded and returns MMF_OK."""

    REAL = ("mmf_workspace_bytes", "mmf_packed_row_words", "mmf_packed_words", "mmf_status_string",
            "mmf_last_error")

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in self.REAL:
            return getattr(self.real, name)
        if not name.startswith("mmf_"):
            raise AttributeError(name)

        def record(*args):
            self.calls.append((name, args))
            return mmf.MMF_OK
        return record

    def last(self, name):
        hits = [a for n, a in self.calls if n == name]
        assert hits, (name, [n for n, _ in self.calls])
        return hits[-1]


@pytest.fixture()
def fake(monkeypatch):
    mbuild.build()
    rec = _Recorder(mmf.lib())
    monkeypatch.setattr(mmf, "lib", lambda: rec)
    monkeypatch.setattr(mmf, "_stream", lambda device: 0)
    monkeypatch.setattr(mmf, "_ws_cache", {})
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)

    def host_dev(t):
        if not t.is_contiguous():
            raise ValueError("expected a contiguous tensor")
        return t
    monkeypatch.setattr(mmf, "_dev", host_dev)
    monkeypatch.setattr(mmf, "_cuda", lambda t, name: t)
    return rec


def _packed(n, k):
    return mmf.PackedTernary(torch.zeros(n, mmf.packed_row_words(k), dtype=torch.int32), torch.ones(1), n, k)


def _block(d, inner):
    shapes = {"i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d), "gate": (2 * inner, d), "down": (d, inner)}
    packed = {p: _packed(n, k) for p, (n, k) in shapes.items()}
    norms = {f"nw_{p}": torch.ones(k) for p, (n, k) in shapes.items()}
    norms["gnorm_w"] = torch.ones(d)
    return mmf.Block(d, inner, packed, norms)


def _ws_ok(ptr, nbytes, op, *sizes):
    need = mmf.workspace_bytes(op, *sizes)
    assert ptr is not None and nbytes >= need


def test_bitlinear_fwd_marshalling(fake):
    x = torch.randn(5, 64, dtype=torch.bfloat16)
    nw = torch.ones(64)
    w = _packed(24, 64)
    y, q, deq, acc = mmf.bitlinear_fwd(x, nw, w, y_dtype=torch.float32, debug=True)
    a = fake.last("mmf_bitlinear_fwd")
    assert a[0] == x.data_ptr() and a[1] == mmf.MMF_BF16 and a[2] == 5 and a[3] == nw.data_ptr()
    tw = a[4]._obj
    assert (tw.codes, tw.scale, tw.n, tw.k) == (w.codes.data_ptr(), w.scale.data_ptr(), 24, 64)
    assert a[5] == y.data_ptr() and a[6] == mmf.MMF_F32 and tuple(y.shape) == (5, 24) and y.dtype == torch.float32
    assert (a[7], a[8], a[9]) == (q.data_ptr(), deq.data_ptr(), acc.data_ptr())
    assert tuple(q.shape) == (5, 64) and q.dtype == torch.int8 and tuple(acc.shape) == (5, 24)
    _ws_ok(a[10], a[11], mmf.MMF_OP_BITLINEAR, 5, 64, 24, 0)
    # leading dimensions fold into rows
    y3 = mmf.bitlinear_fwd(torch.randn(2, 3, 64), None, w)
    a = fake.last("mmf_bitlinear_fwd")
    assert a[2] == 6 and a[3] is None and tuple(y3.shape) == (2, 3, 24) and a[6] == mmf.MMF_F32


def test_hgrn_scan_marshalling_of_strided_gates(fake):
    b, t, d = 2, 7, 16
    z = torch.randn(b, t, 3 * d, dtype=torch.bfloat16)
    zi, zf = z[:, :, :d], z[:, :, d:2 * d]
    h0 = torch.randn(b, d)
    h, hl = mmf.hgrn_scan(zf, zi, h0, h_dtype=torch.bfloat16)
    a = fake.last("mmf_hgrn_scan")
    assert a[0] == zf.data_ptr() and a[1] == zi.data_ptr() and a[2] == mmf.MMF_BF16
    assert a[3] == 3 * d and (a[4], a[5], a[6]) == (b, t, d) and a[7] == h0.data_ptr()
    assert a[8] == h.data_ptr() and a[9] == mmf.MMF_BF16 and a[10] == hl.data_ptr()
    assert tuple(h.shape) == (b, t, d) and tuple(hl.shape) == (b, d) and hl.dtype == torch.float32
    _ws_ok(a[11], a[12], mmf.MMF_OP_SCAN, b * t, d, 0, 0)


def test_block_decode_and_stack_marshalling(fake):
    d, inner, b, t = 32, 48, 2, 5
    blocks = [_block(d, inner), _block(d, inner)]
    x = torch.randn(b, t, d)
    y, hl = mmf.block_fwd(blocks[0], x)
    a = fake.last("mmf_block_fwd")
    bw = a[0]._obj
    assert (bw.d, bw.inner) == (d, inner) and bw.gate.n == 2 * inner and bw.down.k == inner
    assert bw.nw_down == blocks[0].norms["nw_down"].data_ptr() and bw.gnorm_w == blocks[0].norms["gnorm_w"].data_ptr()
    assert a[1] == x.data_ptr() and a[2] == mmf.MMF_F32 and (a[3], a[4]) == (b, t) and a[5] is None
    assert a[6] == y.data_ptr() and a[7] == hl.data_ptr()
    _ws_ok(a[8], a[9], mmf.MMF_OP_BLOCK, b * t, d, inner, 1)

    xs = torch.randn(b, d, dtype=torch.bfloat16)
    state = torch.zeros(2, b, d)
    out = torch.empty_like(xs)
    ys = mmf.decode_step(blocks, xs, state, out=out)
    a = fake.last("mmf_decode_step")
    assert ys is out and len(a[0]) == 2 and a[0][1].down.codes == blocks[1].packed["down"].codes.data_ptr()
    assert a[1] == 2 and a[2] == xs.data_ptr() and a[3] == mmf.MMF_BF16 and a[4] == b
    assert a[5] == state.data_ptr() and a[6] == out.data_ptr()
    _ws_ok(a[7], a[8], mmf.MMF_OP_DECODE, b, d, inner, 2)

    table = torch.randn(100, d, dtype=torch.bfloat16)
    ids = torch.randint(0, 100, (b, t), dtype=torch.int32)
    y, h_last = mmf.stack_fwd(blocks, ids, table, want_state=True)
    a = fake.last("mmf_stack_fwd")
    assert a[1] == 2 and a[2] == ids.data_ptr() and (a[3], a[4]) == (b, t) and a[5] == table.data_ptr()
    assert a[6] == 100 and a[7] == mmf.MMF_BF16 and a[8] == y.data_ptr() and a[9] == h_last.data_ptr()
    assert tuple(y.shape) == (b, t, d) and tuple(h_last.shape) == (2, b, d)
    _ws_ok(a[10], a[11], mmf.MMF_OP_STACK, b * t, d, inner, 2)


def test_head_embed_and_next_rows_marshalling(fake):
    d, vocab, b = 32, 300, 3
    x = torch.randn(b, d)
    nw = torch.ones(d)
    table = torch.randn(vocab, d, dtype=torch.bfloat16)
    ids_out = torch.empty(b, dtype=torch.int32)
    ids, logits = mmf.lm_head_argmax(x, nw, table, want_logits=True, ids_out=ids_out)
    a = fake.last("mmf_lm_head_argmax")
    assert ids is ids_out and a[0] == x.data_ptr() and (a[2], a[3]) == (b, d) and a[4] == nw.data_ptr()
    assert a[6] == table.data_ptr() and a[7] == mmf.MMF_BF16 and a[8] == vocab and a[9] == ids_out.data_ptr()
    assert a[10] == logits.data_ptr() and tuple(logits.shape) == (b, vocab)
    _ws_ok(a[11], a[12], mmf.MMF_OP_HEAD, 0, d, vocab, 0)

    tok = torch.tensor([3, 0, 299], dtype=torch.int32)
    rows = mmf.embed_gather(tok, table)
    a = fake.last("mmf_embed_gather")
    assert a[0] == tok.data_ptr() and a[1] == 3 and a[2] == table.data_ptr() and (a[4], a[5]) == (vocab, d)
    assert a[6] == rows.data_ptr() and tuple(rows.shape) == (3, d)

    bb, t, dd = 2, 9, 16
    zf, zi, h, dh = (torch.randn(bb, t, dd) for _ in range(4))
    h0 = torch.randn(bb, dd)
    dzf, dzi, dh0 = mmf.hgrn_scan_backward(zf, zi, h, dh, h0)
    a = fake.last("mmf_hgrn_scan_backward")
    assert a[:4] == (zf.data_ptr(), zi.data_ptr(), h.data_ptr(), dh.data_ptr()) and a[4] == mmf.MMF_F32
    assert a[5:8] == (bb, t, dd) and a[8] == h0.data_ptr()
    assert a[9:12] == (dzf.data_ptr(), dzi.data_ptr(), dh0.data_ptr())
    _ws_ok(a[12], a[13], mmf.MMF_OP_SCAN, bb * t, dd, 0, 0)

    m, k, n = 6, 64, 24
    w = _packed(n, k)
    xk = torch.randn(m, k)
    q = torch.zeros(m, k, dtype=torch.int8)
    deq = torch.ones(m)
    dy = torch.randn(m, n, dtype=torch.bfloat16)
    dx, dnw, dW = mmf.bitlinear_backward(xk, torch.ones(k), w, q, deq, dy)
    a = fake.last("mmf_bitlinear_backward")
    assert a[0] == xk.data_ptr() and a[2] == m and a[6] == q.data_ptr() and a[7] == deq.data_ptr()
    assert a[8] == dy.data_ptr() and a[9] == mmf.MMF_BF16
    assert a[10:13] == (dx.data_ptr(), dnw.data_ptr(), dW.data_ptr()) and tuple(dW.shape) == (n, k)
    _ws_ok(a[13], a[14], mmf.MMF_OP_BITLINEAR_BWD, m, k, n, 0)

    qh, fh = torch.randn(2, 5, 3, 8), torch.rand(2, 5, 3, 8)
    ih = torch.randn(2, 5, 3, 12)
    o, s = mmf.hgrn2_recurrence(qh, fh, ih, want_state=True)
    a = fake.last("mmf_hgrn2_recurrence")
    assert a[:3] == (qh.data_ptr(), fh.data_ptr(), ih.data_ptr()) and a[4:9] == (2, 5, 3, 8, 12)
    assert a[9] is None and a[10] == s.data_ptr() and a[11] == o.data_ptr() and tuple(o.shape) == (2, 5, 3, 12)


def test_wrappers_refuse_mismatched_arguments(fake):
    w = _packed(24, 64)
    with pytest.raises(ValueError, match="k = 64"):
        mmf.bitlinear_fwd(torch.randn(5, 63), None, w)
    with pytest.raises(ValueError, match="norm_w"):
        mmf.bitlinear_fwd(torch.randn(5, 64), torch.ones(64, dtype=torch.bfloat16), w)
    with pytest.raises(ValueError, match="norm_w"):
        mmf.bitlinear_fwd(torch.randn(5, 64), torch.ones(65), w)
    z = torch.randn(2, 7, 16)
    with pytest.raises(ValueError, match="one shape"):
        mmf.hgrn_scan(z, torch.randn(2, 7, 17))
    with pytest.raises(ValueError, match="h0"):
        mmf.hgrn_scan(z, z, torch.randn(2, 17))
    with pytest.raises(ValueError, match="h0"):
        mmf.hgrn_scan(z, z, torch.randn(2, 16, dtype=torch.float64))
    blk = _block(32, 48)
    with pytest.raises(ValueError, match="hidden size"):
        mmf.block_fwd(blk, torch.randn(2, 5, 31))
    with pytest.raises(ValueError, match="h0"):
        mmf.block_fwd(blk, torch.randn(2, 5, 32), torch.randn(3, 32))
    xs = torch.randn(2, 32)
    with pytest.raises(ValueError, match="state"):
        mmf.decode_step([blk, blk], xs, torch.zeros(1, 2, 32))
    with pytest.raises(ValueError, match="state"):
        mmf.decode_step([blk], xs, torch.zeros(1, 2, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out"):
        mmf.decode_step([blk], xs, torch.zeros(1, 2, 32), out=xs)
    with pytest.raises(ValueError, match="hidden size"):
        mmf.decode_step([blk], torch.randn(2, 16), torch.zeros(1, 2, 16))
    table = torch.randn(100, 32)
    with pytest.raises(ValueError, match="int32"):
        mmf.stack_fwd([blk], torch.zeros(2, 5, dtype=torch.int64), table)
    with pytest.raises(ValueError, match="int32"):
        mmf.embed_gather(torch.zeros(3, dtype=torch.int64), table)
    with pytest.raises(ValueError, match="hidden size"):
        mmf.stack_fwd([blk], torch.zeros(2, 5, dtype=torch.int32), torch.randn(100, 16))
    with pytest.raises(ValueError, match="table"):
        mmf.lm_head_argmax(xs, None, torch.randn(100, 16))
    with pytest.raises(ValueError, match="ids_out"):
        mmf.lm_head_argmax(xs, None, table, ids_out=torch.empty(3, dtype=torch.int32))
    with pytest.raises(ValueError, match="norm_w"):
        mmf.lm_head_argmax(xs, torch.ones(31), table)
    with pytest.raises(ValueError, match="k = 64"):
        mmf.bitlinear_backward(torch.randn(6, 32), None, w, torch.zeros(6, 32, dtype=torch.int8), torch.ones(6),
                               torch.randn(6, 24))
    with pytest.raises(ValueError, match="h0"):
        mmf.hgrn_scan_backward(z, z, z, z, torch.randn(2, 15))
    assert not [n for n, _ in fake.calls if n not in _Recorder.REAL]


def test_wrappers_refuse_host_tensors():
    # without the recorder: a host tensor never reaches the library (no CPU path exists)
    w = _packed(24, 64)
    blk = _block(32, 48)
    table = torch.randn(100, 32)
    calls = [
        lambda: mmf.bitlinear_fwd(torch.randn(5, 64), None, w),
        lambda: mmf.hgrn_scan(torch.randn(2, 7, 16), torch.randn(2, 7, 16)),
        lambda: mmf.block_fwd(blk, torch.randn(2, 5, 32)),
        lambda: mmf.decode_step([blk], torch.randn(2, 32), torch.zeros(1, 2, 32)),
        lambda: mmf.stack_fwd([blk], torch.zeros(2, 5, dtype=torch.int32), table),
        lambda: mmf.embed_gather(torch.zeros(3, dtype=torch.int32), table),
        lambda: mmf.lm_head_argmax(torch.randn(2, 32), None, table),
    ]
    for c in calls:
        with pytest.raises(ValueError, match="CUDA"):
            c()


def test_set_wait_limit_passes_microseconds(fake):
    mmf.set_wait_limit(1500)
    assert fake.last("mmf_set_wait_limit") == (1500,)
    assert ctypes.sizeof(ctypes.c_uint32) == 4
