"""Python binding of libmmf, the sm_100a HGRNBit block-forward library (include/mmf.h).

Argument marshalling only: every step of the forward runs in the library's CUDA kernels.
PyTorch supplies device memory (inputs, outputs and scratch workspaces) and the current CUDA
stream. There is no CPU or PyTorch fallback: when ``libmmf.so`` is missing, or the device is not
an sm_100a part, every call raises.

The function names mirror the C ABI (``mmf_pack_ternary`` -> ``pack_ternary`` and so on); the raw
C entry points are available as ``lib().mmf_*``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmmf.so")

MMF_OK, MMF_ERR_INVALID_ARG, MMF_ERR_UNSUPPORTED, MMF_ERR_WORKSPACE, MMF_ERR_CUDA, MMF_ERR_TIMEOUT = range(6)
MMF_F32, MMF_BF16 = 0, 1
(MMF_OP_PACK, MMF_OP_BITLINEAR, MMF_OP_BLOCK, MMF_OP_DECODE, MMF_OP_STACK, MMF_OP_SCAN, MMF_OP_HEAD,
 MMF_OP_BITLINEAR_BWD) = range(8)
MMF_GEMM_AUTO, MMF_GEMM_TENSOR, MMF_GEMM_SIMT = range(3)
MMF_DECODE_AUTO, MMF_DECODE_FUSED, MMF_DECODE_SKINNY, MMF_DECODE_BLOCK = range(4)

EXPORTED = (
    "mmf_packed_row_words", "mmf_packed_words", "mmf_workspace_bytes", "mmf_pack_ternary",
    "mmf_bitlinear_fwd", "mmf_hgrn_scan", "mmf_block_fwd", "mmf_block_fwd_taps", "mmf_decode_step",
    "mmf_embed_gather", "mmf_lm_head_argmax", "mmf_hgrn2_recurrence", "mmf_hgrn_scan_backward",
    "mmf_bitlinear_backward", "mmf_validate_packed",
    "mmf_stack_fwd", "mmf_sync_status", "mmf_status_string", "mmf_last_error",
    "mmf_set_gemm_path", "mmf_set_wait_limit", "mmf_launch_count", "mmf_timing_enable", "mmf_timing_read",
    "mmf_bitlinear_fwd_noalloc", "mmf_decode_step_taps", "mmf_set_decode_path", "mmf_decode_path_for",
)
NOALLOC_SCRATCH_BYTES = 8 << 20


class MmfError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


class Ternary(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("n", ctypes.c_int32), ("k", ctypes.c_int32)]


class BlockWeightsC(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("inner", ctypes.c_int32), ("eps", ctypes.c_float)] + \
        [(f"nw_{p}", ctypes.c_void_p) for p in ("i", "f", "g", "o", "gate", "down")] + \
        [("gnorm_w", ctypes.c_void_p)] + \
        [(p, Ternary) for p in ("i", "f", "g", "o", "gate", "down")]


class BlockTapsC(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "q_ifg", "deq_ifg", "z", "h", "q_o", "deq_o", "x1", "q_gate", "deq_gate", "gu", "q_down", "deq_down",
        "v")]


class DecodeTapsC(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "q_ifg", "deq_ifg", "z", "h", "q_o", "deq_o", "x1", "q_gate", "deq_gate", "gu", "v", "q_down", "deq_down",
        "y")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmmf.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m ternary_weight_matmul_b200.build` "
                          "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
    sig = {
        "mmf_packed_row_words": (i32, [i32]),
        "mmf_packed_words": (sz, [i32, i32]),
        "mmf_workspace_bytes": (sz, [ctypes.c_int, i64, i32, i32, i32]),
        "mmf_pack_ternary": (ctypes.c_int, [vp, ctypes.c_int, i32, i32, vp, vp, vp, sz, st]),
        "mmf_bitlinear_fwd": (ctypes.c_int, [vp, ctypes.c_int, i64, vp, ctypes.POINTER(Ternary), vp,
                                             ctypes.c_int, vp, vp, vp, vp, sz, st]),
        "mmf_bitlinear_fwd_noalloc": (ctypes.c_int, [vp, ctypes.c_int, i64, vp, ctypes.POINTER(Ternary), vp,
                                                     ctypes.c_int, st]),
        "mmf_hgrn_scan": (ctypes.c_int, [vp, vp, ctypes.c_int, i64, i32, i64, i32, vp, vp, ctypes.c_int, vp, vp, sz,
                                         st]),
        "mmf_block_fwd": (ctypes.c_int, [ctypes.POINTER(BlockWeightsC), vp, ctypes.c_int, i32, i64, vp, vp, vp,
                                         vp, sz, st]),
        "mmf_block_fwd_taps": (ctypes.c_int, [ctypes.POINTER(BlockWeightsC), vp, ctypes.c_int, i32, i64, vp, vp,
                                              vp, ctypes.POINTER(BlockTapsC), vp, sz, st]),
        "mmf_decode_step": (ctypes.c_int, [ctypes.POINTER(BlockWeightsC), i32, vp, ctypes.c_int, i32, vp, vp,
                                           vp, sz, st]),
        "mmf_decode_step_taps": (ctypes.c_int, [ctypes.POINTER(BlockWeightsC), i32, vp, ctypes.c_int, i32, vp, vp,
                                                ctypes.POINTER(DecodeTapsC), vp, sz, st]),
        "mmf_embed_gather": (ctypes.c_int, [vp, i64, vp, ctypes.c_int, i32, i32, vp, st]),
        "mmf_lm_head_argmax": (ctypes.c_int, [vp, ctypes.c_int, i32, i32, vp, ctypes.c_float, vp, ctypes.c_int, i32,
                                              vp, vp, vp, sz, st]),
        "mmf_hgrn2_recurrence": (ctypes.c_int, [vp, vp, vp, ctypes.c_int, i32, i64, i32, i32, i32, vp, vp, vp, st]),
        "mmf_hgrn_scan_backward": (ctypes.c_int, [vp, vp, vp, vp, ctypes.c_int, i32, i64, i32, vp, vp, vp, vp, vp,
                                                   ctypes.c_size_t, st]),
        "mmf_validate_packed": (ctypes.c_int, [ctypes.POINTER(Ternary), vp, st]),
        "mmf_bitlinear_backward": (ctypes.c_int, [vp, ctypes.c_int, i64, vp, ctypes.c_float, ctypes.POINTER(Ternary),
                                                  vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, sz, st]),
        "mmf_stack_fwd": (ctypes.c_int, [ctypes.POINTER(BlockWeightsC), i32, vp, i32, i64, vp, i32,
                                         ctypes.c_int, vp, vp, vp, sz, st]),
        "mmf_sync_status": (ctypes.c_int, [st]),
        "mmf_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "mmf_last_error": (ctypes.c_char_p, []),
        "mmf_set_gemm_path": (ctypes.c_int, [ctypes.c_int]),
        "mmf_set_decode_path": (ctypes.c_int, [ctypes.c_int]),
        "mmf_decode_path_for": (i32, [i32, i32, i32]),
        "mmf_set_wait_limit": (ctypes.c_int, [ctypes.c_uint32]),
        "mmf_launch_count": (ctypes.c_uint64, []),
        "mmf_timing_enable": (ctypes.c_int, [ctypes.c_int]),
        "mmf_timing_read": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != MMF_OK:
        L = lib()
        raise MmfError(status, where, L.mmf_last_error().decode() or L.mmf_status_string(status).decode())


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return MMF_F32
    if t == torch.bfloat16:
        return MMF_BF16
    raise TypeError(f"unsupported dtype {t}: float32 or bfloat16")


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    """A CUDA tensor of any strides (strided views the library reads through a row stride)."""
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    return t


def _f32(t: torch.Tensor | None, shape: tuple[int, ...], name: str) -> torch.Tensor | None:
    """An optional contiguous float32 CUDA tensor of the given shape (norm gains, states): the
    library reads exactly that many float32 values from its pointer."""
    if t is None:
        return None
    if t.dtype != torch.float32 or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected float32 of shape {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    return _dev(t)


def _i32(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.int32:
        raise ValueError(f"{name}: expected int32 token ids, got {t.dtype}")
    return _dev(t)


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


_ws_cache: dict[tuple[int, int], torch.Tensor] = {}


def workspace(op: int, m: int, d: int, inner: int, n_layers: int, device: torch.device) -> torch.Tensor:
    """A scratch buffer of at least mmf_workspace_bytes(...) bytes, cached per (device, stream)."""
    need = int(lib().mmf_workspace_bytes(op, m, d, inner, n_layers))
    key = (device.index if device.index is not None else torch.cuda.current_device(), _stream(device))
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def workspace_bytes(op: int, m: int, d: int, inner: int, n_layers: int = 1) -> int:
    return int(lib().mmf_workspace_bytes(op, m, d, inner, n_layers))


def packed_row_words(k: int) -> int:
    return int(lib().mmf_packed_row_words(k))


# ---------------------------------------------------------------------------------------------
# weights
# ---------------------------------------------------------------------------------------------
@dataclass
class PackedTernary:
    """A packed ternary matrix: codes [n][packed_row_words(k)] (u32 stored as int32) and scale [1]."""

    codes: torch.Tensor
    scale: torch.Tensor
    n: int
    k: int

    def c(self) -> Ternary:
        return Ternary(self.codes.data_ptr(), self.scale.data_ptr(), self.n, self.k)


def pack_ternary(w: torch.Tensor) -> PackedTernary:
    """mmf_pack_ternary: ternarise and pack a [n, k] float32/bfloat16 CUDA weight."""
    _dev(w)
    n, k = w.shape
    L = lib()
    codes = torch.empty((n, packed_row_words(k)), dtype=torch.int32, device=w.device)
    scale = torch.empty(1, dtype=torch.float32, device=w.device)
    ws = workspace(MMF_OP_PACK, n * k, 0, 0, 0, w.device)
    _check(L.mmf_pack_ternary(w.data_ptr(), _dt(w.dtype), n, k, codes.data_ptr(), scale.data_ptr(),
                              ws.data_ptr(), ws.numel(), _stream(w.device)), "mmf_pack_ternary")
    return PackedTernary(codes, scale, n, k)


PROJS = ("i", "f", "g", "o", "gate", "down")


@dataclass
class Block:
    """Device weights of one HGRNBit block: packed projections and float32 norm gains."""

    d: int
    inner: int
    packed: dict[str, PackedTernary]
    norms: dict[str, torch.Tensor]        # nw_<p> for p in PROJS, and gnorm_w
    eps: float = 1e-8
    _c: BlockWeightsC | None = field(default=None, repr=False)

    def c(self) -> BlockWeightsC:
        if self._c is None:
            kw = {"d": self.d, "inner": self.inner, "eps": self.eps}
            for p in PROJS:
                kw[f"nw_{p}"] = self.norms[f"nw_{p}"].data_ptr()
                kw[p] = self.packed[p].c()
            kw["gnorm_w"] = self.norms["gnorm_w"].data_ptr()
            self._c = BlockWeightsC(**kw)
        return self._c


def make_block(params: dict, device: torch.device | str = "cuda", weight_dtype: torch.dtype = torch.float32) -> Block:
    """Upload latent weights W_<p> [N,K] and gains (numpy or torch) and pack them on the device."""
    device = torch.device(device)
    packed, norms = {}, {}
    for p in PROJS:
        w = torch.as_tensor(params[f"W_{p}"]).to(device=device, dtype=weight_dtype).contiguous()
        packed[p] = pack_ternary(w)
        norms[f"nw_{p}"] = torch.as_tensor(params[f"nw_{p}"]).to(device=device, dtype=torch.float32).contiguous()
    norms["gnorm_w"] = torch.as_tensor(params["gnorm_w"]).to(device=device, dtype=torch.float32).contiguous()
    d = packed["o"].n
    inner = packed["down"].k
    return Block(d, inner, packed, norms)


def _blocks_array(blocks: list[Block]):
    arr = (BlockWeightsC * len(blocks))(*[b.c() for b in blocks])
    return arr


# ---------------------------------------------------------------------------------------------
# calls
# ---------------------------------------------------------------------------------------------
def bitlinear_fwd(x: torch.Tensor, norm_w: torch.Tensor | None, w: PackedTernary,
                  y_dtype: torch.dtype | None = None, debug: bool = False):
    """mmf_bitlinear_fwd on x [..., k]. Returns y, or (y, q, deq, acc) with debug=True."""
    if x.dim() < 1 or x.shape[-1] != w.k:
        raise ValueError(f"x: last dimension {tuple(x.shape)[-1:]} is not the weight's k = {w.k}")
    _f32(norm_w, (w.k,), "norm_w")
    _dev(x)
    lead = x.shape[:-1]
    m = int(x.numel() // w.k) if w.k else 0
    y = torch.empty(*lead, w.n, dtype=y_dtype or x.dtype, device=x.device)
    q = deq = acc = None
    if debug:
        q = torch.empty(m, w.k, dtype=torch.int8, device=x.device)
        deq = torch.empty(m, dtype=torch.float32, device=x.device)
        acc = torch.empty(m, w.n, dtype=torch.int32, device=x.device)
    ws = workspace(MMF_OP_BITLINEAR, m, w.k, w.n, 0, x.device)
    tw = w.c()
    _check(lib().mmf_bitlinear_fwd(x.data_ptr(), _dt(x.dtype), m, _ptr(norm_w), ctypes.byref(tw), y.data_ptr(),
                                   _dt(y.dtype), _ptr(q), _ptr(deq), _ptr(acc), ws.data_ptr(), ws.numel(),
                                   _stream(x.device)), "mmf_bitlinear_fwd")
    return (y, q, deq, acc) if debug else y


def hgrn_scan(zf: torch.Tensor, zi: torch.Tensor, h0: torch.Tensor | None = None,
              h_dtype: torch.dtype = torch.float32):
    """mmf_hgrn_scan on [b, t, d] gate pre-activations (rows may be strided views with unit
    inner stride). Returns (h [b, t, d], h_last [b, d] float32)."""
    b, t, d = zf.shape
    _cuda(zf, "zf")
    _cuda(zi, "zi")
    if tuple(zi.shape) != (b, t, d):
        raise ValueError("zf and zi need one shape [b, t, d]")
    _f32(h0, (b, d), "h0")
    if zf.stride(2) != 1 or zi.stride() != zf.stride() or zf.dtype != zi.dtype:
        raise ValueError("zf and zi need the same dtype and strides, unit inner stride")
    if t > 1 and zf.stride(0) != t * zf.stride(1):
        raise ValueError("rows of zf must be evenly strided across the batch")
    h = torch.empty(b, t, d, dtype=h_dtype, device=zf.device)
    h_last = torch.empty(b, d, dtype=torch.float32, device=zf.device)
    zstride = zf.stride(1) if t > 1 else max(d, zf.stride(0) if b > 1 else d)
    ws = workspace(MMF_OP_SCAN, b * t, d, 0, 0, zf.device)
    _check(lib().mmf_hgrn_scan(zf.data_ptr(), zi.data_ptr(), _dt(zf.dtype), zstride, b, t, d, _ptr(h0),
                               h.data_ptr(), _dt(h_dtype), h_last.data_ptr(), ws.data_ptr(), ws.numel(),
                               _stream(zf.device)), "mmf_hgrn_scan")
    return h, h_last


def validate_packed(w: "PackedTernary") -> int:
    """mmf_validate_packed: the number of malformed 2-bit fields in w (0 when well formed): fields
    of real columns holding the unused pattern 10 plus nonzero fields in the padding columns,
    each malformed field counted once."""
    _dev(w.codes)
    bad = torch.empty(1, dtype=torch.int64, device=w.codes.device)
    tw = w.c()
    _check(lib().mmf_validate_packed(ctypes.byref(tw), bad.data_ptr(), _stream(w.codes.device)),
           "mmf_validate_packed")
    return int(bad.item())


def bitlinear_backward(x: torch.Tensor, norm_w: torch.Tensor | None, w: "PackedTernary", q: torch.Tensor,
                       deq: torch.Tensor, dy: torch.Tensor, eps: float = 1e-8, want_dnorm_w: bool = True,
                       want_dW: bool = True):
    """mmf_bitlinear_backward: (dx [m, k], dnorm_w [k] or None, dW [n, k] or None), float32, from
    x [m, k], the forward's codes q [m, k] int8 and factors deq [m] float32, and dy [m, n]
    (contiguous)."""
    for a in (x, q, deq, dy):
        _dev(a)
        if not a.is_contiguous():
            raise ValueError("x, q, deq and dy need contiguous storage")
    m, k = x.shape
    if k != w.k:
        raise ValueError(f"x: {k} columns, the weight has k = {w.k}")
    _f32(norm_w, (k,), "norm_w")
    if tuple(q.shape) != (m, k) or q.dtype != torch.int8 or tuple(deq.shape) != (m,) or tuple(dy.shape) != (m, w.n):
        raise ValueError("shapes: x, q [m, k] (q int8), deq [m], dy [m, n]")
    dx = torch.empty(m, k, dtype=torch.float32, device=x.device)
    dnw = torch.empty(k, dtype=torch.float32, device=x.device) if want_dnorm_w else None
    dW = torch.empty(w.n, k, dtype=torch.float32, device=x.device) if want_dW else None
    ws = workspace(MMF_OP_BITLINEAR_BWD, m, k, w.n, 0, x.device)
    tw = w.c()
    _check(lib().mmf_bitlinear_backward(x.data_ptr(), _dt(x.dtype), m, _ptr(norm_w), eps, ctypes.byref(tw),
                                        q.data_ptr(), deq.data_ptr(), dy.data_ptr(), _dt(dy.dtype), dx.data_ptr(),
                                        _ptr(dnw), _ptr(dW), ws.data_ptr(), ws.numel(), _stream(x.device)),
           "mmf_bitlinear_backward")
    return dx, dnw, dW


def hgrn_scan_backward(zf: torch.Tensor, zi: torch.Tensor, h: torch.Tensor, dh: torch.Tensor,
                       h0: torch.Tensor | None = None):
    """mmf_hgrn_scan_backward on [b, t, d] tensors of one dtype (contiguous): the gradients
    (dzf, dzi [b, t, d], dh0 [b, d] float32) given the forward's states h and dL/dh."""
    for a in (zf, zi, h, dh):
        _dev(a)
        if a.dtype != zf.dtype or tuple(a.shape) != tuple(zf.shape):
            raise ValueError("zf, zi, h and dh need one dtype and one shape [b, t, d]")
    b, t, d = zf.shape
    _f32(h0, (b, d), "h0")
    dzf = torch.empty_like(zf)
    dzi = torch.empty_like(zf)
    dh0 = torch.empty(b, d, dtype=torch.float32, device=zf.device)
    ws = workspace(MMF_OP_SCAN, b * t, d, 0, 0, zf.device)
    _check(lib().mmf_hgrn_scan_backward(zf.data_ptr(), zi.data_ptr(), h.data_ptr(), dh.data_ptr(), _dt(zf.dtype),
                                        b, t, d, _ptr(h0), dzf.data_ptr(), dzi.data_ptr(), dh0.data_ptr(),
                                        ws.data_ptr(), ws.numel(), _stream(zf.device)), "mmf_hgrn_scan_backward")
    return dzf, dzi, dh0


def hgrn2_recurrence(q: torch.Tensor, f: torch.Tensor, i: torch.Tensor, s0: torch.Tensor | None = None,
                     want_state: bool = False):
    """mmf_hgrn2_recurrence on q, f [b, t, heads, dk] and i [b, t, heads, dv] (one dtype,
    contiguous): o [b, t, heads, dv] and, with want_state, the final state [b, heads, dk, dv]
    float32."""
    for a in (q, f, i):
        _dev(a)
        if not a.is_contiguous() or a.dtype != q.dtype:
            raise ValueError("q, f and i need one dtype and contiguous storage")
    b, t, heads, dk = q.shape
    dv = i.shape[-1]
    if tuple(f.shape) != (b, t, heads, dk) or tuple(i.shape[:3]) != (b, t, heads):
        raise ValueError("shapes: q, f [b, t, heads, dk] and i [b, t, heads, dv]")
    if s0 is not None and (tuple(s0.shape) != (b, heads, dk, dv) or s0.dtype != torch.float32
                           or not s0.is_contiguous()):
        raise ValueError("s0 must be a contiguous float32 [b, heads, dk, dv]")
    o = torch.empty(b, t, heads, dv, dtype=q.dtype, device=q.device)
    s_out = torch.empty(b, heads, dk, dv, dtype=torch.float32, device=q.device) if want_state else None
    _check(lib().mmf_hgrn2_recurrence(q.data_ptr(), f.data_ptr(), i.data_ptr(), _dt(q.dtype), b, t, heads, dk, dv,
                                      _ptr(s0), _ptr(s_out), o.data_ptr(), _stream(q.device)),
           "mmf_hgrn2_recurrence")
    return (o, s_out) if want_state else o


def block_fwd(block: Block, x: torch.Tensor, h0: torch.Tensor | None = None):
    """mmf_block_fwd on x [b, t, d]. Returns (y, h_last [b, d] float32)."""
    _dev(x)
    b, t, d = x.shape
    if d != block.d:
        raise ValueError(f"x: hidden size {d}, the block's is {block.d}")
    _f32(h0, (b, d), "h0")
    y = torch.empty_like(x)
    h_last = torch.empty(b, d, dtype=torch.float32, device=x.device)
    ws = workspace(MMF_OP_BLOCK, b * t, block.d, block.inner, 1, x.device)
    bw = block.c()
    _check(lib().mmf_block_fwd(ctypes.byref(bw), x.data_ptr(), _dt(x.dtype), b, t, _ptr(h0), y.data_ptr(),
                               h_last.data_ptr(), ws.data_ptr(), ws.numel(), _stream(x.device)), "mmf_block_fwd")
    return y, h_last


def block_fwd_taps(block: Block, x: torch.Tensor, h0: torch.Tensor | None = None):
    """mmf_block_fwd_taps: the block forward plus every intermediate (see mmf_block_taps).
    Returns (y, h_last, taps) with taps a dict of tensors."""
    _dev(x)
    b, t, d = x.shape
    if d != block.d:
        raise ValueError(f"x: hidden size {d}, the block's is {block.d}")
    _f32(h0, (b, d), "h0")
    m, inner, dev, dt = b * t, block.inner, x.device, x.dtype
    y = torch.empty_like(x)
    h_last = torch.empty(b, d, dtype=torch.float32, device=dev)
    taps = {
        "q_ifg": torch.empty(3, m, d, dtype=torch.int8, device=dev),
        "deq_ifg": torch.empty(3, m, dtype=torch.float32, device=dev),
        "z": torch.empty(m, 3 * d, dtype=dt, device=dev),
        "h": torch.empty(m, d, dtype=dt, device=dev),
        "q_o": torch.empty(m, d, dtype=torch.int8, device=dev),
        "deq_o": torch.empty(m, dtype=torch.float32, device=dev),
        "x1": torch.empty(m, d, dtype=dt, device=dev),
        "q_gate": torch.empty(m, d, dtype=torch.int8, device=dev),
        "deq_gate": torch.empty(m, dtype=torch.float32, device=dev),
        "gu": torch.empty(m, 2 * inner, dtype=dt, device=dev),
        "q_down": torch.empty(m, inner, dtype=torch.int8, device=dev),
        "deq_down": torch.empty(m, dtype=torch.float32, device=dev),
        "v": torch.empty(m, inner, dtype=dt, device=dev),
    }
    tc = BlockTapsC(**{k: v.data_ptr() for k, v in taps.items()})
    ws = workspace(MMF_OP_BLOCK, m, block.d, inner, 1, dev)
    bw = block.c()
    _check(lib().mmf_block_fwd_taps(ctypes.byref(bw), x.data_ptr(), _dt(dt), b, t, _ptr(h0), y.data_ptr(),
                                    h_last.data_ptr(), ctypes.byref(tc), ws.data_ptr(), ws.numel(), _stream(dev)),
           "mmf_block_fwd_taps")
    return y, h_last, taps


def _decode_shapes(blocks: list[Block], d: int, b: int, state: torch.Tensor) -> None:
    if not blocks:
        raise ValueError("no blocks")
    if d != blocks[0].d:
        raise ValueError(f"x: hidden size {d}, the blocks' is {blocks[0].d}")
    _f32(state, (len(blocks), b, d), "state")


def decode_step(blocks: list[Block], x: torch.Tensor, state: torch.Tensor, out: torch.Tensor | None = None):
    """mmf_decode_step: x [b, d] through every block with state [L, b, d] float32 updated in place."""
    _dev(x)
    b, d = x.shape
    _decode_shapes(blocks, d, b, state)
    if out is not None and (tuple(out.shape) != (b, d) or out.dtype != x.dtype or out is x):
        raise ValueError("out: needs x's shape and dtype and may not be x")
    y = _dev(out) if out is not None else torch.empty_like(x)
    ws = workspace(MMF_OP_DECODE, b, blocks[0].d, blocks[0].inner, len(blocks), x.device)
    arr = _blocks_array(blocks)
    _check(lib().mmf_decode_step(arr, len(blocks), x.data_ptr(), _dt(x.dtype), b, state.data_ptr(), y.data_ptr(),
                                 ws.data_ptr(), ws.numel(), _stream(x.device)), "mmf_decode_step")
    return y


def decode_step_taps(blocks: list[Block], x: torch.Tensor, state: torch.Tensor):
    """mmf_decode_step_taps: decode_step plus every layer's intermediates (see mmf_decode_taps).
    Returns (y, taps) with taps a list (one dict of tensors per layer)."""
    _dev(x)
    b, d = x.shape
    _decode_shapes(blocks, d, b, state)
    inner, dev, dt = blocks[0].inner, x.device, x.dtype
    y = torch.empty_like(x)
    taps = []
    for _ in blocks:
        taps.append({
            "q_ifg": torch.empty(3, b, d, dtype=torch.int8, device=dev),
            "deq_ifg": torch.empty(3, b, dtype=torch.float32, device=dev),
            "z": torch.empty(b, 3 * d, dtype=torch.float32, device=dev),
            "h": torch.empty(b, d, dtype=torch.float32, device=dev),
            "q_o": torch.empty(b, d, dtype=torch.int8, device=dev),
            "deq_o": torch.empty(b, dtype=torch.float32, device=dev),
            "x1": torch.empty(b, d, dtype=dt, device=dev),
            "q_gate": torch.empty(b, d, dtype=torch.int8, device=dev),
            "deq_gate": torch.empty(b, dtype=torch.float32, device=dev),
            "gu": torch.full((b, 2 * inner), float("nan"), dtype=dt, device=dev),
            "v": torch.full((b, inner), float("nan"), dtype=dt, device=dev),
            "q_down": torch.empty(b, inner, dtype=torch.int8, device=dev),
            "deq_down": torch.empty(b, dtype=torch.float32, device=dev),
            "y": torch.empty(b, d, dtype=dt, device=dev),
        })
    arr_t = (DecodeTapsC * len(blocks))(*[DecodeTapsC(**{k: v.data_ptr() for k, v in t.items()}) for t in taps])
    ws = workspace(MMF_OP_DECODE, b, blocks[0].d, inner, len(blocks), dev)
    arr = _blocks_array(blocks)
    _check(lib().mmf_decode_step_taps(arr, len(blocks), x.data_ptr(), _dt(dt), b, state.data_ptr(), y.data_ptr(),
                                      arr_t, ws.data_ptr(), ws.numel(), _stream(dev)), "mmf_decode_step_taps")
    return y, taps


def decode_path(b: int, d: int, inner: int) -> int:
    """mmf_decode_path_for: the path (MMF_DECODE_FUSED / SKINNY / BLOCK) a decode step of b rows
    takes under the current settings."""
    return int(lib().mmf_decode_path_for(b, d, inner))


def set_decode_path(path: int) -> None:
    """mmf_set_decode_path: MMF_DECODE_AUTO, _FUSED, _SKINNY or _BLOCK (process-wide)."""
    _check(lib().mmf_set_decode_path(path), "mmf_set_decode_path")


def decode_fused(b: int, d: int, inner: int) -> bool:
    """Whether a decode step of b rows takes the fused four-launch CUDA-core path."""
    return decode_path(b, d, inner) == MMF_DECODE_FUSED


def embed_gather(ids: torch.Tensor, table: torch.Tensor) -> torch.Tensor:
    """mmf_embed_gather: rows of table [vocab, d] for int32 ids."""
    _i32(ids, "ids")
    _dev(table)
    out = torch.empty(*ids.shape, table.shape[1], dtype=table.dtype, device=table.device)
    _check(lib().mmf_embed_gather(ids.data_ptr(), ids.numel(), table.data_ptr(), _dt(table.dtype), table.shape[0],
                                  table.shape[1], out.data_ptr(), _stream(table.device)), "mmf_embed_gather")
    return out


def lm_head_argmax(x: torch.Tensor, norm_w: torch.Tensor | None, table: torch.Tensor, eps: float = 1e-8,
                   want_logits: bool = False, ids_out: torch.Tensor | None = None):
    """mmf_lm_head_argmax: greedy next token ids [b] (int32) of x [b, d] through the final
    RMSNorm and the tied head `table` [vocab, d]; with want_logits also the logits [b, vocab]."""
    _dev(x)
    _dev(table)
    b, d = x.shape
    if table.dim() != 2 or table.shape[1] != d:
        raise ValueError(f"table: expected [vocab, {d}], got {tuple(table.shape)}")
    _f32(norm_w, (d,), "norm_w")
    if ids_out is not None and (_i32(ids_out, "ids_out").numel() != b):
        raise ValueError(f"ids_out: expected {b} int32 entries")
    vocab = table.shape[0]
    ids = ids_out if ids_out is not None else torch.empty(b, dtype=torch.int32, device=x.device)
    logits = torch.empty(b, vocab, dtype=torch.float32, device=x.device) if want_logits else None
    ws = workspace(MMF_OP_HEAD, 0, d, vocab, 0, x.device)
    _check(lib().mmf_lm_head_argmax(x.data_ptr(), _dt(x.dtype), b, d, norm_w.data_ptr() if norm_w is not None else None,
                                    eps, table.data_ptr(), _dt(table.dtype), vocab, ids.data_ptr(),
                                    logits.data_ptr() if logits is not None else None, ws.data_ptr(), ws.numel(),
                                    _stream(x.device)), "mmf_lm_head_argmax")
    return (ids, logits) if want_logits else ids


def stack_fwd(blocks: list[Block], ids: torch.Tensor, table: torch.Tensor, want_state: bool = False,
              out: torch.Tensor | None = None):
    """mmf_stack_fwd: embedding gather + every block on ids [b, t] int32. Returns (y, h_last or None)."""
    _i32(ids, "ids")
    _dev(table)
    b, t = ids.shape
    d = table.shape[1]
    if not blocks or blocks[0].d != d:
        raise ValueError(f"table: hidden size {d} does not match the blocks")
    if out is not None and (tuple(out.shape) != (b, t, d) or out.dtype != table.dtype):
        raise ValueError(f"out: expected {table.dtype} of shape {(b, t, d)}")
    y = _dev(out) if out is not None else torch.empty(b, t, d, dtype=table.dtype, device=table.device)
    h_last = torch.empty(len(blocks), b, d, dtype=torch.float32, device=table.device) if want_state else None
    ws = workspace(MMF_OP_STACK, b * t, blocks[0].d, blocks[0].inner, len(blocks), table.device)
    arr = _blocks_array(blocks)
    _check(lib().mmf_stack_fwd(arr, len(blocks), ids.data_ptr(), b, t, table.data_ptr(), table.shape[0],
                               _dt(table.dtype), y.data_ptr(), _ptr(h_last), ws.data_ptr(), ws.numel(),
                               _stream(table.device)), "mmf_stack_fwd")
    return y, h_last


def sync_status(device: torch.device | str | None = None) -> int:
    """mmf_sync_status on the current stream: synchronises and returns the status (does not raise)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    return int(lib().mmf_sync_status(_stream(dev)))


_gemm_path = MMF_GEMM_AUTO


def set_gemm_path(path: int) -> None:
    global _gemm_path
    _check(lib().mmf_set_gemm_path(path), "mmf_set_gemm_path")
    _gemm_path = path


def glu_fused(m: int, inner: int) -> bool:
    """Whether a block forward on m tokens forms SiLU(gate) * up in gate_proj's epilogue (taps
    then carry ``v`` instead of ``gu``): the tensor-core engine with inner % 64 == 0."""
    tensor = _gemm_path == MMF_GEMM_TENSOR or (_gemm_path == MMF_GEMM_AUTO and m >= 8)
    return tensor and inner % 64 == 0


KERNEL_CLASSES = {"gemm_tc": 0, "gemm_simt": 1, "norm_quant": 2, "scan": 3, "other": 4}


def launch_count() -> int:
    return int(lib().mmf_launch_count())


def timing_enable(on: bool) -> None:
    _check(lib().mmf_timing_enable(1 if on else 0), "mmf_timing_enable")


def timing_read(cls: str) -> tuple[int, float, float]:
    """(launches, total device ms, total algorithmic work) of one kernel class since the last read."""
    n, ms, wk = ctypes.c_int64(), ctypes.c_double(), ctypes.c_double()
    _check(lib().mmf_timing_read(KERNEL_CLASSES[cls], ctypes.byref(n), ctypes.byref(ms), ctypes.byref(wk)),
           "mmf_timing_read")
    return n.value, ms.value, wk.value


def set_wait_limit(microseconds: int) -> None:
    """mmf_set_wait_limit: the cap of every bounded in-kernel wait (0 restores the default)."""
    _check(lib().mmf_set_wait_limit(microseconds), "mmf_set_wait_limit")
