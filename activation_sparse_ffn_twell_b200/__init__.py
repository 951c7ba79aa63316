"""Activation-sparse ReLU FFN forward pass with on-the-fly TwELL packing, for B200.

Thin Python binding over the C ABI in ``include/twell.h`` (library
``libtwell_b200.so``, built in-tree for sm_100a).  This module only marshals
arguments: torch supplies device memory and the current stream, and every step of
the layer runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing, importing the ops raises.

    y, a = twell_ffn_forward(x, W_up, b, W_down, tile_w=128, ell_w=16)

Names follow the method: TwELL (Tile-wise ELLPACK) packs each token's hidden
nonzeros per fixed-width tile of hidden columns into ELL slots (value, in-tile
index); (token, tile) pairs that overflow the ELL width keep their dense segment
in a small dense backup ("Sparser, Faster, Lighter Transformer Language Models",
upppp.jp 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

__all__ = [
    "TwellError", "TwELL", "lib", "library_path", "workspace_bytes",
    "twell_pack", "twell_up_pack", "twell_up_pack_stats", "twell_spmm", "twell_ffn_forward",
    "twell_ffn_backward", "twell_spmm_token_overflow", "read_status",
    "DOWN_MODES", "STATUS", "default_ovf_capacity", "down_schedule",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtwell_b200.so")

STATUS = {0: "TWELL_OK", 1: "TWELL_ERR_INVALID_ARG", 2: "TWELL_ERR_UNSUPPORTED",
          3: "TWELL_ERR_OVERFLOW_CAPACITY", 4: "TWELL_ERR_CUDA", 5: "TWELL_ERR_TIMEOUT",
          6: "TWELL_ERR_WORKSPACE"}
DOWN_MODES = {"auto": 0, "gather": 1, "mma": 2, "sparse": 3}


class TwellError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS.get(self.code, self.code)} "
                         f"({_lib().twell_status_string(self.code).decode()})")


class _Matrix(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("tile_w", ctypes.c_int32),
                ("ell_w", ctypes.c_int32), ("vals", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("nnz", ctypes.c_void_p), ("ovf_capacity", ctypes.c_int32),
                ("n_ovf", ctypes.c_void_p), ("ovf_pos", ctypes.c_void_p),
                ("ovf_dense", ctypes.c_void_p), ("status", ctypes.c_void_p)]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "twell_version": (ctypes.c_int, []),
    "twell_status_string": (ctypes.c_char_p, [_I]),
    "twell_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "twell_pack": (_I, [_P, _I, _I, _I, _I, _I, ctypes.POINTER(_Matrix), _P, ctypes.c_size_t, _P]),
    "twell_up_pack": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(_Matrix), _P, _P,
                           ctypes.c_size_t, _P]),
    "twell_up_pack_stats": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(_Matrix), _P,
                                 _P, _P, ctypes.c_size_t, _P]),
    "twell_spmm": (_I, [ctypes.POINTER(_Matrix), _P, _I, _P, _I, _P, ctypes.c_size_t, _P]),
    "twell_ffn_forward": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(_Matrix), _P,
                               _I, _P, ctypes.c_size_t, _P]),
    "twell_read_status": (_I, [ctypes.POINTER(_Matrix), _P, ctypes.POINTER(ctypes.c_int32)]),
    "twell_pack_noalloc": (_I, [_P, _I, _I, _I, _I, _I, ctypes.POINTER(_Matrix), _P]),
    "twell_selftest_bounded_wait": (_I, [_P, _P, _P]),
    "twell_down_schedule": (_I, [_I, _I, _I, _I, _I, _I, _P, _I]),
    "twell_backward_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "twell_token_overflow_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "twell_spmm_token_overflow": (_I, [ctypes.POINTER(_Matrix), _P, _I, _P, _I, _P, _P,
                                       ctypes.c_size_t, _P]),
    "twell_ffn_backward": (_I, [_P, _P, _P, ctypes.POINTER(_Matrix), _P, _I, _I, _I, _P, _P, _P, _P,
                                _P, ctypes.c_size_t, _P]),
}


def library_path() -> str:
    return _LIB_PATH


def _lib():
    """Load libtwell_b200.so (raises if it was not built: no fallback exists)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(
                f"{_LIB_PATH} is missing; build it with "
                "`python -m activation_sparse_ffn_twell_b200.build` (needs nvcc)")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


lib = _lib


def _check(code: int, where: str):
    if code != 0:
        raise TwellError(code, where)


def _torch():
    import torch
    return torch


def _stream_handle(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _need_bf16(name, t, shape=None):
    torch = _torch()
    if t is None:
        return
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def default_ovf_capacity(M: int, n_tiles: int) -> int:
    """Backup capacity used when the caller gives none: 1/8 of all (token, tile)
    pairs, at least 4096 pairs, never more than all of them."""
    return min(M * n_tiles, max(4096, (M * n_tiles) // 8))


@dataclasses.dataclass
class TwELL:
    """A TwELL matrix in device memory (torch tensors) plus its dense backup."""

    M: int
    d_ff: int
    tile_w: int
    ell_w: int
    ovf_capacity: int
    vals: "object"       # [M, T, E] bfloat16
    idx: "object"        # [M, T, E] uint8
    nnz: "object"        # [M, T] int16 (bit pattern of the uint16 count)
    n_ovf: "object"      # [1] int32
    ovf_pos: "object"    # [cap] int32
    ovf_dense: "object"  # [cap, tile_w] bfloat16
    status: "object"     # [1] int32

    @property
    def n_tiles(self) -> int:
        return self.d_ff // self.tile_w

    @staticmethod
    def allocate(M: int, d_ff: int, tile_w: int, ell_w: int, ovf_capacity: Optional[int] = None,
                 device=None) -> "TwELL":
        torch = _torch()
        T = d_ff // tile_w
        if ovf_capacity is None:
            ovf_capacity = default_ovf_capacity(M, T)
        dev = device if device is not None else torch.device("cuda")
        cap_alloc = max(ovf_capacity, 1)
        return TwELL(M, d_ff, tile_w, ell_w, ovf_capacity,
                     torch.empty((M, T, ell_w), dtype=torch.bfloat16, device=dev),
                     torch.empty((M, T, ell_w), dtype=torch.uint8, device=dev),
                     torch.empty((M, T), dtype=torch.int16, device=dev),
                     torch.zeros(4, dtype=torch.int32, device=dev)[:1],
                     torch.empty(cap_alloc, dtype=torch.int32, device=dev),
                     torch.empty((cap_alloc, tile_w), dtype=torch.bfloat16, device=dev),
                     torch.zeros(4, dtype=torch.int32, device=dev)[:1])

    def cstruct(self) -> _Matrix:
        return _Matrix(self.M, self.d_ff, self.tile_w, self.ell_w, _ptr(self.vals), _ptr(self.idx),
                       _ptr(self.nnz), self.ovf_capacity, _ptr(self.n_ovf), _ptr(self.ovf_pos),
                       _ptr(self.ovf_dense), _ptr(self.status))

    def nnz_u16(self):
        """nnz as int32 (the stored bits are uint16)."""
        return self.nnz.to(_torch().int32) & 0xFFFF


def workspace_bytes(M, d_model, d_ff, tile_w, ell_w, gated, ovf_capacity) -> int:
    return int(_lib().twell_workspace_bytes(M, d_model, d_ff, tile_w, ell_w, int(bool(gated)),
                                            ovf_capacity))


_WS_CACHE = {}


def _workspace(nbytes: int, device):
    torch = _torch()
    key = (str(device), torch.cuda.current_stream(device).cuda_stream)
    buf = _WS_CACHE.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _WS_CACHE[key] = buf
    return buf


def twell_pack(h, tile_w: int, ell_w: int, out: Optional[TwELL] = None,
               ovf_capacity: Optional[int] = None, stream=None) -> TwELL:
    """Dense bf16 h [M, d_ff] -> TwELL (+ dense backup)."""
    _need_bf16("h", h)
    M, f = h.shape
    a = out or TwELL.allocate(M, f, tile_w, ell_w, ovf_capacity, device=h.device)
    nb = workspace_bytes(M, 64, f, tile_w, ell_w, 0, a.ovf_capacity)
    ws = _workspace(nb, h.device)
    m = a.cstruct()
    _check(_lib().twell_pack(_ptr(h), M, f, h.stride(0), tile_w, ell_w, ctypes.byref(m), _ptr(ws),
                             ws.numel(), _stream_handle(stream)), "twell_pack")
    return a


def twell_up_pack(x, W_up, b=None, W_gate=None, *, tile_w: int, ell_w: int,
                  out: Optional[TwELL] = None, ovf_capacity: Optional[int] = None, z_debug=None,
                  stream=None) -> TwELL:
    """Fused up (and gate) projection + activation + TwELL packing."""
    M, d = x.shape
    f = W_up.shape[0]
    _need_bf16("x", x); _need_bf16("W_up", W_up, (f, d)); _need_bf16("W_gate", W_gate, (f, d))
    _need_bf16("b", b, (f,))
    a = out or TwELL.allocate(M, f, tile_w, ell_w, ovf_capacity, device=x.device)
    nb = workspace_bytes(M, d, f, tile_w, ell_w, W_gate is not None, a.ovf_capacity)
    ws = _workspace(nb, x.device)
    m = a.cstruct()
    _check(_lib().twell_up_pack(_ptr(x), _ptr(W_up), _ptr(W_gate), _ptr(b), M, d, f, tile_w,
                                ell_w, ctypes.byref(m), _ptr(z_debug), _ptr(ws), ws.numel(),
                                _stream_handle(stream)), "twell_up_pack")
    return a


def twell_up_pack_stats(x, W_up, b=None, W_gate=None, *, tile_w: int, ell_w: int,
                        out: Optional[TwELL] = None, ovf_capacity: Optional[int] = None,
                        stream=None):
    """twell_up_pack plus per-token activation statistics.

    Returns (TwELL, l1 [M] fp32 = sum of |h| per token, nnz_row [M] int32)."""
    torch = _torch()
    M, d = x.shape
    f = W_up.shape[0]
    _need_bf16("x", x); _need_bf16("W_up", W_up, (f, d)); _need_bf16("W_gate", W_gate, (f, d))
    _need_bf16("b", b, (f,))
    a = out or TwELL.allocate(M, f, tile_w, ell_w, ovf_capacity, device=x.device)
    l1 = torch.empty((M,), dtype=torch.float32, device=x.device)
    nnz_row = torch.empty((M,), dtype=torch.int32, device=x.device)
    nb = workspace_bytes(M, d, f, tile_w, ell_w, W_gate is not None, a.ovf_capacity)
    ws = _workspace(nb, x.device)
    m = a.cstruct()
    _check(_lib().twell_up_pack_stats(_ptr(x), _ptr(W_up), _ptr(W_gate), _ptr(b), M, d, f, tile_w,
                                      ell_w, ctypes.byref(m), _ptr(l1), _ptr(nnz_row), _ptr(ws),
                                      ws.numel(), _stream_handle(stream)), "twell_up_pack_stats")
    return a, l1, nnz_row


def twell_spmm(a: TwELL, W_down, mode: str = "auto", y=None, stream=None):
    """y = h W_down from the packed form only.  Returns y [M, d_model] bf16."""
    torch = _torch()
    f, d = W_down.shape
    _need_bf16("W_down", W_down, (a.d_ff, d))
    if y is None:
        y = torch.empty((a.M, d), dtype=torch.bfloat16, device=W_down.device)
    _need_bf16("y", y, (a.M, d))
    nb = workspace_bytes(a.M, d, a.d_ff, a.tile_w, a.ell_w, 0, a.ovf_capacity)
    ws = _workspace(nb, W_down.device)
    m = a.cstruct()
    _check(_lib().twell_spmm(ctypes.byref(m), _ptr(W_down), d, _ptr(y), DOWN_MODES[mode], _ptr(ws),
                             ws.numel(), _stream_handle(stream)), "twell_spmm")
    return y


def twell_ffn_forward(x, W_up, b, W_down, *, tile_w: int, ell_w: int, W_gate=None,
                      mode: str = "auto", out: Optional[TwELL] = None, y=None,
                      ovf_capacity: Optional[int] = None, stream=None):
    """The whole layer.  Returns (y [M, d_model] bf16, TwELL intermediate)."""
    torch = _torch()
    M, d = x.shape
    f = W_up.shape[0]
    _need_bf16("x", x); _need_bf16("W_up", W_up, (f, d)); _need_bf16("W_gate", W_gate, (f, d))
    _need_bf16("b", b, (f,)); _need_bf16("W_down", W_down, (f, d))
    a = out or TwELL.allocate(M, f, tile_w, ell_w, ovf_capacity, device=x.device)
    if y is None:
        y = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    _need_bf16("y", y, (M, d))
    nb = workspace_bytes(M, d, f, tile_w, ell_w, W_gate is not None, a.ovf_capacity)
    ws = _workspace(nb, x.device)
    m = a.cstruct()
    _check(_lib().twell_ffn_forward(_ptr(x), _ptr(W_up), _ptr(W_gate), _ptr(b), _ptr(W_down), M, d,
                                    f, tile_w, ell_w, ctypes.byref(m), _ptr(y), DOWN_MODES[mode],
                                    _ptr(ws), ws.numel(), _stream_handle(stream)),
           "twell_ffn_forward")
    return y, a


def twell_ffn_backward(x, W_up, W_down, h: TwELL, dY, *, ell_w_t: Optional[int] = None,
                       ovf_capacity_t: Optional[int] = None, stream=None):
    """Backward pass of the non-gated layer through the forward's TwELL `h`.

    Returns (dX [M, d] bf16, dW_up [f, d] bf16, db [f] fp32, dW_down [f, d] bf16).
    ell_w_t / ovf_capacity_t size the internal transposed TwELL (tiles of 128
    tokens); by default ell_w_t = the forward's ell_w and the capacity covers
    every (unit, token tile) pair."""
    torch = _torch()
    M, d = x.shape
    f = W_up.shape[0]
    _need_bf16("x", x); _need_bf16("W_up", W_up, (f, d)); _need_bf16("W_down", W_down, (f, d))
    _need_bf16("dY", dY, (M, d))
    et = ell_w_t or h.ell_w
    cap_t = ovf_capacity_t if ovf_capacity_t is not None else f * (M // 128)
    dX = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    dW_up = torch.empty((f, d), dtype=torch.bfloat16, device=x.device)
    dW_down = torch.empty((f, d), dtype=torch.bfloat16, device=x.device)
    db = torch.empty((f,), dtype=torch.float32, device=x.device)
    nb = _lib().twell_backward_workspace_bytes(M, d, f, h.tile_w, h.ell_w, h.ovf_capacity, et, cap_t)
    if nb == 0:
        raise TwellError(2, f"twell_ffn_backward (M={M}, d_ff={f}, tile_w={h.tile_w})")
    ws = _workspace(nb, x.device)
    m = h.cstruct()
    _check(_lib().twell_ffn_backward(_ptr(x), _ptr(W_up), _ptr(W_down), ctypes.byref(m), _ptr(dY), d,
                                     et, cap_t, _ptr(dX), _ptr(dW_up), _ptr(db), _ptr(dW_down),
                                     _ptr(ws), ws.numel(), _stream_handle(stream)),
           "twell_ffn_backward")
    return dX, dW_up, db, dW_down


def twell_spmm_token_overflow(a: TwELL, W_down, cap_tok: int, y=None, stream=None):
    """y = h W_down with the whole-token reading of the backup (tokens with any
    over-full tile run as a small dense product).  Returns (y, n_tok device int32)."""
    torch = _torch()
    f, d = W_down.shape
    _need_bf16("W_down", W_down, (a.d_ff, d))
    if y is None:
        y = torch.empty((a.M, d), dtype=torch.bfloat16, device=W_down.device)
    _need_bf16("y", y, (a.M, d))
    n_tok = torch.zeros((4,), dtype=torch.int32, device=W_down.device)
    nb = _lib().twell_token_overflow_workspace_bytes(a.M, d, a.d_ff, a.tile_w, a.ell_w, cap_tok)
    if nb == 0:
        raise TwellError(1, "twell_spmm_token_overflow")
    ws = _workspace(nb, W_down.device)
    m = a.cstruct()
    _check(_lib().twell_spmm_token_overflow(ctypes.byref(m), _ptr(W_down), d, _ptr(y), cap_tok,
                                            _ptr(n_tok), _ptr(ws), ws.numel(), _stream_handle(stream)),
           "twell_spmm_token_overflow")
    return y, n_tok[:1]


def read_status(a: TwELL, stream=None):
    """Synchronise and return (status code, true overflow count)."""
    n = ctypes.c_int32(0)
    m = a.cstruct()
    code = _lib().twell_read_status(ctypes.byref(m), _stream_handle(stream), ctypes.byref(n))
    return int(code), int(n.value)


def down_schedule(M: int, d_model: int, d_ff: int, tile_w: int, ell_w: int, num_sms: int):
    """The work split of the token-major tensor-core down-projection for these
    sizes on num_sms SMs, from the library's own planning code (host only).
    Returns None for shapes that do not take that kernel, else a dict with
    `split` (0 whole tiles, 1 split-K, 2 even deal of K chunks), `ctas`, `tiles`,
    `k_steps` and `segments`: (cta, tile, k0, k1, sharers, counter, slot) tuples."""
    fn = _lib().twell_down_schedule
    n = fn(M, d_model, d_ff, tile_w, ell_w, num_sms, None, 0)
    if n < 0:
        return None
    buf = (ctypes.c_int32 * n)()
    fn(M, d_model, d_ff, tile_w, ell_w, num_sms, ctypes.cast(buf, ctypes.c_void_p), n)
    v = list(buf)
    segs = [tuple(v[i:i + 7]) for i in range(4, n, 7)]
    return {"split": v[0], "ctas": v[1], "tiles": v[2], "k_steps": v[3], "segments": segs}

