"""Thin ctypes binding of the C ABI in ``include/csa.h`` (``libcsa.so``).

Argument marshalling only: tensors are torch CUDA tensors, passed by device
pointer; every step of the path runs in the library's CUDA kernels. The
functions keep the C names. A non-OK status raises ``CsaError``.

The library is loaded from the package directory (built in-tree by
``long_context_sparse_07_b200.build``). There is no fallback: if it is missing
or fails to load, import of this module's functions raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

CSA_F32, CSA_BF16, CSA_E4M3, CSA_E2M1 = 0, 1, 2, 3
STATUS = {0: "CSA_OK", -1: "CSA_ERR_INVALID_ARG", -2: "CSA_ERR_UNSUPPORTED",
          -3: "CSA_ERR_CUDA", -4: "CSA_ERR_TIMEOUT", -5: "CSA_ERR_BOUNDS"}

# every symbol that include/csa.h declares
EXPORTS = ("csa_abi_version", "csa_status_string", "csa_last_message", "csa_compress_kv",
           "csa_indexer_scores", "csa_topk", "csa_topk_workspace_size", "csa_indexer_topk",
           "csa_indexer_topk_workspace_size", "csa_indexer_topk_launches", "csa_sparse_mqa",
           "hca_dense_mqa", "csa_mqa_workspace_size", "csa_sparse_mqa_noalloc",
           "csa_noalloc_scratch_bytes", "csa_norm_rope", "csa_grouped_out_proj",
           "csa_debug_wait_probe", "csa_get_error")


class CsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS.get(status, status), message))
        self.status = status


class _Entries(ctypes.Structure):
    _fields_ = [("body", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("rope", ctypes.c_void_p), ("c", ctypes.c_int), ("rope_dims", ctypes.c_int),
                ("scale_group", ctypes.c_int), ("dt", ctypes.c_int)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_S = ctypes.c_size_t
_lib = None


def load(path: str = LIB_PATH):
    """Load ``libcsa.so`` and declare its signatures (raises if missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libcsa.so not built: run `python -m long_context_sparse_07_b200.build`")
    L = ctypes.CDLL(path)
    L.csa_abi_version.restype = _I
    L.csa_status_string.restype = ctypes.c_char_p
    L.csa_status_string.argtypes = [_I]
    L.csa_last_message.restype = ctypes.c_char_p
    L.csa_compress_kv.restype = _I
    L.csa_compress_kv.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _Entries, _P]
    L.csa_indexer_scores.restype = _I
    L.csa_indexer_scores.argtypes = [_P, _P, _P, _Entries, _P, _I, _I64, _I64, _I, _I, _I, _I,
                                     _P, _I64, _P]
    L.csa_topk.restype = _I
    L.csa_topk.argtypes = [_P, _I64, _I64, _I64, _P, _I, _I, _P, _P, _S, _P]
    L.csa_topk_workspace_size.restype = _S
    L.csa_topk_workspace_size.argtypes = [_I64, _I64, _I]
    L.csa_indexer_topk.restype = _I
    L.csa_indexer_topk.argtypes = [_P, _P, _P, _Entries, _P, _I, _I64, _I64, _I, _I, _I, _I, _I,
                                   _P, _P, _S, _P]
    L.csa_indexer_topk_workspace_size.restype = _S
    L.csa_indexer_topk_workspace_size.argtypes = [_I, _I64, _I64, _I, _I, _I, _I]
    L.csa_indexer_topk_launches.restype = _I
    L.csa_indexer_topk_launches.argtypes = [_I, _I64, _I64, _I, _I, _I, _I]
    L.csa_sparse_mqa.restype = _I
    L.csa_sparse_mqa.argtypes = [_P, _I, _Entries, _I64, _I, _P, _I, _P, _I64, _P, _I, _P, _P,
                                 _I, _I64, _I, _F, _P, _P, _P, _S, _P]
    L.hca_dense_mqa.restype = _I
    L.hca_dense_mqa.argtypes = [_P, _I, _Entries, _I64, _I, _P, _I64, _P, _I, _P, _P, _I, _I64,
                                _I, _F, _P, _P, _P, _S, _P]
    L.csa_mqa_workspace_size.restype = _S
    L.csa_mqa_workspace_size.argtypes = [_I, _I64, _I, _I, _I64]
    L.csa_sparse_mqa_noalloc.restype = _I
    L.csa_sparse_mqa_noalloc.argtypes = [_P, _I, _Entries, _I64, _I, _P, _I, _P, _I64, _P, _I, _P,
                                         _P, _I, _I64, _I, _F, _P, _P, _P]
    L.csa_noalloc_scratch_bytes.restype = _S
    L.csa_noalloc_scratch_bytes.argtypes = []
    L.csa_norm_rope.restype = _I
    L.csa_norm_rope.argtypes = [_P, _I, _P, _I64, _I, _I, _I, _P, _I64, _I64, _I, _F, _F, _P]
    L.csa_grouped_out_proj.restype = _I
    L.csa_grouped_out_proj.argtypes = [_P, _P, _P, _I64, _I, _I, _I, _I, _I, _P, _P, _P]
    L.csa_debug_wait_probe.restype = _I
    L.csa_debug_wait_probe.argtypes = [ctypes.c_uint64, _P]
    L.csa_get_error.restype = _I
    L.csa_get_error.argtypes = [ctypes.c_char_p, _S]
    _lib = L
    return L


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CSA_F32
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return CSA_E4M3
    raise TypeError("unsupported dtype %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(st: int):
    if st != 0:
        msg = load().csa_last_message().decode()
        raise CsaError(st, msg)


@dataclasses.dataclass
class Entries:
    """A table of KV entries (``csa_entries``): plain [rows, c] f32/bf16, or
    the fp8 layout (e4m3 body [rows, c - rope_dims] with per-group float32
    scales, optional bf16 rope part [rows, rope_dims]), or the fp4 layout of
    indexer keys (fp4=True: uint8 body [rows, c / 2] of packed e2m1 codes,
    uint8 block exponents [rows, c / 32] in ``scale``, scale_group 32)."""
    body: torch.Tensor
    c: int
    scale: Optional[torch.Tensor] = None
    rope: Optional[torch.Tensor] = None
    rope_dims: int = 0
    scale_group: int = 0
    fp4: bool = False

    def struct(self) -> _Entries:
        dt = CSA_E2M1 if self.fp4 else dtype_code(self.body)
        return _Entries(_ptr(self.body), _ptr(self.scale), _ptr(self.rope), self.c,
                        self.rope_dims, self.scale_group, dt)


def csa_abi_version() -> int:
    return load().csa_abi_version()


def csa_compress_kv(Ca, Cb, Za, Zb, Ba, Bb, m: int, overlap: bool, out: Entries, stream=None):
    n, c = Ca.shape[0], Ca.shape[-1]
    _check(load().csa_compress_kv(_ptr(Ca), _ptr(Cb), _ptr(Za), _ptr(Zb), _ptr(Ba), _ptr(Bb),
                                  n, c, m, int(bool(overlap)), dtype_code(Ca), out.struct(),
                                  _stream(stream)))


def csa_indexer_scores(qI, qI_scale, wI, kI: Entries, q_pos, m: int, scores, E: int,
                       stream=None):
    B, n_q, hI, cI = qI.shape
    _check(load().csa_indexer_scores(_ptr(qI), _ptr(qI_scale), _ptr(wI), kI.struct(),
                                     _ptr(q_pos), B, n_q, E, hI, cI, m, dtype_code(qI),
                                     _ptr(scores), scores.shape[-1], _stream(stream)))


def csa_topk_workspace_size(rows: int, E: int, k: int) -> int:
    return int(load().csa_topk_workspace_size(rows, E, k))


def csa_topk(scores, q_pos, m: int, k: int, idx, E: Optional[int] = None, workspace=None,
             stream=None):
    ld = scores.shape[-1]
    rows = scores.numel() // ld if ld else 0
    E = ld if E is None else E
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().csa_topk(_ptr(scores), rows, E, ld, _ptr(q_pos), m, k, _ptr(idx),
                           _ptr(workspace), ws, _stream(stream)))


def csa_indexer_topk_workspace_size(B: int, n_q: int, E: int, hI: int, cI: int, k: int,
                                    dt) -> int:
    code = dt if isinstance(dt, int) else dtype_code(dt)
    return int(load().csa_indexer_topk_workspace_size(B, n_q, E, hI, cI, k, code))


def csa_indexer_topk_launches(B: int, n_q: int, E: int, hI: int, cI: int, k: int, dt) -> int:
    """Kernel launches of csa_indexer_topk for these shapes (6: candidate path)."""
    code = dt if isinstance(dt, int) else dtype_code(dt)
    return int(load().csa_indexer_topk_launches(B, n_q, E, hI, cI, k, code))


def csa_indexer_topk(qI, qI_scale, wI, kI: Entries, q_pos, m: int, k: int, idx, E: int,
                     workspace=None, stream=None):
    """Indexer scores and top-k in one call: idx [B * n_q, k] as
    csa_indexer_scores followed by csa_topk would give."""
    B, n_q, hI, cI = qI.shape
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().csa_indexer_topk(_ptr(qI), _ptr(qI_scale), _ptr(wI), kI.struct(), _ptr(q_pos),
                                   B, n_q, E, hI, cI, m, dtype_code(qI), k, _ptr(idx),
                                   _ptr(workspace), ws, _stream(stream)))


def csa_mqa_workspace_size(B: int, n_q: int, h: int, c: int, max_keys: int) -> int:
    return int(load().csa_mqa_workspace_size(B, n_q, h, c, max_keys))


def csa_sparse_mqa(q, kv: Entries, E: int, m: int, idx, k: int, kwin, win_pos0, n_win: int,
                   q_pos, sink, scale: float, out, lse=None, workspace=None, stream=None):
    B, n_q, h, c = q.shape
    win_rows = kwin.shape[-2] if kwin is not None else 0
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().csa_sparse_mqa(_ptr(q), dtype_code(q), kv.struct(), E, m, _ptr(idx), k,
                                 _ptr(kwin), win_rows, _ptr(win_pos0), n_win, _ptr(q_pos),
                                 _ptr(sink), B, n_q, h, scale, _ptr(out), _ptr(lse),
                                 _ptr(workspace), ws, _stream(stream)))


def csa_sparse_mqa_noalloc(q, kv: Entries, E: int, m: int, idx, k: int, kwin, win_pos0,
                           n_win: int, q_pos, sink, scale: float, out, lse=None, stream=None):
    """csa_sparse_mqa with the library's fixed device scratch instead of a
    workspace: for callers that cannot allocate device memory."""
    B, n_q, h, c = q.shape
    win_rows = kwin.shape[-2] if kwin is not None else 0
    _check(load().csa_sparse_mqa_noalloc(_ptr(q), dtype_code(q), kv.struct(), E, m, _ptr(idx), k,
                                         _ptr(kwin), win_rows, _ptr(win_pos0), n_win,
                                         _ptr(q_pos), _ptr(sink), B, n_q, h, scale, _ptr(out),
                                         _ptr(lse), _stream(stream)))


def csa_noalloc_scratch_bytes() -> int:
    return int(load().csa_noalloc_scratch_bytes())


def hca_dense_mqa(q, kv: Entries, E: int, m: int, kwin, win_pos0, n_win: int, q_pos, sink,
                  scale: float, out, lse=None, workspace=None, stream=None):
    B, n_q, h, c = q.shape
    win_rows = kwin.shape[-2] if kwin is not None else 0
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().hca_dense_mqa(_ptr(q), dtype_code(q), kv.struct(), E, m, _ptr(kwin),
                                win_rows, _ptr(win_pos0), n_win, _ptr(q_pos), _ptr(sink), B,
                                n_q, h, scale, _ptr(out), _ptr(lse), _ptr(workspace), ws,
                                _stream(stream)))


def csa_norm_rope(x, rope_dims: int, pos=None, pos_mul: int = 1, pos_add: int = 0, gamma=None,
                  normalise: bool = True, eps: float = 1e-6, base: float = 10000.0, stream=None):
    """In-place RMSNorm and partial RoPE of x [rows, heads, c] or [rows, c]."""
    c = x.shape[-1]
    rows = x.shape[0]
    heads = x.numel() // (rows * c) if rows else 1
    _check(load().csa_norm_rope(_ptr(x), dtype_code(x), _ptr(gamma), rows, heads, c, rope_dims,
                                _ptr(pos), pos_mul, pos_add, int(bool(normalise)), eps, base,
                                _stream(stream)))


def csa_grouped_out_proj(o, Wg, Wo, g: int, u, out, stream=None):
    """Grouped output projection: o [n, h, c] -> u [n, g dg] -> out [n, d]."""
    n, h, c = o.shape
    dg = Wg.shape[0] // g
    d = Wo.shape[0]
    _check(load().csa_grouped_out_proj(_ptr(o), _ptr(Wg), _ptr(Wo), n, h, c, g, dg, d, _ptr(u),
                                       _ptr(out), _stream(stream)))


def csa_debug_wait_probe(limit_ns: int, stream=None):
    """Launch one bounded device wait that nothing completes; the next
    csa_get_error() reports CSA_ERR_TIMEOUT."""
    _check(load().csa_debug_wait_probe(int(limit_ns), _stream(stream)))


def csa_get_error() -> int:
    """Synchronise, read and clear the device error word; raises on error."""
    buf = ctypes.create_string_buffer(256)
    st = load().csa_get_error(buf, 256)
    if st != 0:
        raise CsaError(st, buf.value.decode())
    return st
