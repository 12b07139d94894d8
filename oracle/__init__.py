"""ctypes front end of the float64 CPU oracle (``csa_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``; the product package never
imports it. It shares no code with the CUDA library.

Inputs arrive as torch tensors or numpy arrays in their storage dtypes and are
decoded exactly to float64 here (float32 and bfloat16 widen exactly; e4m3
codes are decoded by the C oracle from the format's definition and multiplied
by their scales there). Every step of the method runs in ``csa_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libcsa_oracle.so")
_lib = None
_lock = threading.Lock()

_d = ctypes.POINTER(ctypes.c_double)
_f = ctypes.POINTER(ctypes.c_float)
_u8 = ctypes.POINTER(ctypes.c_uint8)
_i32 = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.POINTER(ctypes.c_int64)
_I64 = ctypes.c_int64
_I = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE arithmetic, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.oracle_visible.restype = _I64
            L.oracle_visible.argtypes = [_I64, _I, _I64]
            L.oracle_e4m3_value.restype = ctypes.c_double
            L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_code.restype = ctypes.c_uint8
            L.oracle_e4m3_code.argtypes = [ctypes.c_double]
            L.oracle_quantize_e4m3.argtypes = [_d, _I64, _I, _I, _u8, _f]
            L.oracle_dequantize.argtypes = [_u8, _f, _I64, _I, _I, _d]
            L.oracle_e2m1_value.restype = ctypes.c_double
            L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
            L.oracle_e2m1_code.restype = ctypes.c_uint8
            L.oracle_e2m1_code.argtypes = [ctypes.c_double]
            L.oracle_quantize_e2m1.argtypes = [_d, _I64, _I, _u8, _u8]
            L.oracle_dequantize_e2m1.argtypes = [_u8, _u8, _I64, _I, _d]
            L.oracle_compress.argtypes = [_d, _d, _d, _d, _d, _d, _I64, _I, _I, _I, _d]
            L.oracle_indexer.argtypes = [_d, _d, _d, _i64, _I, _I64, _I64, _I, _I, _I, _d]
            L.oracle_topk.argtypes = [_d, _I64, _I64, _I64, _i64, _I, _I, _i32]
            L.oracle_norm_rope.argtypes = [_d, _I64, _I, _I, _I, _i64, _d, _I, ctypes.c_double,
                                           ctypes.c_double]
            L.oracle_attend.restype = _I
            L.oracle_attend.argtypes = [_d, _d, _I64, _i32, _I, _I, _d, _I64, _i64, _I,
                                        _i64, _d, _I, _I64, _I, _I, ctypes.c_double, _d, _d]
            _lib = L
    return _lib


# ----------------------------------------------------------------------------
# decoding of storage dtypes


def f64(x) -> np.ndarray:
    """Exact float64 copy of a float32 / bfloat16 / float64 tensor or array."""
    if isinstance(x, torch.Tensor):
        if x.dtype in (torch.float8_e4m3fn, torch.uint8):
            raise TypeError("e4m3 codes need their scales: use dequantize()")
        return np.ascontiguousarray(x.detach().cpu().to(torch.float64).numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _codes(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.uint8).numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


# ----------------------------------------------------------------------------
# steps


def visible(t: int, m: int, E: int) -> int:
    return int(lib().oracle_visible(int(t), int(m), int(E)))


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(int(code)))


def e4m3_code(x: float) -> int:
    return int(lib().oracle_e4m3_code(float(x)))


def quantize_e4m3(x, group: int) -> Tuple[np.ndarray, np.ndarray]:
    """Codes (uint8, same shape) and float32 scales [..., cols / group]."""
    a = f64(x)
    cols = a.shape[-1]
    rows = a.size // cols
    codes = np.empty(a.shape, dtype=np.uint8)
    scales = np.empty(a.shape[:-1] + (cols // group,), dtype=np.float32)
    lib().oracle_quantize_e4m3(_p(a, _d), rows, cols, group, _p(codes, _u8), _p(scales, _f))
    return codes, scales


def dequantize(codes, scales, group: int) -> np.ndarray:
    c = _codes(codes)
    s = np.ascontiguousarray(f64(scales).astype(np.float32))
    cols = c.shape[-1]
    out = np.empty(c.shape, dtype=np.float64)
    lib().oracle_dequantize(_p(c, _u8), _p(s, _f), c.size // cols, cols, group, _p(out, _d))
    return out


def e2m1_value(code: int) -> float:
    return float(lib().oracle_e2m1_value(int(code)))


def e2m1_code(x: float) -> int:
    return int(lib().oracle_e2m1_code(float(x)))


def quantize_e2m1(x) -> Tuple[np.ndarray, np.ndarray]:
    """FP4 indexer-key storage of rows x [..., cols] (cols % 32 == 0): packed
    codes uint8 [..., cols / 2] (even channel in the low nibble) and block
    exponents uint8 [..., cols / 32] (block scale 2^(e - 127))."""
    a = f64(x)
    cols = a.shape[-1]
    rows = a.size // cols
    packed = np.zeros(a.shape[:-1] + (cols // 2,), dtype=np.uint8)
    exps = np.empty(a.shape[:-1] + (cols // 32,), dtype=np.uint8)
    lib().oracle_quantize_e2m1(_p(a, _d), rows, cols, _p(packed, _u8), _p(exps, _u8))
    return packed, exps


def dequantize_e2m1(packed, exps) -> np.ndarray:
    """Values [..., 2 * packed cols] of FP4 rows."""
    c = _codes(packed)
    e = _codes(exps)
    cols = 2 * c.shape[-1]
    out = np.empty(c.shape[:-1] + (cols,), dtype=np.float64)
    lib().oracle_dequantize_e2m1(_p(c, _u8), _p(e, _u8), c.size // c.shape[-1], cols,
                                 _p(out, _d))
    return out


def compress(Ca, Cb, Za, Zb, Ba, Bb, m: int, overlap: bool = True) -> np.ndarray:
    """Compressed entries [n // m, c] (Eq. 9-12; with overlap=False, Eq. 20-23
    where Ca, Za, Ba are C, Z, B and Cb, Zb, Bb are unused)."""
    Ca, Za, Ba = f64(Ca), f64(Za), f64(Ba)
    Cb = f64(Cb) if Cb is not None else Ca
    Zb = f64(Zb) if Zb is not None else Za
    Bb = f64(Bb) if Bb is not None else Ba
    n, c = Ca.shape
    out = np.empty((n // m, c), dtype=np.float64)
    lib().oracle_compress(_p(Ca, _d), _p(Cb, _d), _p(Za, _d), _p(Zb, _d), _p(Ba, _d),
                          _p(Bb, _d), n, c, m, int(bool(overlap)), _p(out, _d))
    return out


def indexer(qI, wI, kI, q_pos, m: int) -> np.ndarray:
    """Scores [B, nq, E]: qI [B, nq, hI, cI], wI [B, nq, hI], kI [B, E, cI]
    (all float64 values), q_pos [B, nq]."""
    qI, wI, kI = f64(qI), f64(wI), f64(kI)
    pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64))
    B, nq, hI, cI = qI.shape
    E = kI.shape[1]
    out = np.empty((B, nq, E), dtype=np.float64)
    lib().oracle_indexer(_p(qI, _d), _p(wI, _d), _p(kI, _d), _p(pos, _i64), B, nq, E, hI,
                         cI, m, _p(out, _d))
    return out


def topk(scores, q_pos, m: int, k: int) -> np.ndarray:
    """Selection [rows, k] int32 from score rows [rows, E]."""
    s = f64(scores)
    rows, E = s.shape
    pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64).reshape(rows))
    out = np.empty((rows, k), dtype=np.int32)
    lib().oracle_topk(_p(s, _d), rows, E, E, _p(pos, _i64), m, k, _p(out, _i32))
    return out


def attend(q, entries, idx, k: int, m: int, kwin, win_pos0, n_win: int, q_pos, sink,
           scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Shared-KV attention with window and sink. q [B, nq, h, c];
    entries [B, E, c]; idx [B * nq, k] int32 or None (every visible entry);
    kwin [B, wrows, c] with row r holding position win_pos0[b] + r."""
    q, ent = f64(q), f64(entries)
    B, nq, h, c = q.shape
    E = ent.shape[1]
    if kwin is None:
        kw = np.zeros((B, 1, c))
        n_win = 0
    else:
        kw = f64(kwin)
    wp = np.ascontiguousarray(np.asarray(win_pos0, dtype=np.int64).reshape(B))
    pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64).reshape(B, nq))
    sk = f64(sink).reshape(h)
    ix = None
    if idx is not None:
        ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(B * nq, k))
    out = np.empty((B, nq, h, c), dtype=np.float64)
    lse = np.empty((B, nq, h), dtype=np.float64)
    rc = lib().oracle_attend(_p(q, _d), _p(ent, _d), E,
                             _p(ix, _i32) if ix is not None else None, k, m, _p(kw, _d),
                             kw.shape[1], _p(wp, _i64), n_win, _p(pos, _i64), _p(sk, _d),
                             B, nq, h, c, float(scale), _p(out, _d), _p(lse, _d))
    if rc != 0:
        raise ValueError("oracle_attend: selection index or window position out of range")
    return out, lse


def norm_rope(x, pos, rope_dims: int, gamma=None, normalise: bool = True, eps: float = 1e-6,
              base: float = 10000.0) -> np.ndarray:
    """RMSNorm of each head vector (x [rows, heads, c] or [rows, c]) and RoPE
    on its last rope_dims dims at position pos[row] (Module D); float64 copy."""
    a = np.array(f64(x), dtype=np.float64, copy=True)
    shp = a.shape
    if a.ndim == 2:
        a = a[:, None, :]
    rows, heads, c = a.shape
    a = np.ascontiguousarray(a)
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(rows))
    g = None if gamma is None else np.ascontiguousarray(f64(gamma).reshape(c))
    lib().oracle_norm_rope(_p(a, _d), rows, heads, c, int(rope_dims), _p(p, _i64),
                           _p(g, _d) if g is not None else None, int(bool(normalise)),
                           float(eps), float(base))
    return a.reshape(shp)
