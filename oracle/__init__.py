"""CPU oracle for the FP8 block-scaled NT GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(``cpu_baseline`` / ``--impl reference``) may import this package.  The product
library under ``moe_grouped_gemm_weight_b200/`` never imports, links or runs it,
and the two share no code.

The arithmetic lives in ``dg_oracle.c`` (plain C, FP64); this module compiles it
with gcc on first use and wraps it with numpy arrays.  See the header of
``dg_oracle.c`` for the definition it follows and the readings it takes.

Parity status of each function (what pins it is in ``tests/test_oracle_pins.py``):
  e4m3_table            pinned (bit definition anchors + torch float8_e4m3fn)
  bf16_rne              pinned (torch float->bf16 + nearest/ties-even property)
  gemm_nt               pinned (brute-force dequantise-then-matmul, integer
                        exactness, linearity, K-tail zero-extension)
  grouped_contiguous    pinned (equals gemm_nt per segment; -1 rows untouched)
  grouped_masked        pinned (equals gemm_nt on the first masked_m rows)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, BAD_ARG, BAD_INDEX = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile dg_oracle.c into liboracle.so (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _SO, "-lm"]
        subprocess.run(cmd, check=True)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # DG_ORACLE_SO lets the mutation test load a deliberately broken
            # build of this same source; normal use always builds dg_oracle.c.
            so = os.environ.get("DG_ORACLE_SO")
            if not so:
                so = build()
            lib = ctypes.CDLL(so)
            P = ctypes.c_void_p
            I, I64 = ctypes.c_int, ctypes.c_int64
            lib.dgo_e4m3_decode.restype = ctypes.c_double
            lib.dgo_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.dgo_e4m3_table.argtypes = [P]
            lib.dgo_bf16_rne.restype = ctypes.c_uint16
            lib.dgo_bf16_rne.argtypes = [ctypes.c_double]
            lib.dgo_bf16_rne_array.argtypes = [P, P, I64]
            lib.dgo_bf16_to_double.restype = ctypes.c_double
            lib.dgo_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.dgo_gemm_nt.restype = I
            lib.dgo_gemm_nt.argtypes = [P, P, I64, P, P, I, I, I, P, I64, P, P, P]
            lib.dgo_grouped_contiguous.restype = I
            lib.dgo_grouped_contiguous.argtypes = [P, P, I64, P, P, P, I, I, I, I, P, I64, P, P, P]
            lib.dgo_grouped_masked.restype = I
            lib.dgo_grouped_masked.argtypes = [P, P, I64, P, P, P, I, I, I, I, P, I64, P, P, P]
            lib.dgo_num_threads.restype = I
            lib.dgo_e4m3_encode.restype = ctypes.c_uint8
            lib.dgo_e4m3_encode.argtypes = [ctypes.c_float]
            lib.dgo_e4m3_encode_array.argtypes = [P, P, I64]
            lib.dgo_cast_1x128.restype = I
            lib.dgo_cast_1x128.argtypes = [P, I, I, P, P, I64]
            lib.dgo_cast_128x128.restype = I
            lib.dgo_cast_128x128.argtypes = [P, I, I, P, P]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def num_threads() -> int:
    return int(_load().dgo_num_threads())


def e4m3_decode(code: int) -> float:
    return float(_load().dgo_e4m3_decode(int(code) & 0xFF))


def e4m3_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _load().dgo_e4m3_table(_ptr(out))
    return out


def bf16_rne(x) -> np.ndarray:
    """Round doubles to bf16 (RNE), returning the uint16 bit patterns."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.uint16)
    _load().dgo_bf16_rne_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f64(bits) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rows_arg(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size


def gemm_nt(A, sa, sa_stride, B, sb, M, N, K, rows=None, D=None, want_d64=True, want_mag=True):
    """Dense scaled NT GEMM.  Returns (D bits uint16 [M,N], D64 or None, MAG or None).

    A uint8 [M,K]; sa float32 flat, sa[kb*sa_stride + m]; B uint8 [N,K];
    sb float32 [ceil(N/128), ceil(K/128)].  ``rows`` restricts the computed rows;
    ``D`` (uint16 [M,N]) may be passed pre-filled so that untouched rows keep it.
    """
    lib = _load()
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sa, sb = _c(sa, np.float32), _c(sb, np.float32)
    if D is None:
        D = np.zeros((M, N), dtype=np.uint16)
    D = _c(D, np.uint16)
    D64 = np.full((M, N), np.nan) if want_d64 else None
    MAG = np.full((M, N), np.nan) if want_mag else None
    r, nr = _rows_arg(rows)
    rc = lib.dgo_gemm_nt(_ptr(A), _ptr(sa), sa_stride, _ptr(B), _ptr(sb), M, N, K,
                         _ptr(r), nr, _ptr(D), _ptr(D64), _ptr(MAG))
    if rc != OK:
        raise ValueError(f"oracle gemm_nt rejected its arguments (code {rc})")
    return D, D64, MAG


def grouped_contiguous(A, sa, sa_stride, B, sb, m_indices, M, N, K, G, rows=None, D=None,
                       want_d64=True, want_mag=True):
    """Contiguous-layout grouped GEMM.  m_indices int32 [M]; -1 rows untouched."""
    lib = _load()
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sa, sb = _c(sa, np.float32), _c(sb, np.float32)
    mi = _c(m_indices, np.int32)
    if D is None:
        D = np.zeros((M, N), dtype=np.uint16)
    D = _c(D, np.uint16)
    D64 = np.full((M, N), np.nan) if want_d64 else None
    MAG = np.full((M, N), np.nan) if want_mag else None
    r, nr = _rows_arg(rows)
    rc = lib.dgo_grouped_contiguous(_ptr(A), _ptr(sa), sa_stride, _ptr(B), _ptr(sb), _ptr(mi),
                                    M, N, K, G, _ptr(r), nr, _ptr(D), _ptr(D64), _ptr(MAG))
    if rc != OK:
        raise ValueError(f"oracle grouped_contiguous rejected its arguments (code {rc})")
    return D, D64, MAG


def grouped_masked(A, sa, sa_stride, B, sb, masked_m, G, Mmax, N, K, rows=None, D=None,
                   want_d64=True, want_mag=True):
    """Masked-layout grouped GEMM.  A uint8 [G,Mmax,K]; D uint16 [G,Mmax,N]."""
    lib = _load()
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sa, sb = _c(sa, np.float32), _c(sb, np.float32)
    mm = _c(masked_m, np.int32)
    if D is None:
        D = np.zeros((G, Mmax, N), dtype=np.uint16)
    D = _c(D, np.uint16)
    D64 = np.full((G, Mmax, N), np.nan) if want_d64 else None
    MAG = np.full((G, Mmax, N), np.nan) if want_mag else None
    r, nr = _rows_arg(rows)
    rc = lib.dgo_grouped_masked(_ptr(A), _ptr(sa), sa_stride, _ptr(B), _ptr(sb), _ptr(mm),
                                G, Mmax, N, K, _ptr(r), nr, _ptr(D), _ptr(D64), _ptr(MAG))
    if rc != OK:
        raise ValueError(f"oracle grouped_masked rejected its arguments (code {rc})")
    return D, D64, MAG


def e4m3_encode(x) -> np.ndarray:
    """e4m3 codes (uint8) of float32 values: RNE, saturating to +-448, NaN -> 0x7F."""
    x = _c(np.atleast_1d(np.asarray(x, dtype=np.float32)), np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().dgo_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def cast_1x128(X_bf16, M, K, sa_stride):
    """Activation cast: bf16 bits [M,K] -> (e4m3 codes [M,K], sa float32 flat with
    sa[kb*sa_stride + m])."""
    X = _c(X_bf16, np.uint16)
    Q = np.zeros((M, K), dtype=np.uint8)
    sa = np.zeros((K // 128) * sa_stride, dtype=np.float32)
    rc = _load().dgo_cast_1x128(_ptr(X), M, K, _ptr(Q), _ptr(sa), sa_stride)
    if rc != OK:
        raise ValueError(f"oracle cast_1x128 rejected its arguments (code {rc})")
    return Q, sa


def cast_128x128(W_bf16, N, K):
    """Weight cast: bf16 bits [N,K] -> (e4m3 codes [N,K], sb float32 [ceil(N/128), K/128])."""
    W = _c(W_bf16, np.uint16)
    Q = np.zeros((N, K), dtype=np.uint8)
    sb = np.zeros(((N + 127) // 128, K // 128), dtype=np.float32)
    rc = _load().dgo_cast_128x128(_ptr(W), N, K, _ptr(Q), _ptr(sb))
    if rc != OK:
        raise ValueError(f"oracle cast_128x128 rejected its arguments (code {rc})")
    return Q, sb
