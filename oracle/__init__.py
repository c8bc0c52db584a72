"""CPU oracle: ctypes bindings over ``oracle.c``.

TEST INFRASTRUCTURE ONLY. The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers. The product path never
imports this package; it shares no code with the CUDA library.

``build()`` compiles ``oracle.c`` with gcc (plain C99, OpenMP over output rows,
``-ffp-contract=off`` so that the fp32 lens rule rounds every operation).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

Q4_K = 12
Q6_K = 14
RECORD_BYTES = {Q4_K: 144, Q6_K: 210}


def build(force: bool = False) -> str:
    """Compile liboracle.so next to the source if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = C.CDLL(_LIB)
            P = C.c_void_p
            i, f, d = C.c_int, C.c_float, C.c_double
            sig = {
                "orc_max_threads": (i, []),
                "orc_quantize_int8": (None, [P, i, i, P, P]),
                "orc_dequant_depth": (d, [C.c_int8, f, i]),
                "orc_gemv_depth": (None, [P, P, i, i, P, P, i, P, P, i]),
                "orc_gemv_residual": (None, [P, P, i, i, P, P, P, i, P, P, i]),
                "orc_store_bytes": (C.c_size_t, [i, i]),
                "orc_pack_planes": (None, [P, P, i, i, P]),
                "orc_unpack_planes": (None, [P, i, i, P, P]),
                "orc_lens_kappa": (i, [f, i, i]),
                "orc_level_map": (None, [P, i, P, P, i, f, f, i, i, i, P, i, P]),
                "orc_memory_bits": (d, [P, i, P, P]),
                "orc_level_decide": (i, [P, i, i, P, i, i, i, i, d, d, P, P]),
                "orc_spec_accept": (None, [P, P, i, P, P]),
                "orc_logit_gate": (None, [P, i, i, d, d, P, P, P, P]),
                "orc_dequant_q4k": (None, [P, P]),
                "orc_dequant_q6k": (None, [P, i, P]),
                "orc_gemv_kquant": (i, [P, i, i, i, P, i, P, P, i]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 inputs are passed as their uint16 bit patterns"
    return x


def max_threads() -> int:
    return int(_load().orc_max_threads())


def quantize_int8(w: np.ndarray):
    w = np.ascontiguousarray(w, dtype=np.float32)
    out, inn = w.shape
    q = np.empty((out, inn), np.int8)
    s = np.empty((out, inn // 128), np.float32)
    _load().orc_quantize_int8(_p(w), out, inn, _p(q), _p(s))
    return q, s


def dequant_depth(q: int, s: float, depth: int) -> float:
    return float(_load().orc_dequant_depth(int(q), float(s), int(depth)))


def gemv_depth(q, s, levels, x_bf16, nthreads: int = 0, with_mass: bool = False):
    """y [batch, out] in float64; with_mass also returns sum_c |w_d| |x| per output."""
    q = np.ascontiguousarray(q, np.int8)
    s = np.ascontiguousarray(s, np.float32)
    levels = np.ascontiguousarray(levels, np.uint8)
    x = _bf16_bits(x_bf16)
    out, inn = q.shape
    batch = x.shape[0]
    y = np.empty((batch, out), np.float64)
    m = np.empty((batch, out), np.float64) if with_mass else None
    _load().orc_gemv_depth(_p(q), _p(s), out, inn, _p(levels), _p(x), batch, _p(y), _p(m) if with_mass else None,
                           nthreads)
    return (y, m) if with_mass else y


def gemv_residual(q, s, from_levels, to_levels, x_bf16, nthreads: int = 0, with_mass: bool = False):
    q = np.ascontiguousarray(q, np.int8)
    s = np.ascontiguousarray(s, np.float32)
    a = np.ascontiguousarray(from_levels, np.uint8)
    b = np.ascontiguousarray(to_levels, np.uint8)
    x = _bf16_bits(x_bf16)
    out, inn = q.shape
    batch = x.shape[0]
    y = np.empty((batch, out), np.float64)
    m = np.empty((batch, out), np.float64) if with_mass else None
    _load().orc_gemv_residual(_p(q), _p(s), out, inn, _p(a), _p(b), _p(x), batch, _p(y),
                              _p(m) if with_mass else None, nthreads)
    return (y, m) if with_mass else y


def store_bytes(out: int, inn: int) -> int:
    return int(_load().orc_store_bytes(out, inn))


def pack_planes(q, s) -> np.ndarray:
    q = np.ascontiguousarray(q, np.int8)
    s = np.ascontiguousarray(s, np.float32)
    out, inn = q.shape
    store = np.empty(store_bytes(out, inn), np.uint8)
    _load().orc_pack_planes(_p(q), _p(s), out, inn, _p(store))
    return store


def unpack_planes(store, out: int, inn: int):
    store = np.ascontiguousarray(store, np.uint8)
    q = np.empty((out, inn), np.int8)
    s = np.empty((out, inn // 128), np.float32)
    _load().orc_unpack_planes(_p(store), out, inn, _p(q), _p(s))
    return q, s


def lens_kappa(g: float, gamma: int, m: int) -> int:
    return int(_load().orc_lens_kappa(float(g), int(gamma), int(m)))


def level_map(xy, cxy, r, f, g, gamma, m, stops, combine: int) -> np.ndarray:
    xy = np.ascontiguousarray(xy, np.float32).reshape(-1, 2)
    cxy = np.ascontiguousarray(cxy, np.float32).reshape(-1, 2)
    r = np.ascontiguousarray(r, np.float32).reshape(-1)
    stops = np.ascontiguousarray(stops, np.float32).reshape(-1)
    if stops.size == 0:
        stops = np.zeros(1, np.float32)
        nst = 0
    else:
        nst = stops.size
    lev = np.empty(xy.shape[0], np.uint8)
    _load().orc_level_map(_p(xy), xy.shape[0], _p(cxy), _p(r), cxy.shape[0], float(f), float(g), int(gamma),
                          int(m), nst, _p(stops), int(combine), _p(lev))
    return lev


def level_decide(y, scales, gamma: int, kappa: int, rule: int, lam: float = 0.0, f: float = 0.0):
    """In-pass level decision from a layer's base-level outputs y [batch, out] and its
    scales [out, in / 128]: (levels uint8 [out / 64], reduced scores float64 [out / 64])."""
    y = np.ascontiguousarray(y, np.float32)
    if y.ndim == 1:
        y = y[None]
    s = np.ascontiguousarray(scales, np.float32)
    batch, out = y.shape
    assert s.shape[0] == out
    inn = 128 * s.shape[1]
    nb = out // 64
    lev = np.empty(nb, np.uint8)
    red = np.empty(nb, np.float64)
    rc = _load().orc_level_decide(_p(y), batch, out, _p(s), inn, int(gamma), int(kappa), int(rule), float(lam),
                                  float(f), _p(lev), _p(red))
    if rc != 0:
        raise ValueError(f"orc_level_decide: bad arguments ({rc})")
    return lev, red


def spec_accept(draft, verified):
    """Greedy verified speculation over one window: (accepted, emitted)."""
    dr = np.ascontiguousarray(draft, np.int32).reshape(-1)
    vf = np.ascontiguousarray(verified, np.int32).reshape(-1)
    assert dr.shape == vf.shape
    a, e = np.zeros(1, np.int32), np.zeros(1, np.int32)
    _load().orc_spec_accept(_p(dr), _p(vf), len(dr), _p(a), _p(e))
    return int(a[0]), int(e[0])


def memory_bits(levels, wb, bits_of_level) -> float:
    levels = np.ascontiguousarray(levels, np.uint8)
    wb = np.ascontiguousarray(wb, np.float64)
    bol = np.ascontiguousarray(bits_of_level, np.float64)
    return float(_load().orc_memory_bits(_p(levels), levels.size, _p(wb), _p(bol)))


def logit_gate(logits, tau_h: float, tau_m: float):
    z = np.ascontiguousarray(logits, np.float32)
    if z.ndim == 1:
        z = z[None]
    batch, vocab = z.shape
    H = np.empty(batch, np.float64)
    M = np.empty(batch, np.float64)
    top2 = np.empty((batch, 2), np.int32)
    esc = np.empty(batch, np.uint8)
    _load().orc_logit_gate(_p(z), vocab, batch, float(tau_h), float(tau_m), _p(H), _p(M), _p(top2), _p(esc))
    return H, M, top2, esc


def dequant_superblock(rec: np.ndarray, ggml_type: int, row: int = 0) -> np.ndarray:
    """Dequantize one record; a Q6_K record's layout depends on the parity of its row."""
    rec = np.ascontiguousarray(rec, np.uint8)
    w = np.empty(256, np.float64)
    if ggml_type == Q4_K:
        assert rec.size == 144
        _load().orc_dequant_q4k(_p(rec), _p(w))
    elif ggml_type == Q6_K:
        assert rec.size == 210
        _load().orc_dequant_q6k(_p(rec), int(row) & 1, _p(w))
    else:
        raise ValueError("unsupported type")
    return w


def gemv_kquant(blocks, ggml_type: int, out: int, inn: int, x_bf16, nthreads: int = 0, with_mass: bool = False):
    blocks = np.ascontiguousarray(blocks, np.uint8)
    x = _bf16_bits(x_bf16)
    batch = x.shape[0]
    assert batch <= 16
    y = np.empty((batch, out), np.float64)
    m = np.empty((batch, out), np.float64) if with_mass else None
    rc = _load().orc_gemv_kquant(_p(blocks), int(ggml_type), out, inn, _p(x), batch, _p(y),
                                 _p(m) if with_mass else None, nthreads)
    if rc != 0:
        raise ValueError("unsupported K-quant type")
    return (y, m) if with_mass else y
