"""Thin Python binding over libfl.so: the C-ABI entry points under the same names.

Argument marshalling only: tensors become raw pointers, ``stream=None`` means
torch's current CUDA stream, and a non-zero status raises :class:`FlError`
with the library's message. Every step of the read path runs in the CUDA
library; importing this module fails loudly when libfl.so is missing (build it
with ``python -m variable_precision_weight_b200.build``).
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfl.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libfl.so not found at {LIB_PATH}; run `python -m variable_precision_weight_b200.build`")

_lib = C.CDLL(LIB_PATH)

FL_OK = 0
FL_MAX_BATCH = 16
FL_MAX_GEMV_BATCH = 32
FL_MAX_STOPS = 16
FL_MAX_PROBLEMS = 256
FL_GGML_Q4_K = 12
FL_GGML_Q6_K = 14
FL_GEMV_STATIC_SCRATCH_BYTES = 4 << 20
STATUS = {0: "FL_OK", -1: "FL_ERR_ARG", -2: "FL_ERR_SHAPE", -3: "FL_ERR_UNSUPPORTED", -4: "FL_ERR_ALIGN",
          -5: "FL_ERR_CUDA", -6: "FL_ERR_WORKSPACE", -7: "FL_ERR_TIMEOUT"}


class FlError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class fl_plane_weight(C.Structure):
    _fields_ = [("store", C.c_void_p), ("out", C.c_int), ("in_", C.c_int)]


class fl_lens_params(C.Structure):
    _fields_ = [("f", C.c_float), ("g", C.c_float), ("gamma", C.c_int), ("m", C.c_int), ("nstops", C.c_int),
                ("stops", C.c_float * FL_MAX_STOPS), ("combine", C.c_int)]


class fl_gemv_problem(C.Structure):
    _fields_ = [("w", fl_plane_weight), ("levels", C.c_void_p), ("to_levels", C.c_void_p), ("x", C.c_void_p),
                ("y", C.c_void_p)]


class fl_gate_spec(C.Structure):
    _fields_ = [("problem", C.c_int), ("tau_h", C.c_float), ("tau_m", C.c_float), ("entropy", C.c_void_p),
                ("margin", C.c_void_p), ("top2", C.c_void_p), ("escalate", C.c_void_p), ("workspace", C.c_void_p),
                ("workspace_bytes", C.c_size_t)]


class fl_kquant_problem(C.Structure):
    _fields_ = [("blocks", C.c_void_p), ("ggml_type", C.c_int), ("out", C.c_int), ("in_", C.c_int),
                ("x", C.c_void_p), ("y", C.c_void_p)]


class fl_decide_problem(C.Structure):
    _fields_ = [("w", fl_plane_weight), ("y", C.c_void_p), ("levels", C.c_void_p), ("score", C.c_void_p),
                ("lifted", C.c_void_p)]


class fl_decide_params(C.Structure):
    _fields_ = [("rule", C.c_int), ("gamma", C.c_int), ("kappa", C.c_int), ("lambda_", C.c_float), ("f", C.c_float),
                ("counters", C.c_void_p)]


FL_DECIDE_LADDER = 0
FL_DECIDE_SHARE = 1

_P, _I, _F, _S = C.c_void_p, C.c_int, C.c_float, C.c_size_t
_sigs = {
    "fl_status_string": (C.c_char_p, [_I]),
    "fl_last_error": (C.c_char_p, []),
    "fl_version": (_I, []),
    "fl_plane_store_bytes": (_S, [_I, _I]),
    "fl_pack_planes": (_I, [_P, _P, _I, _I, _P, _P]),
    "fl_level_map": (_I, [_P, _I, _P, _P, _I, C.POINTER(fl_lens_params), _P, _P, _P]),
    "fl_gemv_workspace_bytes": (_S, [_I, _I, _I]),
    "fl_device_status": (_I, []),
    "fl_selftest_wait_timeout": (_I, [_P]),
    "fl_gemv_depth": (_I, [C.POINTER(fl_plane_weight), _P, _P, _I, _P, _P, _S, _P]),
    "fl_gemv_depth_static": (_I, [C.POINTER(fl_plane_weight), _P, _P, _I, _P, _P]),
    "fl_gemv_residual": (_I, [C.POINTER(fl_plane_weight), _P, _P, _P, _I, _P, _P, _S, _P]),
    "fl_gemv_batched": (_I, [C.POINTER(fl_gemv_problem), _I, _I, _I, _P]),
    "fl_gemv_batched_listed": (_I, [C.POINTER(fl_gemv_problem), C.POINTER(C.c_void_p), C.POINTER(C.c_int), _I, _I,
                                    _I, _P]),
    "fl_gemv_gate_workspace_bytes": (_S, [_I]),
    "fl_gemv_batched_gate": (_I, [C.POINTER(fl_gemv_problem), _I, _I, _I, C.POINTER(fl_gate_spec), _P]),
    "fl_gemv_batched_gate_if": (_I, [C.POINTER(fl_gemv_problem), _I, _I, _I, C.POINTER(fl_gate_spec), _P, _P, _P]),
    "fl_gemv_batched_gate_partial": (_I, [C.POINTER(fl_gemv_problem), _I, _I, _I, C.POINTER(fl_gate_spec), _P, _P, _I,
                                          _P, _P]),
    "fl_logit_gate": (_I, [_P, _I, _I, _F, _F, _P, _P, _P, _P, _P]),
    "fl_kquant_bytes": (_S, [_I, _I, _I]),
    "fl_kquant_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "fl_gemv_kquant": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _S, _P]),
    "fl_gemv_kquant_batched": (_I, [C.POINTER(fl_kquant_problem), _I, _I, _P]),
    "fl_level_decide": (_I, [C.POINTER(fl_decide_problem), _I, _I, C.POINTER(fl_decide_params), _P]),
    "fl_spec_accept": (_I, [_P, _P, _I, _P, _P, _P]),
    "fl_shard_blocks": (_I, [_P, _I, _I, _I, _P]),
    "fl_logit_gate_partial": (_I, [_P, _I, _I, _I, _P, _P]),
    "fl_logit_gate_merge": (_I, [_P, _I, _I, _F, _F, _P, _P, _P, _P, _P]),
}
for _name, (_res, _args) in _sigs.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_sigs)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(status: int) -> None:
    if status != FL_OK:
        raise FlError(status, (_lib.fl_last_error() or b"").decode())


def fl_status_string(status: int) -> str:
    return _lib.fl_status_string(status).decode()


def fl_last_error() -> str:
    return (_lib.fl_last_error() or b"").decode()


def fl_version() -> int:
    return int(_lib.fl_version())


def fl_plane_store_bytes(out: int, inn: int) -> int:
    return int(_lib.fl_plane_store_bytes(out, inn))


def fl_pack_planes(codes, scales, out: int, inn: int, store, stream=None) -> None:
    _check(_lib.fl_pack_planes(_ptr(codes), _ptr(scales), out, inn, _ptr(store), _stream(stream)))


def plane_weight(store, out: int, inn: int) -> fl_plane_weight:
    return fl_plane_weight(_ptr(store), out, inn)


def lens_params(f: float, g: float, gamma: int, m: int, stops, combine: int) -> fl_lens_params:
    p = fl_lens_params()
    p.f, p.g, p.gamma, p.m, p.combine = float(f), float(g), int(gamma), int(m), int(combine)
    stops = [float(s) for s in stops]
    p.nstops = len(stops)
    for i, s in enumerate(stops):
        p.stops[i] = s
    return p


def fl_level_map(xy, nblocks: int, centers, radii, nlenses: int, params: fl_lens_params, levels, counts=None,
                 stream=None) -> None:
    _check(_lib.fl_level_map(_ptr(xy), nblocks, _ptr(centers), _ptr(radii), nlenses, C.byref(params), _ptr(levels),
                             _ptr(counts), _stream(stream)))


def fl_device_status() -> None:
    """Raises FlError(FL_ERR_TIMEOUT) if a kernel's bounded wait ran out since the last call."""
    _check(_lib.fl_device_status())


def fl_selftest_wait_timeout(stream=None) -> None:
    _check(_lib.fl_selftest_wait_timeout(_stream(stream)))


def fl_gemv_workspace_bytes(out: int, inn: int, batch: int) -> int:
    return int(_lib.fl_gemv_workspace_bytes(out, inn, batch))


def fl_gemv_depth(w: fl_plane_weight, levels, x, batch: int, y, workspace=None, workspace_bytes: int = 0,
                  stream=None) -> None:
    _check(_lib.fl_gemv_depth(C.byref(w), _ptr(levels), _ptr(x), batch, _ptr(y), _ptr(workspace), workspace_bytes,
                              _stream(stream)))


def fl_gemv_depth_static(w: fl_plane_weight, levels, x, batch: int, y, stream=None) -> None:
    _check(_lib.fl_gemv_depth_static(C.byref(w), _ptr(levels), _ptr(x), batch, _ptr(y), _stream(stream)))


def fl_gemv_residual(w: fl_plane_weight, from_levels, to_levels, x, batch: int, y, workspace=None,
                     workspace_bytes: int = 0, stream=None) -> None:
    _check(_lib.fl_gemv_residual(C.byref(w), _ptr(from_levels), _ptr(to_levels), _ptr(x), batch, _ptr(y),
                                 _ptr(workspace), workspace_bytes, _stream(stream)))


def gemv_problems(items) -> "C.Array":
    """items: iterable of (store, out, in, levels, to_levels, x, y) -> fl_gemv_problem array."""
    items = list(items)
    arr = (fl_gemv_problem * len(items))()
    for i, (store, out, inn, lv, lt, x, y) in enumerate(items):
        arr[i] = fl_gemv_problem(fl_plane_weight(_ptr(store), out, inn), _ptr(lv), _ptr(lt), _ptr(x), _ptr(y))
    return arr


def fl_gemv_batched(problems, n: int, batch: int, mode: int, stream=None) -> None:
    _check(_lib.fl_gemv_batched(problems, n, batch, mode, _stream(stream)))


def block_lists(lists, counts):
    """Device block lists and their host counts -> (pointer array, count array) for
    fl_gemv_batched_listed."""
    ptrs = (C.c_void_p * len(lists))(*[_ptr(l) for l in lists])
    cnts = (C.c_int * len(counts))(*[int(c) for c in counts])
    return ptrs, cnts


def fl_gemv_batched_listed(problems, lists, counts, n: int, batch: int, mode: int, stream=None) -> None:
    """lists, counts: the pair block_lists() returns."""
    _check(_lib.fl_gemv_batched_listed(problems, lists, counts, n, batch, mode, _stream(stream)))


def fl_gemv_gate_workspace_bytes(batch: int) -> int:
    return int(_lib.fl_gemv_gate_workspace_bytes(batch))


def gate_spec(problem: int, tau_h: float, tau_m: float, entropy, margin, top2, escalate, workspace,
              workspace_bytes: int) -> fl_gate_spec:
    return fl_gate_spec(problem, float(tau_h), float(tau_m), _ptr(entropy), _ptr(margin), _ptr(top2), _ptr(escalate),
                        _ptr(workspace), workspace_bytes)


def fl_gemv_batched_gate(problems, n: int, batch: int, mode: int, gate: fl_gate_spec, stream=None) -> None:
    _check(_lib.fl_gemv_batched_gate(problems, n, batch, mode, C.byref(gate), _stream(stream)))


def fl_gemv_batched_gate_if(problems, n: int, batch: int, mode: int, gate: fl_gate_spec, run_if, runs=None,
                            stream=None) -> None:
    _check(_lib.fl_gemv_batched_gate_if(problems, n, batch, mode, C.byref(gate), _ptr(run_if), _ptr(runs),
                                        _stream(stream)))


def fl_gemv_batched_gate_partial(problems, n: int, batch: int, mode: int, gate: fl_gate_spec, run_if, runs,
                                 index_base: int, partial, stream=None) -> None:
    _check(_lib.fl_gemv_batched_gate_partial(problems, n, batch, mode, C.byref(gate), _ptr(run_if), _ptr(runs),
                                             index_base, _ptr(partial), _stream(stream)))


def fl_logit_gate(logits, vocab: int, batch: int, tau_h: float, tau_m: float, entropy, margin, top2, escalate,
                  stream=None) -> None:
    _check(_lib.fl_logit_gate(_ptr(logits), vocab, batch, float(tau_h), float(tau_m), _ptr(entropy), _ptr(margin),
                              _ptr(top2), _ptr(escalate), _stream(stream)))


def fl_kquant_bytes(ggml_type: int, out: int, inn: int) -> int:
    return int(_lib.fl_kquant_bytes(ggml_type, out, inn))


def fl_kquant_workspace_bytes(ggml_type: int, out: int, inn: int, batch: int) -> int:
    return int(_lib.fl_kquant_workspace_bytes(ggml_type, out, inn, batch))


def fl_gemv_kquant(blocks, ggml_type: int, out: int, inn: int, x, batch: int, y, workspace=None,
                   workspace_bytes: int = 0, stream=None) -> None:
    _check(_lib.fl_gemv_kquant(_ptr(blocks), ggml_type, out, inn, _ptr(x), batch, _ptr(y), _ptr(workspace),
                               workspace_bytes, _stream(stream)))


def kquant_problems(items) -> "C.Array":
    """items: iterable of (blocks, ggml_type, out, in, x, y) -> fl_kquant_problem array."""
    items = list(items)
    arr = (fl_kquant_problem * len(items))()
    for i, (blk, t, out, inn, x, y) in enumerate(items):
        arr[i] = fl_kquant_problem(_ptr(blk), t, out, inn, _ptr(x), _ptr(y))
    return arr


def fl_gemv_kquant_batched(problems, n: int, batch: int, stream=None) -> None:
    _check(_lib.fl_gemv_kquant_batched(problems, n, batch, _stream(stream)))


def decide_problems(items) -> "C.Array":
    """items: iterable of (store, out, in, y, levels, score or None[, lifted or None])
    -> fl_decide_problem array."""
    items = list(items)
    arr = (fl_decide_problem * len(items))()
    for i, it in enumerate(items):
        store, out, inn, y, lv, sc = it[:6]
        lifted = it[6] if len(it) > 6 else None
        arr[i] = fl_decide_problem(fl_plane_weight(_ptr(store), out, inn), _ptr(y), _ptr(lv), _ptr(sc),
                                   _ptr(lifted))
    return arr


def decide_params(rule: int, gamma: int, kappa: int, lam: float = 0.0, f: float = 0.0,
                  counters=None) -> fl_decide_params:
    """counters: a zero-filled device int32 tensor of one entry per problem makes the share rule
    one launch (the last CTA to score a layer selects it)."""
    return fl_decide_params(rule, gamma, kappa, float(lam), float(f), _ptr(counters))


def fl_level_decide(problems, n: int, batch: int, params: fl_decide_params, stream=None) -> None:
    _check(_lib.fl_level_decide(problems, n, batch, C.byref(params), _stream(stream)))


def fl_spec_accept(draft_top2, verified_top2, k: int, result, totals=None, stream=None) -> None:
    _check(_lib.fl_spec_accept(_ptr(draft_top2), _ptr(verified_top2), k, _ptr(result), _ptr(totals),
                               _stream(stream)))


# ----------------------------------------------------------------------------- the read split over ranks

GATE_PARTIAL_BYTES = 32  # one fl_gate_partial


def fl_shard_blocks(levels, inn: int, nranks: int) -> list:
    """Host levels (uint8 numpy array) -> [nranks + 1] first-block indices of each rank's range."""
    import numpy as np
    lv = np.ascontiguousarray(levels, dtype=np.uint8)
    first = (C.c_int * (nranks + 1))()
    _check(_lib.fl_shard_blocks(lv.ctypes.data if lv.size else None, int(lv.size), inn, nranks, first))
    return [int(v) for v in first]


def fl_logit_gate_partial(logits, vocab: int, batch: int, index_base: int, partial, stream=None) -> None:
    """partial: a device buffer of batch * 32 bytes (fl_gate_partial records)."""
    _check(_lib.fl_logit_gate_partial(_ptr(logits), vocab, batch, index_base, _ptr(partial), _stream(stream)))


def fl_logit_gate_merge(partials, nparts: int, batch: int, tau_h: float, tau_m: float, entropy, margin, top2,
                        escalate, stream=None) -> None:
    """partials: device [nparts][batch] fl_gate_partial records (nparts * batch * 32 bytes)."""
    _check(_lib.fl_logit_gate_merge(_ptr(partials), nparts, batch, float(tau_h), float(tau_m), _ptr(entropy),
                                    _ptr(margin), _ptr(top2), _ptr(escalate), _stream(stream)))
