"""The C-ABI library on a host without a GPU: it loads, exports every symbol the
header declares, and rejects bad arguments before launching anything."""
import ctypes as C
import os
import re

import pytest

from variable_precision_weight_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fl():
    build.build()
    from variable_precision_weight_b200 import fl as mod
    return mod


def header_symbols():
    text = open(os.path.join(ROOT, "include", "fl.h")).read()
    return sorted(set(re.findall(r"FL_API\s+[\w\s\*]+?\b(fl_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_symbols()
    for n in ("fl_pack_planes", "fl_level_map", "fl_gemv_depth", "fl_gemv_residual", "fl_logit_gate",
              "fl_gemv_kquant"):
        assert n in names


def test_library_exports_every_declared_symbol(fl):
    lib = C.CDLL(fl.LIB_PATH)
    for n in header_symbols():
        assert hasattr(lib, n), n
    assert set(header_symbols()) == set(fl.EXPORTED)


def test_status_strings(fl):
    assert fl.fl_status_string(0) == "FL_OK"
    assert fl.fl_status_string(-3) == "FL_ERR_UNSUPPORTED"
    assert fl.fl_version() >= 1


def test_byte_counts(fl, orc):
    assert fl.fl_plane_store_bytes(1024, 1024) == orc.store_bytes(1024, 1024) == 16 * 8 * 8448
    assert fl.fl_plane_store_bytes(100, 1024) == 0
    assert fl.fl_kquant_bytes(fl.FL_GGML_Q4_K, 2048, 2048) == 2048 * 8 * 144
    assert fl.fl_kquant_bytes(fl.FL_GGML_Q6_K, 2048, 8192) == 2048 * 32 * 210
    assert fl.fl_kquant_bytes(13, 2048, 2048) == 0


def _status(fl, fn, *args):
    with pytest.raises(fl.FlError) as e:
        fn(*args)
    return e.value.status


def test_host_side_rejections(fl):
    ERR_ARG, ERR_SHAPE, ERR_UNSUP = -1, -2, -3
    s0 = 0  # explicit stream handle so no CUDA runtime call is needed
    assert _status(fl, fl.fl_pack_planes, None, None, 64, 128, None, s0) == ERR_ARG
    assert _status(fl, fl.fl_pack_planes, 16, 16, 100, 128, 16, s0) == ERR_SHAPE
    w = fl.plane_weight(16, 64, 100)
    assert _status(fl, fl.fl_gemv_depth, w, 16, 16, 1, 16, None, 0, s0) == ERR_SHAPE
    w = fl.plane_weight(None, 64, 128)
    assert _status(fl, fl.fl_gemv_depth, w, 16, 16, 1, 16, None, 0, s0) == ERR_ARG
    w = fl.plane_weight(16, 64, 128)
    assert _status(fl, fl.fl_gemv_depth, w, 16, 16, 0, 16, None, 0, s0) == ERR_SHAPE       # batch 0
    assert _status(fl, fl.fl_gemv_depth, w, 16, 16, 33, 16, None, 0, s0) == ERR_SHAPE      # batch 33
    assert _status(fl, fl.fl_gemv_depth_static, w, 16, 16, 17, 16, s0) == ERR_SHAPE       # batch 17 (no tcgen05)
    assert _status(fl, fl.fl_gemv_residual, w, 16, None, 16, 1, 16, None, 0, s0) == ERR_ARG
    assert _status(fl, fl.fl_gemv_kquant, 16, 13, 64, 256, 16, 1, 16, None, 0, s0) == ERR_UNSUP   # Q5_K
    assert _status(fl, fl.fl_gemv_kquant, 16, 10, 64, 256, 16, 1, 16, None, 0, s0) == ERR_UNSUP   # Q2_K
    assert _status(fl, fl.fl_gemv_kquant, 16, 14, 32, 256, 16, 1, 16, None, 0, s0) == ERR_SHAPE   # out % 64
    assert _status(fl, fl.fl_gemv_kquant, 16, 12, 64, 384, 16, 1, 16, None, 0, s0) == ERR_SHAPE   # in % 256
    assert _status(fl, fl.fl_logit_gate, 16, 151937, 1, 0.0, 0.0, 16, 16, 16, 16, s0) == ERR_SHAPE
    assert _status(fl, fl.fl_logit_gate, 16, 1024, 0, 0.0, 0.0, 16, 16, 16, 16, s0) == ERR_SHAPE
    p = fl.lens_params(0.3, 0.75, 1, 4, [0.5], 0)                  # kappa - gamma = 2 stops needed
    assert _status(fl, fl.fl_level_map, 16, 10, 16, 16, 8, p, 16, None, s0) == ERR_ARG
    p = fl.lens_params(0.3, 0.75, 1, 4, [1.0, 0.5], 0)             # not ascending
    assert _status(fl, fl.fl_level_map, 16, 10, 16, 16, 8, p, 16, None, s0) == ERR_ARG
    p = fl.lens_params(1.0, 0.75, 1, 4, [0.5, 1.0], 0)             # f must be < 1
    assert _status(fl, fl.fl_level_map, 16, 10, 16, 16, 8, p, 16, None, s0) == ERR_ARG
    probs = fl.gemv_problems([(16, 64, 128, 16, None, 16, 16)])
    assert _status(fl, fl.fl_gemv_batched, probs, 0, 1, 0, s0) == ERR_ARG
    assert _status(fl, fl.fl_gemv_batched, probs, 1, 1, 2, s0) == ERR_ARG                  # mode
    assert _status(fl, fl.fl_gemv_batched, probs, 1, 17, 0, s0) == ERR_SHAPE               # batch 17
    gsz = fl.fl_gemv_gate_workspace_bytes(1)
    assert gsz > 0 and fl.fl_gemv_gate_workspace_bytes(0) == 0
    spec = fl.gate_spec(1, 0.0, 0.0, 16, 16, 16, 16, 16, gsz)                  # problem 1 of 1
    assert _status(fl, fl.fl_gemv_batched_gate, probs, 1, 1, 0, spec, s0) == ERR_ARG
    spec = fl.gate_spec(0, 0.0, 0.0, 16, None, 16, 16, 16, gsz)                # NULL margin
    assert _status(fl, fl.fl_gemv_batched_gate, probs, 1, 1, 0, spec, s0) == ERR_ARG
    spec = fl.gate_spec(0, 0.0, 0.0, 16, 16, 16, 16, 16, gsz - 1)              # workspace too small
    assert _status(fl, fl.fl_gemv_batched_gate, probs, 1, 1, 0, spec, s0) == -6
    spec = fl.gate_spec(0, 0.0, 0.0, 16, 16, 16, 16, 17, gsz)                  # misaligned workspace
    assert _status(fl, fl.fl_gemv_batched_gate, probs, 1, 1, 0, spec, s0) == -4
    spec = fl.gate_spec(0, 0.0, 0.0, 16, 16, 16, 16, 16, gsz)
    assert _status(fl, fl.fl_gemv_batched_gate_if, probs, 1, 1, 1, spec, None, None, s0) == ERR_ARG   # no run_if
    assert _status(fl, fl.fl_gemv_batched_gate_if, probs, 1, 1, 1, spec, 16, 18, s0) == -4           # runs misaligned
    spec = fl.gate_spec(0, 0.0, 0.0, 16, 16, 18, 16, 16, gsz)                  # top2 misaligned
    assert _status(fl, fl.fl_gemv_batched_gate, probs, 1, 1, 0, spec, s0) == -4
    assert _status(fl, fl.fl_logit_gate, 16, 1024, 1, 0.0, 0.0, 16, 17, 16, 16, s0) == -4          # margin
    kp = fl.kquant_problems([(16, 11, 64, 256, 16, 16)])
    assert _status(fl, fl.fl_gemv_kquant_batched, kp, 1, 1, s0) == ERR_UNSUP
    assert "Q4_K" in fl.fl_last_error()
    # in-pass level decision
    dp = fl.decide_problems([(16, 64, 128, 16, 16, None)])
    lad = fl.decide_params(fl.FL_DECIDE_LADDER, 2, 4, lam=1.0)
    assert _status(fl, fl.fl_level_decide, dp, 0, 1, lad, s0) == ERR_ARG                    # n = 0
    assert _status(fl, fl.fl_level_decide, dp, 1, 17, lad, s0) == ERR_SHAPE                 # batch 17
    for bad in ((fl.FL_DECIDE_LADDER, 0, 4, 1.0, 0.0), (fl.FL_DECIDE_LADDER, 3, 2, 1.0, 0.0),
                (fl.FL_DECIDE_LADDER, 2, 5, 1.0, 0.0), (fl.FL_DECIDE_LADDER, 2, 4, -1.0, 0.0),
                (fl.FL_DECIDE_LADDER, 2, 4, float("nan"), 0.0), (fl.FL_DECIDE_SHARE, 2, 4, 0.0, 1.5),
                (fl.FL_DECIDE_SHARE, 2, 4, 0.0, 0.5), (2, 2, 4, 0.0, 0.0)):
        # the share rule also needs a score array, which dp lacks
        assert _status(fl, fl.fl_level_decide, dp, 1, 1, fl.decide_params(*bad), s0) == ERR_ARG, bad
    dp = fl.decide_problems([(16, 64, 100, 16, 16, None)])
    assert _status(fl, fl.fl_level_decide, dp, 1, 1, lad, s0) == ERR_SHAPE                  # in % 128
    dp = fl.decide_problems([(16, 64, 128, None, 16, None)])
    assert _status(fl, fl.fl_level_decide, dp, 1, 1, lad, s0) == ERR_ARG                    # NULL y
    dp = fl.decide_problems([(16, 64, 128, 20, 16, None)])
    assert _status(fl, fl.fl_level_decide, dp, 1, 1, lad, s0) == -4                         # y not 8-aligned
    dp = fl.decide_problems([(24, 64, 128, 16, 16, None)])
    assert _status(fl, fl.fl_level_decide, dp, 1, 1, lad, s0) == -4                         # store not 16-aligned
    # listed pass
    probs = fl.gemv_problems([(16, 128, 128, 16, 16, 16, 16)])
    lists, counts = fl.block_lists([16], [3])                                           # 3 > 128 / 64
    assert _status(fl, fl.fl_gemv_batched_listed, probs, lists, counts, 1, 1, 1, s0) == ERR_ARG
    lists, counts = fl.block_lists([16], [-1])
    assert _status(fl, fl.fl_gemv_batched_listed, probs, lists, counts, 1, 1, 1, s0) == ERR_ARG
    lists, counts = fl.block_lists([None], [1])                                         # NULL list
    assert _status(fl, fl.fl_gemv_batched_listed, probs, lists, counts, 1, 1, 1, s0) == ERR_ARG
    assert _status(fl, fl.fl_gemv_batched_listed, probs, None, counts, 1, 1, 1, s0) == ERR_ARG
    lists, counts = fl.block_lists([18], [1])                                           # misaligned list
    assert _status(fl, fl.fl_gemv_batched_listed, probs, lists, counts, 1, 1, 1, s0) == -4
    lists, counts = fl.block_lists([None], [0])                                         # nothing listed
    fl.fl_gemv_batched_listed(probs, lists, counts, 1, 1, 1, s0)                          # returns FL_OK
    # verified speculation
    assert _status(fl, fl.fl_spec_accept, None, 16, 4, 16, None, s0) == ERR_ARG
    assert _status(fl, fl.fl_spec_accept, 16, 16, 0, 16, None, s0) == ERR_SHAPE                 # k = 0
    assert _status(fl, fl.fl_spec_accept, 16, 16, 17, 16, None, s0) == ERR_SHAPE                # k > 16
    assert _status(fl, fl.fl_spec_accept, 16, 16, 4, 18, None, s0) == -4                        # result misaligned


def test_misaligned_pointers_rejected(fl):
    s0 = 0
    w = fl.plane_weight(17, 64, 128)
    assert _status(fl, fl.fl_gemv_depth, w, 16, 16, 1, 16, None, 0, s0) == -4
    w = fl.plane_weight(16, 64, 128)
    assert _status(fl, fl.fl_gemv_depth, w, 16, 16, 1, 18, None, 0, s0) == -4                   # y
    assert _status(fl, fl.fl_gemv_batched, fl.gemv_problems([(16, 64, 128, 16, None, 16, 18)]), 1, 1, 0, s0) == -4
    assert _status(fl, fl.fl_gemv_kquant, 16, 12, 64, 256, 16, 1, 18, None, 0, s0) == -4       # y
    assert _status(fl, fl.fl_gemv_kquant_batched, fl.kquant_problems([(16, 12, 64, 256, 16, 18)]), 1, 1, s0) == -4
    p = fl.lens_params(0.3, 0.75, 1, 4, [0.5, 1.0], 0)
    assert _status(fl, fl.fl_level_map, 18, 10, 16, 16, 8, p, 16, None, s0) == -4              # xy
    assert _status(fl, fl.fl_level_map, 16, 10, 16, 16, 8, p, 16, 17, s0) == -4                # counts
    assert _status(fl, fl.fl_pack_planes, 18, 16, 64, 128, 16, s0) == -4
