"""The allocation-free depth GEMV (fixed scratch array in the library's device image),
through the C-ABI.

Two calls in a row on different shapes, batches and depth maps: the second runs on
the scratch the first left behind. Both shapes split their columns across CTAs, so
the scratch is really used. Each output is checked against the CPU oracle at the
path's bar, |y_static - y_oracle| <= 2e-3 * sum_c |w||x| + 1e-5, and against
fl_gemv_depth with a caller workspace at the same bar. Once the library's device
image is loaded, further calls must not change the device's free memory.
"""
import numpy as np
import pytest

from variable_precision_weight_b200 import synth

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-5


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from variable_precision_weight_b200 import build
    build.build()
    from variable_precision_weight_b200 import fl
    torch.cuda.set_device(0)
    return torch, fl


def _dev(torch, a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


@pytest.mark.parametrize("order", ["small_first", "large_first"])
def test_static_scratch_matches_caller_workspace(env, orc, order):
    torch, fl = env
    cases = [(1024, 4096, 1, 11), (2048, 6144, 3, 12)]
    if order == "large_first":
        cases = cases[::-1]
    for out, inn, batch, seed in cases:
        wsb = fl.fl_gemv_workspace_bytes(out, inn, batch)
        assert 0 < wsb <= fl.FL_GEMV_STATIC_SCRATCH_BYTES, wsb
        q, s = synth.int8_layer(out, inn, seed, 1)
        lv = synth.seeded_levels(out // 64, seed, 2)
        x = synth.bf16_normal((batch, inn), seed, 3)
        store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(_dev(torch, q), _dev(torch, s), out, inn, store)
        w = fl.plane_weight(store, out, inn)
        lv_d, x_d = _dev(torch, lv), _dev(torch, x)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        y_ws = torch.empty((batch, out), dtype=torch.float32, device="cuda")
        fl.fl_gemv_depth(w, lv_d, x_d, batch, y_ws, ws, wsb)
        y_st = torch.full((batch, out), float("nan"), dtype=torch.float32, device="cuda")
        fl.fl_gemv_depth_static(w, lv_d, x_d, batch, y_st)
        torch.cuda.synchronize()
        yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
        bound = REL * mass + ABS
        y_static = y_st.cpu().numpy().astype(np.float64)
        err = np.abs(y_static - yref)
        assert np.all(err <= bound), (out, inn, batch, float(np.nanmax(err / bound)))
        err_ws = np.abs(y_static - y_ws.cpu().numpy())
        assert np.all(err_ws <= bound), (out, inn, batch, float(np.nanmax(err_ws / bound)))


def test_static_calls_allocate_nothing(env):
    """After one call has loaded the library's image, calls of several shapes leave the
    device's free memory where it was (cudaMemGetInfo counts every allocation on the device,
    torch's caching allocator included)."""
    torch, fl = env
    shapes = [(1024, 4096, 1), (2048, 6144, 3), (512, 14336, 16), (256, 1024, 2)]
    bufs = []
    for out, inn, batch in shapes:
        q, s = synth.int8_layer(out, inn, 5, out)
        store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(_dev(torch, q), _dev(torch, s), out, inn, store)
        lv = _dev(torch, synth.seeded_levels(out // 64, 6, out))
        x = _dev(torch, synth.bf16_normal((batch, inn), 7, out))
        y = torch.empty((batch, out), dtype=torch.float32, device="cuda")
        bufs.append((fl.plane_weight(store, out, inn), lv, x, batch, y))
    w, lv, x, batch, y = bufs[0]
    fl.fl_gemv_depth_static(w, lv, x, batch, y)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        for w, lv, x, batch, y in bufs:
            fl.fl_gemv_depth_static(w, lv, x, batch, y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    fl.fl_device_status()


def test_static_scratch_rejects_oversized_split(env):
    torch, fl = env
    out, inn, batch = 65536, 8192, 16
    assert fl.fl_gemv_workspace_bytes(out, inn, batch) > fl.FL_GEMV_STATIC_SCRATCH_BYTES
    # rejected on the host before anything is read: the buffers are never touched
    dummy = torch.empty(256, dtype=torch.uint8, device="cuda")
    w = fl.plane_weight(dummy, out, inn)
    with pytest.raises(fl.FlError) as e:
        fl.fl_gemv_depth_static(w, dummy, dummy, batch, dummy)
    assert e.value.status == -6 and "scratch" in str(e.value)
