"""CUDA path vs the CPU oracle, element by element, through the C-ABI.

Bars: bit-exact for the plane store, level maps, top-2 indices and gate
decisions (outside a band where fp32 rounding could flip them); for
outputs |y_gpu - y_ref| <= 2e-3 * sum_c |w||x| + 1e-5 (fp32 accumulation).
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
    return torch, fl


def dev(torch, a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def check_close(y_gpu, y_ref, mass, what=""):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bound = REL * mass + ABS
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} outputs outside tolerance, worst ratio {(err / bound).max():.3g}"
    return float((err / bound).max())


def pack_gpu(torch, fl, q, s):
    out, inn = q.shape
    store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
    fl.fl_pack_planes(dev(torch, q), dev(torch, s), out, inn, store)
    return store


def gemv_gpu(torch, fl, store, out, inn, levels, x, mode=0, to_levels=None, y0=None):
    batch = x.shape[0]
    y = torch.zeros((batch, out), dtype=torch.float32, device="cuda") if y0 is None else dev(torch, y0.astype(np.float32))
    wsb = fl.fl_gemv_workspace_bytes(out, inn, batch)
    ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    w = fl.plane_weight(store, out, inn)
    if mode == 0:
        fl.fl_gemv_depth(w, dev(torch, levels), dev(torch, x), batch, y, ws, wsb)
    else:
        fl.fl_gemv_residual(w, dev(torch, levels), dev(torch, to_levels), dev(torch, x), batch, y, ws, wsb)
    torch.cuda.synchronize()
    return y.cpu().numpy(), ws


# ----------------------------------------------------------------------------- plane store

@pytest.mark.parametrize("out,inn", [(64, 128), (192, 1664), (1024, 1024), (128, 14336)])
def test_pack_bit_exact(env, orc, out, inn):
    torch, fl = env
    rng = synth.rng(11, out, inn)
    q = rng.integers(-128, 128, size=(out, inn)).astype(np.int8)
    s = rng.random((out, inn // 128), dtype=np.float32)
    st = pack_gpu(torch, fl, q, s).cpu().numpy()
    assert np.array_equal(st, orc.pack_planes(q, s))


def test_pack_all_codes(env, orc):
    torch, fl = env
    q = (np.arange(64 * 256) % 256 - 128).astype(np.int8).reshape(64, 256)
    s = np.linspace(0, 1, 128, dtype=np.float32).reshape(64, 2)
    assert np.array_equal(pack_gpu(torch, fl, q, s).cpu().numpy(), orc.pack_planes(q, s))


# ----------------------------------------------------------------------------- depth GEMV

CASES = [
    # out, in, batch, level spec
    (1024, 1024, 1, "uniform"),       # config-0 shape, seeded mixed depths
    (448, 1664, 1, "uniform"),        # 13 groups: ragged tiles at every depth
    (448, 1664, 3, "uniform"),
    (448, 1664, 4, "uniform"),
    (448, 1664, 5, "uniform"),        # second N-tile
    (320, 2048, 8, "uniform"),
    (320, 2048, 16, "uniform"),
    (256, 14336, 1, "uniform"),       # few blocks, wide rows: column slices + tickets
    (256, 14336, 16, "uniform"),
    (2048, 1024, 1, "d4"),
    (640, 3072, 2, "zero_heavy"),
    # batch 9 and up: the tcgen05 tensor-core path (block pairs, digits in shared memory)
    (448, 1664, 9, "uniform"),        # 7 blocks: the last pair holds one block
    (448, 1664, 17, "uniform"),
    (320, 2048, 24, "uniform"),
    (2048, 1024, 32, "d4"),
    (640, 3072, 20, "zero_heavy"),
    (64, 4096, 32, "uniform"),        # one block, column slices
    (256, 14336, 32, "uniform"),      # few blocks, wide rows: many column slices + tickets
    (7680, 1664, 16, "uniform"),      # 60 pairs: 13 groups over 10 slices of one or two groups
]


def levels_for(spec, nblocks, key):
    if spec == "uniform":
        return synth.seeded_levels(nblocks, *key)
    if spec == "d4":
        return np.full(nblocks, 2, np.uint8)
    lv = synth.seeded_levels(nblocks, *key)
    lv[::2] = 0
    return lv


@pytest.mark.parametrize("out,inn,batch,spec", CASES)
def test_gemv_depth_vs_oracle(env, orc, out, inn, batch, spec):
    torch, fl = env
    q, s = synth.int8_layer(out, inn, 21, out, inn)
    lv = levels_for(spec, out // 64, (22, out, inn))
    x = synth.bf16_normal((batch, inn), 23, out, inn, batch)
    store = pack_gpu(torch, fl, q, s)
    y, ws = gemv_gpu(torch, fl, store, out, inn, lv, x)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    check_close(y, yref, mass, f"depth {out}x{inn} b{batch}")
    zero_rows = np.repeat(lv == 0, 64)
    assert np.all(y[:, zero_rows] == 0.0)


def test_gemv_workspace_left_zero(env, orc):
    torch, fl = env
    out, inn, batch = 256, 14336, 4
    q, s = synth.int8_layer(out, inn, 24)
    lv = synth.seeded_levels(out // 64, 25)
    x = synth.bf16_normal((batch, inn), 26)
    store = pack_gpu(torch, fl, q, s)
    wsb = fl.fl_gemv_workspace_bytes(out, inn, batch)
    assert wsb > 0
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    y = torch.empty((batch, out), dtype=torch.float32, device="cuda")
    w = fl.plane_weight(store, out, inn)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    for _ in range(3):  # tickets return to zero, so repeated calls stay correct
        fl.fl_gemv_depth(w, dev(torch, lv), dev(torch, x), batch, y, ws, wsb)
        torch.cuda.synchronize()
        check_close(y.cpu().numpy(), yref, mass, "repeat")
    nt = (out // 64) * 4
    assert int(ws[:nt].count_nonzero().item()) == 0
    with pytest.raises(fl.FlError) as e:
        fl.fl_gemv_depth(w, dev(torch, lv), dev(torch, x), batch, y, ws, wsb - 16)
    assert e.value.status == -6


def test_gemv_high_dynamic_range_x(env, orc):
    """One large element per 128-column group, held to the path's bar as it stands."""
    torch, fl = env
    out, inn = 128, 1024
    q, s = synth.int8_layer(out, inn, 27)
    lv = np.array([4, 2], np.uint8)
    xf = synth.rng(28).standard_normal((1, inn), dtype=np.float32)
    xf[0, ::128] = 300.0
    x = synth.f32_to_bf16_bits(xf)
    store = pack_gpu(torch, fl, q, s)
    y, _ = gemv_gpu(torch, fl, store, out, inn, lv, x)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    check_close(y, yref, mass, "high dynamic range")


def outlier_x(batch, inn, k, *key, big=256.0):
    """bf16 activations with, in every 128-column group, one element of magnitude `big` at a
    seeded column and the other 127 elements big * 2^-k * N(0, 1). Returns (x bits, columns)."""
    g = synth.rng(*key)
    xf = (np.float32(big * 2.0 ** -k) * g.standard_normal((batch, inn), dtype=np.float32)).astype(np.float32)
    cols = np.arange(inn // 128) * 128 + g.integers(0, 128, size=inn // 128)
    xf[:, cols] = np.float32(big) * np.where(g.random((batch, cols.size)) < 0.5, -1.0, 1.0).astype(np.float32)
    return synth.f32_to_bf16_bits(xf), cols


# The hardest inputs for the activation representation: the group's largest element meets a
# weight that reconstructs to exactly 0 (a D8 code 0), so it adds nothing to sum |w||x| and
# the bar is set by the small elements alone, 2^k below it.
@pytest.mark.parametrize("k", [10, 14, 20])
@pytest.mark.parametrize("batch", [1, 3, 8, 16, 32])
def test_gemv_outlier_on_a_zero_weight(env, orc, k, batch):
    torch, fl = env
    out, inn = 192, 1664
    q, s = synth.int8_layer(out, inn, 41, k)
    x, cols = outlier_x(batch, inn, k, 42, k, batch)
    q[:, cols] = 0
    store = pack_gpu(torch, fl, q, s)
    lv = np.full(out // 64, 4, np.uint8)
    y, _ = gemv_gpu(torch, fl, store, out, inn, lv, x)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    check_close(y, yref, mass, f"D8 outlier 2^{k} b{batch}")
    lv = synth.seeded_levels(out // 64, 43, k)
    y, _ = gemv_gpu(torch, fl, store, out, inn, lv, x)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    check_close(y, yref, mass, f"mixed-depth outlier 2^{k} b{batch}")


@pytest.mark.parametrize("k", [10, 20])
def test_residual_outlier_on_a_zero_weight(env, orc, k):
    """Residual from ZERO to D8 (its weights are the D8 weights, 0 at the outlier's column)
    and D4 -> D8 (D4 + residual = D8 at the bar), on the outlier inputs."""
    torch, fl = env
    out, inn, batch = 256, 2048, 2
    q, s = synth.int8_layer(out, inn, 44, k)
    x, cols = outlier_x(batch, inn, k, 45, k)
    q[:, cols] = 0
    store = pack_gpu(torch, fl, q, s)
    a = np.zeros(out // 64, np.uint8)
    b = np.full(out // 64, 4, np.uint8)
    y, _ = gemv_gpu(torch, fl, store, out, inn, a, x, mode=1, to_levels=b)
    dref, mass = orc.gemv_residual(q, s, a, b, x, with_mass=True)
    check_close(y, dref, mass, f"ZERO -> D8 residual outlier 2^{k}")
    d4 = np.full(out // 64, 2, np.uint8)
    y4, _ = gemv_gpu(torch, fl, store, out, inn, d4, x)
    y48, _ = gemv_gpu(torch, fl, store, out, inn, d4, x, mode=1, to_levels=b, y0=y4)
    y8ref, mass8 = orc.gemv_depth(q, s, b, x, with_mass=True)
    check_close(y48, y8ref, mass8, f"D4 + residual outlier 2^{k}")


@pytest.mark.parametrize("ggml_type", [12, 14])
@pytest.mark.parametrize("k", [10, 20])
@pytest.mark.parametrize("batch", [1, 4])
def test_kquant_outlier_on_a_zero_weight(env, orc, ggml_type, k, batch):
    """Q4_K / Q6_K with the outlier's column dequantizing to exactly 0: Q6_K codes 32 (w = 0
    quantizes to q - 32 = 0); Q4_K codes 0 with a zero min in that sub-block (its weights made
    non-negative, so mn = 0 and w = d sc 0 - dmin 0 = 0)."""
    torch, fl = env
    out, inn = 128, 2048
    w = synth.gaussian_weights(out, inn, 46, ggml_type, k)
    x, cols = outlier_x(batch, inn, k, 47, ggml_type, k, batch)
    if ggml_type == 12:
        for c in cols:
            j0 = (c // 32) * 32
            w[:, j0:j0 + 32] = np.abs(w[:, j0:j0 + 32])
    w[:, cols] = 0.0
    blocks = synth.encode_kquant(w, ggml_type)
    y = torch.zeros((batch, out), dtype=torch.float32, device="cuda")
    wsb = fl.fl_kquant_workspace_bytes(ggml_type, out, inn, batch)
    ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    fl.fl_gemv_kquant(dev(torch, blocks), ggml_type, out, inn, dev(torch, x), batch, y, ws, wsb)
    torch.cuda.synchronize()
    yref, mass = orc.gemv_kquant(blocks, ggml_type, out, inn, x, with_mass=True)
    # the outlier's column adds nothing to the mass: its weight dequantizes to exactly 0
    rb, nsb = (144 if ggml_type == 12 else 210), inn // 256
    recs = blocks.reshape(-1, rb)
    for r in (0, 1, 37, out - 1):
        for c in cols:
            rec = recs[((r // 64) * nsb + c // 256) * 64 + r % 64]
            assert orc.dequant_superblock(rec, ggml_type, r)[c % 256] == 0.0
    check_close(y.cpu().numpy(), yref, mass, f"kquant {ggml_type} outlier 2^{k} b{batch}")


def test_residual_vs_oracle_and_identity(env, orc):
    torch, fl = env
    out, inn, batch = 512, 2048, 2
    q, s = synth.int8_layer(out, inn, 31)
    a = synth.seeded_levels(out // 64, 32)
    b = np.maximum(a, synth.seeded_levels(out // 64, 33))
    b[0], a[0] = 2, 3                                  # a non-raising block adds nothing
    x = synth.bf16_normal((batch, inn), 34)
    store = pack_gpu(torch, fl, q, s)
    y0 = synth.rng(35).standard_normal((batch, out)).astype(np.float32)
    y, _ = gemv_gpu(torch, fl, store, out, inn, a, x, mode=1, to_levels=b, y0=y0)
    dref, mass = orc.gemv_residual(q, s, a, b, x, with_mass=True)
    check_close(y, y0.astype(np.float64) + dref, mass, "residual")
    assert np.array_equal(y[:, :64], y0[:, :64])
    # D4 pass + residual(D4 -> D8) == D8 pass
    d4 = np.full(out // 64, 2, np.uint8)
    d8 = np.full(out // 64, 4, np.uint8)
    y4, _ = gemv_gpu(torch, fl, store, out, inn, d4, x)
    y48, _ = gemv_gpu(torch, fl, store, out, inn, d4, x, mode=1, to_levels=d8, y0=y4)
    y8ref, mass8 = orc.gemv_depth(q, s, d8, x, with_mass=True)
    check_close(y48, y8ref, mass8, "D4+res")


@pytest.mark.parametrize("batch", [9, 16, 32])
def test_residual_tensor_core_path(env, orc, batch):
    """Residual from every level pair on the tcgen05 path, column slices included, and
    D4 + residual(D4 -> D8) = D8 there."""
    torch, fl = env
    out, inn = 448, 4096
    q, s = synth.int8_layer(out, inn, 38, batch)
    a = synth.seeded_levels(out // 64, 39, batch)
    b = np.maximum(a, synth.seeded_levels(out // 64, 40, batch))
    b[0], a[0] = 2, 3                                  # a non-raising block adds nothing
    x = synth.bf16_normal((batch, inn), 41, batch)
    store = pack_gpu(torch, fl, q, s)
    y0 = synth.rng(42, batch).standard_normal((batch, out)).astype(np.float32)
    y, _ = gemv_gpu(torch, fl, store, out, inn, a, x, mode=1, to_levels=b, y0=y0)
    dref, mass = orc.gemv_residual(q, s, a, b, x, with_mass=True)
    check_close(y, y0.astype(np.float64) + dref, mass, f"tc residual b{batch}")
    assert np.array_equal(y[:, :64], y0[:, :64])
    d4 = np.full(out // 64, 2, np.uint8)
    d8 = np.full(out // 64, 4, np.uint8)
    y4, _ = gemv_gpu(torch, fl, store, out, inn, d4, x)
    y48, _ = gemv_gpu(torch, fl, store, out, inn, d4, x, mode=1, to_levels=d8, y0=y4)
    y8ref, mass8 = orc.gemv_depth(q, s, d8, x, with_mass=True)
    check_close(y48, y8ref, mass8, f"tc D4+res b{batch}")


def test_tensor_core_path_repeated_calls_leave_workspace_zero(env, orc):
    torch, fl = env
    out, inn, batch = 192, 14336, 24
    q, s = synth.int8_layer(out, inn, 43)
    lv = synth.seeded_levels(out // 64, 44)
    x = synth.bf16_normal((batch, inn), 45)
    store = pack_gpu(torch, fl, q, s)
    wsb = fl.fl_gemv_workspace_bytes(out, inn, batch)
    assert wsb > 0
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    y = torch.empty((batch, out), dtype=torch.float32, device="cuda")
    w = fl.plane_weight(store, out, inn)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    for _ in range(3):
        fl.fl_gemv_depth(w, dev(torch, lv), dev(torch, x), batch, y, ws, wsb)
        torch.cuda.synchronize()
        check_close(y.cpu().numpy(), yref, mass, "tc repeat")
    npair = (out // 64 + 1) // 2
    assert int(ws[:4 * npair].count_nonzero().item()) == 0
    fl.fl_device_status()
    with pytest.raises(fl.FlError) as e:
        fl.fl_gemv_depth(w, dev(torch, lv), dev(torch, x), batch, y, ws, wsb - 16)
    assert e.value.status == -6


def test_residual_split_columns(env, orc):
    torch, fl = env
    out, inn, batch = 128, 8192, 4
    q, s = synth.int8_layer(out, inn, 36)
    a = np.array([1, 2], np.uint8)
    b = np.array([4, 3], np.uint8)
    x = synth.bf16_normal((batch, inn), 37)
    store = pack_gpu(torch, fl, q, s)
    assert fl.fl_gemv_workspace_bytes(out, inn, batch) > 0
    y, _ = gemv_gpu(torch, fl, store, out, inn, a, x, mode=1, to_levels=b)
    dref, mass = orc.gemv_residual(q, s, a, b, x, with_mass=True)
    check_close(y, dref, mass, "residual split")


def test_batched_problems(env, orc):
    torch, fl = env
    shapes = [(2048, 1024), (1024, 1024), (1024, 2048), (3072, 1024), (1024, 3072), (640, 128)]
    batch = 2
    items, refs, keep = [], [], []
    for i, (o, n) in enumerate(shapes):
        q, s = synth.int8_layer(o, n, 41, i)
        lv = synth.seeded_levels(o // 64, 42, i)
        x = synth.bf16_normal((batch, n), 43, i)
        st = pack_gpu(torch, fl, q, s)
        y = torch.zeros((batch, o), dtype=torch.float32, device="cuda")
        lvd, xd = dev(torch, lv), dev(torch, x)
        keep += [st, lvd, xd, y]
        items.append((st, o, n, lvd, None, xd, y))
        refs.append(orc.gemv_depth(q, s, lv, x, with_mass=True))
    arr = fl.gemv_problems(items)
    fl.fl_gemv_batched(arr, len(items), batch, 0)
    torch.cuda.synchronize()
    for (st, o, n, lvd, _, xd, y), (yref, mass) in zip(items, refs):
        check_close(y.cpu().numpy(), yref, mass, f"batched {o}x{n}")


@pytest.mark.parametrize("batch,gate_index", [(1, 3), (3, 1)])
def test_batched_gate_fused(env, orc, batch, gate_index):
    """Gate fused into the batched GEMV: y as the oracle, gate outputs as the oracle's gate on
    the GPU's own logits, for the depth pass and then the residual pass to D8."""
    torch, fl = env
    shapes = [(1024, 1024), (8192, 1024), (2048, 2048), (1024, 3072)]
    items, layers, keep = [], [], []
    for i, (o, n) in enumerate(shapes):
        q, s = synth.int8_layer(o, n, 91, i)
        lv = synth.seeded_levels(o // 64, 92, i)     # the logits include ZERO and D8 blocks
        x = synth.bf16_normal((batch, n), 93, i)
        st = pack_gpu(torch, fl, q, s)
        y = torch.zeros((batch, o), dtype=torch.float32, device="cuda")
        lvd, xd, to = dev(torch, lv), dev(torch, x), torch.full((o // 64,), 4, dtype=torch.uint8, device="cuda")
        keep += [st, lvd, xd, y, to]
        items.append((st, o, n, lvd, to, xd, y))
        layers.append((q, s, lv, x))
    arr = fl.gemv_problems(items)
    V = shapes[gate_index][0]
    wsb = fl.fl_gemv_gate_workspace_bytes(batch)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    e = torch.empty(batch, dtype=torch.float32, device="cuda")
    m = torch.empty(batch, dtype=torch.float32, device="cuda")
    t2 = torch.empty((batch, 2), dtype=torch.int32, device="cuda")
    es = torch.empty(batch, dtype=torch.uint8, device="cuda")
    for mode in (0, 1):
        tau_h, tau_m = 8.5, 1e-4
        spec = fl.gate_spec(gate_index, tau_h, tau_m, e, m, t2, es, ws, wsb)
        fl.fl_gemv_batched_gate(arr, len(items), batch, mode, spec)
        torch.cuda.synchronize()
        for i, ((q, s, lv, x), it) in enumerate(zip(layers, items)):
            to_lv = np.full_like(lv, 4) if mode == 1 else lv
            yref, mass = orc.gemv_depth(q, s, to_lv, x, with_mass=True)
            check_close(it[6].cpu().numpy(), yref, mass, f"fused-gate batch mode {mode} problem {i}")
        z = items[gate_index][6].cpu().numpy()
        H, M, top2, esc = orc.logit_gate(z, tau_h, tau_m)
        ge, gm, gt, gs = e.cpu().numpy(), m.cpu().numpy(), t2.cpu().numpy(), es.cpu().numpy()
        assert np.array_equal(gt, top2), (mode, gt, top2)
        assert np.allclose(ge, H, rtol=1e-5, atol=1e-6), (mode, ge, H)
        assert np.allclose(gm, M, rtol=1e-5, atol=1e-7), (mode, gm, M)
        band = (np.abs(H - tau_h) <= 1e-4 * abs(tau_h) + 1e-6) | (np.abs(M - tau_m) <= 1e-6)
        assert np.array_equal(gs[~band], esc[~band])
        assert np.array_equal(gs, ((ge > np.float32(tau_h)) | (gm < np.float32(tau_m))).astype(np.uint8))
        assert int(ws[:4].view(torch.int32).item()) == 0, "gate counter not left at zero"
        # the standalone gate over the same logits agrees
        e2, m2 = torch.empty_like(e), torch.empty_like(m)
        t22, es2 = torch.empty_like(t2), torch.empty_like(es)
        fl.fl_logit_gate(items[gate_index][6], V, batch, tau_h, tau_m, e2, m2, t22, es2)
        torch.cuda.synchronize()
        assert np.array_equal(t22.cpu().numpy(), gt)
        assert np.allclose(e2.cpu().numpy(), ge, rtol=1e-5, atol=1e-6)


def test_conditional_escalation_on_device(env, orc):
    """The residual pass conditioned on the gate's escalate flag: it runs (y becomes the D8
    result, the run counter ticks) when the flag is set, and leaves y untouched otherwise."""
    torch, fl = env
    shapes = [(1024, 1024), (2048, 1024)]          # problem 1 is the gate's logits
    items, layers = [], []
    for i, (o, n) in enumerate(shapes):
        q, s = synth.int8_layer(o, n, 95, i)
        lv = np.full(o // 64, 2, np.uint8)
        x = synth.bf16_normal((1, n), 96, i)
        st = pack_gpu(torch, fl, q, s)
        y = torch.zeros((1, o), dtype=torch.float32, device="cuda")
        items.append((st, o, n, dev(torch, lv), torch.full((o // 64,), 4, dtype=torch.uint8, device="cuda"),
                      dev(torch, x), y))
        layers.append((q, s, lv, x))
    arr = fl.gemv_problems(items)
    wsb = fl.fl_gemv_gate_workspace_bytes(1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    e, m = torch.empty(1, device="cuda"), torch.empty(1, device="cuda")
    t2, es = torch.empty((1, 2), dtype=torch.int32, device="cuda"), torch.empty(1, dtype=torch.uint8, device="cuda")
    runs = torch.zeros(1, dtype=torch.int32, device="cuda")
    for tau_h, want in ((-1.0, 1), (1e9, 0)):                        # H > -1 always; H > 1e9 never
        spec = fl.gate_spec(1, tau_h, -1.0, e, m, t2, es, ws, wsb)     # margin < -1 never
        fl.fl_gemv_batched_gate(arr, 2, 1, 0, spec)
        fl.fl_gemv_batched_gate_if(arr, 2, 1, 1, spec, es, runs)
        torch.cuda.synchronize()
        assert int(es.item()) == want
        for (q, s, lv, x), it in zip(layers, items):
            yref, mass = orc.gemv_depth(q, s, np.full_like(lv, 4) if want else lv, x, with_mass=True)
            check_close(it[6].cpu().numpy(), yref, mass, f"conditional pass, escalate={want}")
    assert int(runs.item()) == 1


# ----------------------------------------------------------------------------- level map

def test_level_map_bit_exact(env, orc, golden):
    torch, fl = env
    nb = 14708
    xy, cxy, r = synth.lens_inputs(nb, 8, 51)
    for (f, g, gamma, combine) in ((0.3, 0.75, 1, 0), (0.3, 0.75, 1, 1), (0.5, 1.0, 0, 0), (0.3, 0.75, 3, 0),
                                   (0.3, 1.0, 3, 0), (0.9, 0.5, 2, 1), (0.0, 0.75, 1, 0)):
        kappa = orc.lens_kappa(g, gamma, 4)
        stops = synth.even_stops(kappa, gamma)
        ref = orc.level_map(xy, cxy, r * (4 if f < 0.5 else 1), f, g, gamma, 4, stops, combine)
        lev = torch.empty(nb, dtype=torch.uint8, device="cuda")
        cnt = torch.zeros(5, dtype=torch.int32, device="cuda")
        p = fl.lens_params(f, g, gamma, 4, stops, combine)
        fl.fl_level_map(dev(torch, xy), nb, dev(torch, cxy), dev(torch, r * (4 if f < 0.5 else 1)), 8, p, lev, cnt)
        torch.cuda.synchronize()
        got = lev.cpu().numpy()
        assert np.array_equal(got, ref), (f, g, gamma, combine, (got != ref).sum())
        assert np.array_equal(cnt.cpu().numpy(), np.bincount(ref, minlength=5))
    gd = golden("lens_hand_maps.json")
    P = gd["params"]
    one = gd["single_lens"]
    blocks = np.array(one["blocks"], np.float32)
    lev = torch.empty(len(blocks), dtype=torch.uint8, device="cuda")
    p = fl.lens_params(P["f"], P["g"], P["gamma"], P["m"], P["stops"], 0)
    fl.fl_level_map(dev(torch, blocks), len(blocks), dev(torch, np.array([one["center"]], np.float32)),
                    dev(torch, np.array([one["r"]], np.float32)), 1, p, lev, None)
    torch.cuda.synchronize()
    assert lev.cpu().numpy().tolist() == one["levels_sum"]


# ----------------------------------------------------------------------------- gate

@pytest.mark.parametrize("vocab,batch", [(151936, 1), (151936, 3), (128256, 16), (1000, 2), (4, 1)])
def test_logit_gate_vs_oracle(env, orc, vocab, batch):
    torch, fl = env
    z = synth.rng(61, vocab, batch).standard_normal((batch, vocab), dtype=np.float32) * np.float32(0.7)
    if batch > 1:
        z[1, 17] = 9.0
        z[1, 5000 % vocab] = 9.0       # a tie for the top
    H, M, top2, _ = orc.logit_gate(z, 0.0, 0.0)
    tau_h, tau_m = float(np.median(H)), float(np.median(M))
    _, _, _, esc_ref = orc.logit_gate(z, tau_h, tau_m)
    zd = dev(torch, z)
    e = torch.empty(batch, dtype=torch.float32, device="cuda")
    m = torch.empty(batch, dtype=torch.float32, device="cuda")
    t2 = torch.empty((batch, 2), dtype=torch.int32, device="cuda")
    es = torch.empty(batch, dtype=torch.uint8, device="cuda")
    fl.fl_logit_gate(zd, vocab, batch, tau_h, tau_m, e, m, t2, es)
    torch.cuda.synchronize()
    e, m, t2, es = e.cpu().numpy(), m.cpu().numpy(), t2.cpu().numpy(), es.cpu().numpy()
    assert np.array_equal(t2, top2)
    assert np.allclose(e, H, rtol=1e-5, atol=1e-6)
    assert np.allclose(m, M, rtol=1e-5, atol=1e-7)
    band = (np.abs(H - tau_h) <= 1e-4 * abs(tau_h) + 1e-6) | (np.abs(M - tau_m) <= 1e-6)
    assert np.array_equal(es[~band], esc_ref[~band])
    assert np.array_equal(es, ((e > np.float32(tau_h)) | (m < np.float32(tau_m))).astype(np.uint8))


def test_logit_gate_closed_forms(env):
    torch, fl = env
    V = 151936
    z = np.full((2, V), 0.5, np.float32)
    z[1, 1234] = 300.0
    e = torch.empty(2, dtype=torch.float32, device="cuda")
    m = torch.empty(2, dtype=torch.float32, device="cuda")
    t2 = torch.empty((2, 2), dtype=torch.int32, device="cuda")
    es = torch.empty(2, dtype=torch.uint8, device="cuda")
    fl.fl_logit_gate(dev(torch, z), V, 2, 5.0, 0.5, e, m, t2, es)
    torch.cuda.synchronize()
    e, m, t2, es = e.cpu().numpy(), m.cpu().numpy(), t2.cpu().numpy(), es.cpu().numpy()
    assert abs(e[0] - np.log(V)) <= 1e-5 * np.log(V) and m[0] == 0.0 and t2[0].tolist() == [0, 1] and es[0] == 1
    assert e[1] < 1e-6 and m[1] == 1.0 and t2[1].tolist() == [1234, 0] and es[1] == 0


# ----------------------------------------------------------------------------- K-quant

@pytest.mark.parametrize("ggml_type,out,inn,batch", [
    (12, 512, 2048, 1), (12, 192, 8192, 3), (12, 64, 256, 1), (12, 128, 1280, 5), (12, 256, 2048, 16),
    (14, 512, 2048, 1), (14, 192, 8192, 4), (14, 128, 4096, 8), (14, 64, 2048, 16),
    (14, 128, 1280, 3), (14, 64, 768, 1),
])
def test_kquant_vs_oracle(env, orc, ggml_type, out, inn, batch):
    torch, fl = env
    w = synth.gaussian_weights(out, inn, 71, ggml_type, out, inn)
    blocks = synth.encode_kquant(w, ggml_type)
    x = synth.bf16_normal((batch, inn), 72, out, inn, batch)
    y = torch.zeros((batch, out), dtype=torch.float32, device="cuda")
    wsb = fl.fl_kquant_workspace_bytes(ggml_type, out, inn, batch)
    ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    fl.fl_gemv_kquant(dev(torch, blocks), ggml_type, out, inn, dev(torch, x), batch, y, ws, wsb)
    torch.cuda.synchronize()
    yref, mass = orc.gemv_kquant(blocks, ggml_type, out, inn, x, with_mass=True)
    check_close(y.cpu().numpy(), yref, mass, f"kquant {ggml_type} {out}x{inn} b{batch}")


def test_kquant_negative_and_saturated_scales(env, orc):
    """Q6_K int8 scales of both signs (and -128), Q4_K scales/mins at 0 and 63."""
    torch, fl = env
    out, inn = 128, 4096
    w = synth.gaussian_weights(out, inn, 75)
    b6 = synth.encode_kquant(w, fl.FL_GGML_Q6_K).reshape(-1, 210).copy()
    rng = synth.rng(76)
    for i in range(b6.shape[0]):
        base = 192 if i % 2 == 0 else 194
        sc = b6[i, base:base + 16].view(np.int8)
        sc[:] = rng.integers(-128, 128, 16).astype(np.int8)
    b4 = synth.encode_kquant(w, fl.FL_GGML_Q4_K).reshape(-1, 144).copy()
    b4[::3, 4:12] = 63 | (3 << 6)                      # sc = 63, mn low bits 3
    b4[::3, 12:16] = 0xFF                              # mn = 63
    b4[1::3, 4:12] = 0                                 # sc = mn = 0 -> only -dmin*0
    x = synth.bf16_normal((2, inn), 77)
    for t, blk in ((fl.FL_GGML_Q6_K, b6.reshape(-1)), (fl.FL_GGML_Q4_K, b4.reshape(-1))):
        y = torch.zeros((2, out), dtype=torch.float32, device="cuda")
        wsb = fl.fl_kquant_workspace_bytes(t, out, inn, 2)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        fl.fl_gemv_kquant(dev(torch, blk), t, out, inn, dev(torch, x), 2, y, ws, wsb)
        torch.cuda.synchronize()
        yref, mass = orc.gemv_kquant(blk, t, out, inn, x, with_mass=True)
        check_close(y.cpu().numpy(), yref, mass, f"kquant edge {t}")


def test_kquant_batched_mixed_types(env, orc):
    torch, fl = env
    mix = [(12, 2048, 2048), (14, 512, 2048), (12, 512, 2048), (14, 2048, 8192), (12, 1024, 4096)]
    batch = 1
    items, refs, keep = [], [], []
    for i, (t, o, n) in enumerate(mix):
        w = synth.gaussian_weights(o, n, 73, i)
        blk = synth.encode_kquant(w, t)
        x = synth.bf16_normal((batch, n), 74, i)
        bd, xd = dev(torch, blk), dev(torch, x)
        y = torch.zeros((batch, o), dtype=torch.float32, device="cuda")
        keep += [bd, xd, y]
        items.append((bd, t, o, n, xd, y))
        refs.append(orc.gemv_kquant(blk, t, o, n, x, with_mass=True))
    fl.fl_gemv_kquant_batched(fl.kquant_problems(items), len(items), batch)
    torch.cuda.synchronize()
    for (bd, t, o, n, xd, y), (yref, mass) in zip(items, refs):
        check_close(y.cpu().numpy(), yref, mass, f"kq batched {t} {o}x{n}")


def test_kquant_unsupported_type_fails_on_device_box(env):
    torch, fl = env
    x = torch.zeros((1, 256), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    blk = torch.zeros(64 * 176, dtype=torch.uint8, device="cuda")
    with pytest.raises(fl.FlError) as e:
        fl.fl_gemv_kquant(blk, 13, 64, 256, x, 1, y)
    assert e.value.status == -3


# ----------------------------------------------------------------------------- failure detection

def test_device_status_reports_a_bounded_wait_that_ran_out(env, orc):
    """A wait that nothing completes runs out at its deadline (1 ms on the global timer for the
    self-test, 1 s in the kernels); fl_device_status reports it once and clears it, and the
    context keeps working. The wait is timed with CUDA events: the deadline is a time, not a
    poll count, so it must end within a few ms of 1 ms."""
    torch, fl = env
    fl.fl_device_status()                                   # clean slate (raises if anything ran out)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    fl.fl_selftest_wait_timeout()
    ev1.record()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    assert 1.0 <= ms < 50.0, ms
    with pytest.raises(fl.FlError) as e:
        fl.fl_device_status()
    assert e.value.status == -7 and "self-test" in str(e.value)
    fl.fl_device_status()                                   # cleared
    q, s = synth.int8_layer(256, 512, 97, 0)
    lv = synth.seeded_levels(4, 97, 1)
    x = synth.bf16_normal((1, 512), 97, 2)
    y, _ = gemv_gpu(torch, fl, pack_gpu(torch, fl, q, s), 256, 512, lv, x)
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    check_close(y, yref, mass, "GEMV after a reported time-out")
    fl.fl_device_status()
