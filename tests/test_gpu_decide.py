"""In-pass level decision on the GPU vs the oracle, through the C-ABI.

The decision reads the base-level outputs of the layer, which both sides take from the
same buffer (the GPU's base pass), and the layer's scales. Bars: reduced scores within
1e-5 relative; ladder levels equal to the oracle's except where the oracle's score lies
within 1e-4 (relative) of a threshold lambda 16^j, and always equal to the ladder applied
to the kernel's own fp32 scores; share levels equal to the top floor(f n) blocks by the
kernel's own scores (lower index first on ties), and to the oracle's set except where
scores at the cut lie within 1e-4 of each other.
"""
import numpy as np
import pytest

from variable_precision_weight_b200 import synth

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-5
BAND = 1e-4


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


def pack_gpu(torch, fl, q, s):
    out, inn = q.shape
    store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
    fl.fl_pack_planes(dev(torch, q), dev(torch, s), out, inn, store)
    return store


def ladder_of(score, gamma, kappa, lam):
    """The ladder applied in fp32 to the kernel's own scores."""
    sc = np.asarray(score, np.float32)
    lev = np.full(sc.shape, gamma, np.int64)
    thr = np.float32(lam)
    for _ in range(kappa - gamma):
        thr = np.float32(thr * np.float32(16))
        lev += sc >= thr
    return lev.astype(np.uint8)


def share_of(score, gamma, kappa, f):
    sc = np.asarray(score, np.float32)
    nb = len(sc)
    n_up = int(np.floor(np.float64(np.float32(f)) * nb))
    order = np.lexsort((np.arange(nb), -sc.astype(np.float64)))
    lev = np.full(nb, gamma, np.uint8)
    lev[order[:n_up]] = kappa
    return lev


def check_ladder(lev, score, ref_lev, ref_red, gamma, kappa, lam, what):
    assert np.allclose(score, ref_red, rtol=1e-5, atol=0), what
    assert np.array_equal(lev, ladder_of(score, gamma, kappa, lam)), what
    thr = np.float64(np.float32(lam)) * 16.0 ** np.arange(1, kappa - gamma + 1)
    near = np.zeros(len(ref_red), bool)
    for t in thr:
        near |= np.abs(ref_red - t) <= BAND * t
    assert np.array_equal(lev[~near], ref_lev[~near]), what


def check_share(lev, score, ref_lev, ref_red, gamma, kappa, f, what):
    assert np.allclose(score, ref_red, rtol=1e-5, atol=0), what
    assert np.array_equal(lev, share_of(score, gamma, kappa, f)), what
    up, ref_up = lev == kappa, ref_lev == kappa
    assert up.sum() == ref_up.sum(), what
    diff = up != ref_up
    if diff.any():
        cut = np.sort(ref_red)[::-1][up.sum() - 1]
        assert np.all(np.abs(ref_red[diff] - cut) <= BAND * cut), what


def base_layers(torch, fl, shapes, gamma, batch, key):
    """Packed layers, their base-level pass (one batched launch) and the host copies."""
    items, host, keep = [], [], []
    for i, (o, n) in enumerate(shapes):
        q, s = synth.int8_layer(o, n, key, i)
        s = s * synth.rng(key, 50 + i).uniform(0.25, 4.0, (o // 64, 1, 1)).astype(np.float32).repeat(64, 1).reshape(o, -1)
        x = synth.bf16_normal((batch, n), key, 100 + i)
        st = pack_gpu(torch, fl, q, s)
        lv = torch.full((o // 64,), gamma, dtype=torch.uint8, device="cuda")
        xd = dev(torch, x)
        y = torch.empty((batch, o), dtype=torch.float32, device="cuda")
        keep += [st, lv, xd, y]
        items.append((st, o, n, lv, None, xd, y))
        host.append((q, s, x))
    fl.fl_gemv_batched(fl.gemv_problems(items), len(items), batch, 0)
    return items, host, keep


@pytest.mark.parametrize("gamma,batch", [(1, 1), (2, 1), (2, 3), (3, 16)])
def test_ladder_and_share_vs_oracle(env, orc, gamma, batch):
    torch, fl = env
    shapes = [(64 * 37, 384), (1024, 1024), (2048, 1024), (64, 128), (64 * 300, 256)]
    items, host, keep = base_layers(torch, fl, shapes, gamma, batch, 300 + gamma + batch)
    torch.cuda.synchronize()
    kappa = 4
    ys = [it[6].cpu().numpy() for it in items]
    refs = [orc.level_decide(y, s, gamma, kappa, 0, lam=1.0)[1] for y, (q, s, x) in zip(ys, host)]
    allr = np.concatenate(refs)
    lam = float(np.median(allr)) / 16 / 2            # about half lifted once, some twice
    lv_out = [torch.empty(o // 64, dtype=torch.uint8, device="cuda") for o, _ in shapes]
    sc_out = [torch.empty(o // 64, dtype=torch.float32, device="cuda") for o, _ in shapes]
    up_out = [torch.full((o // 64,), -1, dtype=torch.int32, device="cuda") for o, _ in shapes]
    probs = fl.decide_problems([(it[0], it[1], it[2], it[6], lv, sc, up)
                                for it, lv, sc, up in zip(items, lv_out, sc_out, up_out)])
    counters = torch.zeros(len(shapes), dtype=torch.int32, device="cuda")
    for rule, lam_, f, one in ((fl.FL_DECIDE_LADDER, lam, 0.0, False), (fl.FL_DECIDE_LADDER, 0.0, 0.0, False),
                               (fl.FL_DECIDE_LADDER, 1e30, 0.0, False), (fl.FL_DECIDE_SHARE, 0.0, 0.0, False),
                               (fl.FL_DECIDE_SHARE, 0.0, 0.16, False), (fl.FL_DECIDE_SHARE, 0.0, 0.5, False),
                               (fl.FL_DECIDE_SHARE, 0.0, 1.0, False), (fl.FL_DECIDE_SHARE, 0.0, 0.0, True),
                               (fl.FL_DECIDE_SHARE, 0.0, 0.16, True), (fl.FL_DECIDE_SHARE, 0.0, 0.5, True),
                               (fl.FL_DECIDE_SHARE, 0.0, 1.0, True)):
        for t in up_out:
            t.fill_(-1)
        fl.fl_level_decide(probs, len(shapes), batch,
                           fl.decide_params(rule, gamma, kappa, lam_, f, counters if one else None))
        torch.cuda.synchronize()
        assert int(counters.abs().sum().item()) == 0          # the one-launch counters are left zero
        for i, (y, (q, s, x)) in enumerate(zip(ys, host)):
            lev, sc = lv_out[i].cpu().numpy(), sc_out[i].cpu().numpy()
            ref_lev, ref_red = orc.level_decide(y, s, gamma, kappa, rule, lam=lam_, f=np.float32(f))
            what = f"rule {rule} lam {lam_} f {f} one launch {one} problem {i}"
            if rule == fl.FL_DECIDE_LADDER:
                check_ladder(lev, sc, ref_lev, ref_red, gamma, kappa, lam_, what)
            else:
                check_share(lev, sc, ref_lev, ref_red, gamma, kappa, f, what)
                up = np.flatnonzero(lev == kappa) if kappa > gamma else np.arange(0)
                got = up_out[i].cpu().numpy()
                assert np.array_equal(got[:len(up)], up), what          # ascending lifted indices
                assert np.all(got[len(up):] == -1) or len(up) == 0 or rule == fl.FL_DECIDE_SHARE
    # ladder without a score array: the same levels as the ladder over the scores just written
    # (the same fp32 computation), and the oracle's outside the band
    probs = fl.decide_problems([(it[0], it[1], it[2], it[6], lv, None) for it, lv in zip(items, lv_out)])
    fl.fl_level_decide(probs, len(shapes), batch, fl.decide_params(fl.FL_DECIDE_LADDER, gamma, kappa, lam))
    torch.cuda.synchronize()
    for i, (y, (q, s, x)) in enumerate(zip(ys, host)):
        lev, sc = lv_out[i].cpu().numpy(), sc_out[i].cpu().numpy()
        ref_lev, ref_red = orc.level_decide(y, s, gamma, kappa, 0, lam=lam)
        check_ladder(lev, sc, ref_lev, ref_red, gamma, kappa, lam, f"no-score ladder problem {i}")


@pytest.mark.parametrize("one", [False, True])
@pytest.mark.parametrize("nb", [10, 400])
def test_share_ties_go_to_lower_index(env, orc, nb, one):
    """Identical blocks give bit-identical scores; the share lifts the lowest indices (10
    blocks: the one-warp ranking; 400: the radix select, the cut inside the tied group)."""
    torch, fl = env
    o, n = 64 * nb, 256
    q1, s1 = synth.int8_layer(64, n, 61)
    q, s = np.tile(q1, (nb, 1)), np.tile(s1, (nb, 1))
    y = np.tile(synth.rng(62).standard_normal(64).astype(np.float32), (2, nb))
    if nb > 10:                                # blocks 0-99 score higher, then 300 tied ones
        s[:64 * 100] *= np.float32(2)
    st = pack_gpu(torch, fl, q, s)
    yd = torch.from_numpy(y).cuda()
    lv = torch.empty(nb, dtype=torch.uint8, device="cuda")
    sc = torch.empty(nb, dtype=torch.float32, device="cuda")
    f = 0.35
    counters = torch.zeros(1, dtype=torch.int32, device="cuda") if one else None
    fl.fl_level_decide(fl.decide_problems([(st, o, n, yd, lv, sc)]), 1, 2,
                       fl.decide_params(fl.FL_DECIDE_SHARE, 2, 3, f=f, counters=counters))
    torch.cuda.synchronize()
    n_up = int(np.floor(np.float64(np.float32(f)) * nb))
    scores = sc.cpu().numpy()
    tied = scores[-1]
    assert np.all(scores[(100 if nb > 10 else 0):] == tied)
    assert lv.cpu().numpy().tolist() == [3] * n_up + [2] * (nb - n_up)
    assert np.array_equal(orc.level_decide(y, s, 2, 3, 1, f=np.float32(f))[0], lv.cpu().numpy())


@pytest.mark.parametrize("rule,one", [(0, False), (1, False), (1, True)])
def test_in_pass_pipeline(env, orc, rule, one):
    """Base pass at D4 -> decision -> residual pass from D4 to the decided levels, all layers
    in one launch each: y equals the oracle's depth GEMV at the decided levels."""
    torch, fl = env
    gamma, kappa, batch = 2, 4, 1
    shapes = [(1024, 1024), (3072, 1024), (1024, 3072), (64 * 37, 384)]
    items, host, keep = base_layers(torch, fl, shapes, gamma, batch, 400 + rule)
    torch.cuda.synchronize()
    ys = [it[6].cpu().numpy() for it in items]
    allr = np.concatenate([orc.level_decide(y, s, gamma, kappa, 0, lam=1.0)[1] for y, (q, s, x) in zip(ys, host)])
    lam = float(np.quantile(allr, 0.84)) / 16        # about 16% lifted at least one rung
    to = [torch.empty(o // 64, dtype=torch.uint8, device="cuda") for o, _ in shapes]
    sc = [torch.empty(o // 64, dtype=torch.float32, device="cuda") for o, _ in shapes]
    up = [torch.empty(o // 64, dtype=torch.int32, device="cuda") for o, _ in shapes]
    probs = fl.decide_problems([(it[0], it[1], it[2], it[6], t, c, u) for it, t, c, u in zip(items, to, sc, up)])
    counters = torch.zeros(len(shapes), dtype=torch.int32, device="cuda") if one else None
    params = fl.decide_params(rule, gamma, kappa, lam, 0.16, counters)
    fl.fl_level_decide(probs, len(shapes), batch, params)
    res = [(it[0], it[1], it[2], it[3], t, it[5], it[6]) for it, t in zip(items, to)]
    if rule == fl.FL_DECIDE_SHARE:          # residual over the lifted blocks only
        counts = [int(np.floor(np.float64(np.float32(0.16)) * (o // 64))) for o, _ in shapes]
        fl.fl_gemv_batched_listed(fl.gemv_problems(res), *fl.block_lists(up, counts), len(res), batch, 1)
    else:
        fl.fl_gemv_batched(fl.gemv_problems(res), len(res), batch, 1)
    torch.cuda.synchronize()
    lifted = 0
    for i, ((q, s, x), it, t, c, y0) in enumerate(zip(host, items, to, sc, ys)):
        lev = t.cpu().numpy()
        ref_lev, ref_red = orc.level_decide(y0, s, gamma, kappa, rule, lam=lam, f=np.float32(0.16))
        if rule == 0:
            check_ladder(lev, c.cpu().numpy(), ref_lev, ref_red, gamma, kappa, lam, f"pipeline problem {i}")
        else:
            check_share(lev, c.cpu().numpy(), ref_lev, ref_red, gamma, kappa, 0.16, f"pipeline problem {i}")
        lifted += int((lev > gamma).sum())
        yref, mass = orc.gemv_depth(q, s, lev, x, with_mass=True)
        err = np.abs(it[6].cpu().numpy().astype(np.float64) - yref)
        assert np.all(err <= REL * mass + ABS), f"pipeline y, problem {i}"
    assert lifted > 0


@pytest.mark.parametrize("one", [False, True])
def test_share_rule_on_a_layer_too_large_for_shared_memory(env, orc, one):
    """A layer of 12,000 blocks: the selection reads the scores from global memory."""
    torch, fl = env
    o, n = 64 * 12000, 128
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    q = torch.randint(-127, 128, (o, n), dtype=torch.int8, device="cuda", generator=gen)
    s = torch.rand((o, 1), device="cuda", generator=gen).mul_(1e-2)
    s[64 * 100:64 * 140] = s[0:64].repeat(40, 1)          # 41 blocks with equal scales ...
    y = torch.randn((1, o), device="cuda", generator=gen)
    y[:, 64 * 100:64 * 140] = y[:, 0:64].repeat(1, 40)    # ... and equal outputs: equal scores
    st = torch.empty(fl.fl_plane_store_bytes(o, n), dtype=torch.uint8, device="cuda")
    fl.fl_pack_planes(q, s, o, n, st)
    lv = torch.empty(o // 64, dtype=torch.uint8, device="cuda")
    sc = torch.empty(o // 64, dtype=torch.float32, device="cuda")
    ref_red = orc.level_decide(y.cpu().numpy(), s.cpu().numpy(), 2, 4, 0, lam=1.0)[1]
    rank0 = int((ref_red > ref_red[0]).sum())             # blocks scoring above the tied group
    for f in (0.25, (rank0 + 20) / 12000, 0.999):          # the second cuts the tied group
        counters = torch.zeros(1, dtype=torch.int32, device="cuda") if one else None
        fl.fl_level_decide(fl.decide_problems([(st, o, n, y, lv, sc)]), 1, 1,
                           fl.decide_params(fl.FL_DECIDE_SHARE, 2, 4, f=f, counters=counters))
        torch.cuda.synchronize()
        ref_lev, ref_red = orc.level_decide(y.cpu().numpy(), s.cpu().numpy(), 2, 4, 1, f=np.float32(f))
        check_share(lv.cpu().numpy(), sc.cpu().numpy(), ref_lev, ref_red, 2, 4, f, f"large layer f {f}")


@pytest.mark.parametrize("mode,batch", [(1, 1), (1, 5), (0, 2)])
def test_batched_listed_vs_oracle(env, orc, mode, batch):
    """Listed blocks only (any order): they become the oracle's result at their levels; every
    other output row keeps its previous value bit for bit."""
    torch, fl = env
    shapes = [(64 * 37, 384), (1024, 1024), (64, 128), (2048, 256)]
    g = synth.rng(808, mode, batch)
    items, host, keep, lists, counts, picked = [], [], [], [], [], []
    for i, (o, n) in enumerate(shapes):
        q, s = synth.int8_layer(o, n, 809, i)
        x = synth.bf16_normal((batch, n), 810, i)
        st = pack_gpu(torch, fl, q, s)
        nb = o // 64
        frm = np.full(nb, 2, np.uint8)
        to = g.integers(0, 5, nb).astype(np.uint8) if mode == 0 else np.full(nb, 4, np.uint8)
        pick = g.permutation(nb)[:int(g.integers(0, nb + 1)) if i != 2 else 1].astype(np.int32)
        y0 = g.standard_normal((batch, o)).astype(np.float32)
        lvf, lvt, xd, y = dev(torch, frm if mode == 1 else to), dev(torch, to), dev(torch, x), dev(torch, y0)
        lst = dev(torch, pick if len(pick) else np.zeros(1, np.int32))
        keep += [st, lvf, lvt, xd, y, lst]
        items.append((st, o, n, lvf, lvt, xd, y))
        host.append((q, s, x, frm, to, y0))
        lists.append(lst)
        counts.append(len(pick))
        picked.append(pick)
    fl.fl_gemv_batched_listed(fl.gemv_problems(items), *fl.block_lists(lists, counts), len(items), batch, mode)
    torch.cuda.synchronize()
    for i, ((q, s, x, frm, to, y0), it, pick) in enumerate(zip(host, items, picked)):
        y = it[6].cpu().numpy()
        rows = np.zeros(y.shape[1], bool)
        for b in pick:
            rows[64 * b:64 * b + 64] = True
        assert np.array_equal(y[:, ~rows], y0[:, ~rows]), f"unlisted rows changed, problem {i}"
        if rows.any():
            if mode == 1:
                yref, mass = orc.gemv_residual(q, s, frm, to, x, with_mass=True)
                yref = yref + y0
            else:
                yref, mass = orc.gemv_depth(q, s, to, x, with_mass=True)
            err = np.abs(y[:, rows] - yref[:, rows])
            assert np.all(err <= REL * mass[:, rows] + ABS + 1e-6 * np.abs(y0[:, rows])), f"problem {i}"


def test_listed_pass_skips_and_reports_an_index_out_of_range(env, orc):
    """A device list holding an index past the layer: that unit is skipped, the valid ones are
    computed, and fl_device_status reports the bad list."""
    torch, fl = env
    o, n = 1024, 256
    q, s = synth.int8_layer(o, n, 820)
    x = synth.bf16_normal((1, n), 821)
    st = pack_gpu(torch, fl, q, s)
    lv = torch.full((o // 64,), 3, dtype=torch.uint8, device="cuda")
    y = torch.full((1, o), 7.0, dtype=torch.float32, device="cuda")
    xd = dev(torch, x)
    lst = dev(torch, np.array([3, o // 64 + 5, 9], np.int32))
    fl.fl_device_status()                                     # nothing pending before
    fl.fl_gemv_batched_listed(fl.gemv_problems([(st, o, n, lv, None, xd, y)]), *fl.block_lists([lst], [3]), 1, 1, 0)
    with pytest.raises(fl.FlError) as e:
        fl.fl_device_status()
    assert e.value.status == -1 and "out of range" in fl.fl_last_error()
    fl.fl_device_status()                                     # the error word was cleared
    yg = y.cpu().numpy()
    yref, mass = orc.gemv_depth(q, s, np.full(o // 64, 3, np.uint8), x, with_mass=True)
    for b in range(o // 64):
        r = slice(64 * b, 64 * b + 64)
        if b in (3, 9):
            assert np.all(np.abs(yg[:, r] - yref[:, r]) <= REL * mass[:, r] + ABS), b
        else:
            assert np.all(yg[:, r] == 7.0), b
