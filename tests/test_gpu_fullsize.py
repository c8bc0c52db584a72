"""Parity at the configurations' full sizes, in the launch configuration bench.py times, on
sampled outputs the oracle computes one block at a time.

Weights are seeded random int8 codes and scales (or K-quant records) drawn on the device
with torch's generator; the oracle gets the raw codes of the sampled 64-row blocks, never
the packed store. Sampled: the first, a middle and the last block of every tensor. The gate
outputs are checked against the oracle's gate over the full logits the GPU produced.
Bar: |y_gpu - y_ref| <= 2e-3 * sum_c |w||x| + 1e-5.
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


def _check(y, yref, mass, what):
    err = np.abs(y.astype(np.float64) - yref)
    bound = REL * mass + ABS
    assert np.all(err <= bound), f"{what}: worst ratio {(err / bound).max():.3g}"


def _sample_blocks(nblocks):
    return sorted({0, nblocks // 2, nblocks - 1})


def _int8_layer(torch, out, inn, gen):
    q = torch.randint(-127, 128, (out, inn), dtype=torch.int8, device="cuda", generator=gen)
    s = torch.rand((out, inn // 128), device="cuda", generator=gen).mul_(1e-3)
    return q, s


def _x(torch, batch, inn, gen):
    return torch.randn((batch, inn), device="cuda", generator=gen).to(torch.bfloat16).view(torch.int16)


def test_decode_step_batched_pass_full_size(env, orc):
    """The Qwen3-0.6B-shaped step: 197 problems, D4 pass with the gate fused, then the
    conditional residual pass to D8 (forced on), exactly as the bench launches them."""
    torch, fl = env
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2024)
    shapes = synth.qwen3_step_shapes()
    items, samples, keep = [], [], []
    for idx, (name, o, i) in enumerate(shapes):
        q, s = _int8_layer(torch, o, i, gen)
        st = torch.empty(fl.fl_plane_store_bytes(o, i), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(q, s, o, i, st)
        d4 = torch.full((o // 64,), 2, dtype=torch.uint8, device="cuda")
        d8 = torch.full((o // 64,), 4, dtype=torch.uint8, device="cuda")
        x = _x(torch, 1, i, gen)
        y = torch.empty((1, o), dtype=torch.float32, device="cuda")
        keep += [st, d4, d8, x, y]
        items.append((st, o, i, d4, d8, x, y))
        blocks = _sample_blocks(o // 64)
        rows = np.concatenate([np.arange(64 * b, 64 * b + 64) for b in blocks])
        samples.append((rows, q[rows].cpu().numpy(), s[rows].cpu().numpy(), x.cpu().numpy().view(np.uint16)))
        del q, s
    arr = fl.gemv_problems(items)
    n = len(items)
    wsb = fl.fl_gemv_gate_workspace_bytes(1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    e, m = torch.empty(1, device="cuda"), torch.empty(1, device="cuda")
    t2, es = torch.empty((1, 2), dtype=torch.int32, device="cuda"), torch.empty(1, dtype=torch.uint8, device="cuda")
    runs = torch.zeros(1, dtype=torch.int32, device="cuda")
    tau_h, tau_m = -1.0, -1.0                                     # always escalate
    spec = fl.gate_spec(n - 1, tau_h, tau_m, e, m, t2, es, ws, wsb)
    fl.fl_gemv_batched_gate(arr, n, 1, 0, spec)
    torch.cuda.synchronize()
    for level, label in ((2, "D4 pass"), (4, "escalated to D8")):
        if level == 4:
            fl.fl_gemv_batched_gate_if(arr, n, 1, 1, spec, es, runs)
            torch.cuda.synchronize()
            assert int(runs.item()) == 1
        for (rows, qs, ss, xs), it in zip(samples, items):
            lv = np.full(len(rows) // 64, level, np.uint8)
            yref, mass = orc.gemv_depth(qs, ss, lv, xs, with_mass=True)
            _check(it[6].cpu().numpy()[:, rows], yref, mass, f"{label}, {it[1]}x{it[2]}")
        z = items[-1][6].cpu().numpy()
        H, M, top2, esc = orc.logit_gate(z, tau_h, tau_m)
        assert np.array_equal(t2.cpu().numpy(), top2), label
        assert np.allclose(e.cpu().numpy(), H, rtol=1e-5, atol=1e-6), label
        assert np.allclose(m.cpu().numpy(), M, rtol=1e-5, atol=1e-7), label
        assert int(es.item()) == 1


@pytest.mark.parametrize("batch", [1, 8, 16, 32])
def test_large_single_layers_full_size(env, orc, batch):
    """The large-shape sweep at full size (uniform D6), single-layer calls with column splits."""
    torch, fl = env
    gen = torch.Generator(device="cuda")
    gen.manual_seed(3030 + batch)
    for (o, i) in ((14336, 4096), (4096, 14336), (4096, 4096)):
        q, s = _int8_layer(torch, o, i, gen)
        st = torch.empty(fl.fl_plane_store_bytes(o, i), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(q, s, o, i, st)
        lv = torch.full((o // 64,), 3, dtype=torch.uint8, device="cuda")
        x = _x(torch, batch, i, gen)
        y = torch.empty((batch, o), dtype=torch.float32, device="cuda")
        wsb = fl.fl_gemv_workspace_bytes(o, i, batch)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        fl.fl_gemv_depth(fl.plane_weight(st, o, i), lv, x, batch, y, ws, wsb)
        torch.cuda.synchronize()
        rows = np.concatenate([np.arange(64 * b, 64 * b + 64) for b in _sample_blocks(o // 64)])
        yref, mass = orc.gemv_depth(q[rows].cpu().numpy(), s[rows].cpu().numpy(),
                                    np.full(len(rows) // 64, 3, np.uint8), x.cpu().numpy().view(np.uint16),
                                    with_mass=True)
        _check(y.cpu().numpy()[:, rows], yref, mass, f"{i}->{o} batch {batch}")
        del q, s, st


def test_lens_stack_full_size(env, orc):
    """The lens-mapped stack: the level map over 14708 blocks (8 lenses), bit-exact, then the
    35 layers of [64 n_b, 2048] read at those levels in one batched launch."""
    torch, fl = env
    nb = 14708
    xy, cxy, r = synth.lens_inputs(nb, 8, 2, 1)
    stops = synth.even_stops(3, 1)
    p = fl.lens_params(0.3, 0.75, 1, 4, stops, 0)
    lev = torch.empty(nb, dtype=torch.uint8, device="cuda")
    cnt = torch.zeros(5, dtype=torch.int32, device="cuda")
    fl.fl_level_map(torch.from_numpy(xy).cuda(), nb, torch.from_numpy(cxy).cuda(),
                    torch.from_numpy(r).cuda(), 8, p, lev, cnt)
    torch.cuda.synchronize()
    ref = orc.level_map(xy, cxy, r, 0.3, 0.75, 1, 4, stops, 0)
    lv = lev.cpu().numpy()
    assert np.array_equal(lv, ref)
    assert np.array_equal(cnt.cpu().numpy(), np.bincount(ref, minlength=5))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5050)
    per = synth.lens_stack_layers(nb, 35)
    items, samples, keep, b0 = [], [], [], 0
    for l, n in enumerate(per):
        q, s = _int8_layer(torch, 64 * n, 2048, gen)
        st = torch.empty(fl.fl_plane_store_bytes(64 * n, 2048), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(q, s, 64 * n, 2048, st)
        x = _x(torch, 1, 2048, gen)
        y = torch.empty((1, 64 * n), dtype=torch.float32, device="cuda")
        keep += [st, x, y]
        items.append((st, 64 * n, 2048, lev[b0:b0 + n], None, x, y))
        blocks = _sample_blocks(n)
        rows = np.concatenate([np.arange(64 * b, 64 * b + 64) for b in blocks])
        samples.append((rows, q[rows].cpu().numpy(), s[rows].cpu().numpy(), lv[b0 + np.array(blocks)],
                        x.cpu().numpy().view(np.uint16)))
        b0 += n
    fl.fl_gemv_batched(fl.gemv_problems(items), len(items), 1, 0)
    torch.cuda.synchronize()
    for l, ((rows, qs, ss, lvs, xs), it) in enumerate(zip(samples, items)):
        yref, mass = orc.gemv_depth(qs, ss, lvs, xs, with_mass=True)
        _check(it[6].cpu().numpy()[:, rows], yref, mass, f"lens stack layer {l}")


def _kquant_tensor(torch, t, o, i, gen):
    """Random record bytes in the block-tiled order with finite fp16 d (and dmin) fields."""
    rec = 144 if t == synth.Q4_K else 210
    n = o * (i // 256)
    blk = torch.randint(0, 256, (n, rec), dtype=torch.uint8, device="cuda", generator=gen)
    d = (torch.rand((n, 2), device="cuda", generator=gen) * 1e-3 + 1e-4).to(torch.float16).view(torch.uint8)
    if t == synth.Q4_K:
        blk[:, 0:4] = d.view(n, 4)
    else:
        row = torch.arange(n, device="cuda") % 64                  # record order [block][sb][row]
        odd = (row % 2) == 1
        blk[~odd, 208:210] = d[~odd, 0:2]
        blk[odd, 0:2] = d[odd, 0:2]
    return blk.view(-1)


def test_kquant_step_full_size(env, orc):
    """The Llama-3.2-1B-shaped K-quant step: 113 tensors in one batched launch."""
    torch, fl = env
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4040)
    items, samples, keep = [], [], []
    for name, o, i, t in synth.llama32_kquant_mix():
        blk = _kquant_tensor(torch, t, o, i, gen)
        x = _x(torch, 1, i, gen)
        y = torch.empty((1, o), dtype=torch.float32, device="cuda")
        keep += [blk, x, y]
        items.append((blk, t, o, i, x, y))
        per_block = 64 * (i // 256) * (144 if t == synth.Q4_K else 210)
        for b in _sample_blocks(o // 64):
            samples.append((len(items) - 1, b, blk[b * per_block:(b + 1) * per_block].cpu().numpy()))
    arr = fl.kquant_problems(items)
    fl.fl_gemv_kquant_batched(arr, len(items), 1)
    torch.cuda.synchronize()
    ys = {}
    for k, b, recs in samples:
        blk, t, o, i, x, y = items[k]
        if k not in ys:
            ys[k] = y.cpu().numpy()
        yref, mass = orc.gemv_kquant(recs, t, 64, i, x.cpu().numpy().view(np.uint16), with_mass=True)
        _check(ys[k][:, 64 * b:64 * b + 64], yref, mass, f"K-quant type {t} {o}x{i} block {b}")


def test_in_pass_decision_full_size(env, orc):
    """The decode step read at D4, the in-pass decision over all 197 layers' 7,750 blocks in
    one call (checked on every block), then the listed residual pass from D4 over the lifted
    blocks (checked on sampled and on lifted blocks; the others must keep their D4 value)."""
    torch, fl = env
    import test_gpu_decide as dec
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6060)
    items, qs, ss, keep = [], [], [], []
    for name, o, i in synth.qwen3_step_shapes():
        q, s = _int8_layer(torch, o, i, gen)
        s.mul_(torch.rand((o // 64, 1), device="cuda", generator=gen).mul_(3.75).add_(0.25).repeat_interleave(64, 0))
        st = torch.empty(fl.fl_plane_store_bytes(o, i), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(q, s, o, i, st)
        lv = torch.full((o // 64,), 2, dtype=torch.uint8, device="cuda")
        x = _x(torch, 1, i, gen)
        y = torch.empty((1, o), dtype=torch.float32, device="cuda")
        keep += [st, lv, x, y]
        items.append((st, o, i, lv, None, x, y))
        qs.append(q)
        ss.append(s.cpu().numpy())
    n = len(items)
    fl.fl_gemv_batched(fl.gemv_problems(items), n, 1, 0)
    torch.cuda.synchronize()
    ys = [it[6].cpu().numpy() for it in items]
    to = [torch.empty(it[1] // 64, dtype=torch.uint8, device="cuda") for it in items]
    sc = [torch.empty(it[1] // 64, dtype=torch.float32, device="cuda") for it in items]
    up = [torch.empty(it[1] // 64, dtype=torch.int32, device="cuda") for it in items]
    probs = fl.decide_problems([(it[0], it[1], it[2], it[6], t, c, u) for it, t, c, u in zip(items, to, sc, up)])
    allr = np.concatenate([orc.level_decide(y, s, 2, 4, 0, lam=1.0)[1] for y, s in zip(ys, ss)])
    lam = float(np.quantile(allr, 0.84)) / 16
    for rule, f in ((fl.FL_DECIDE_LADDER, 0.0), (fl.FL_DECIDE_SHARE, 0.16)):
        fl.fl_level_decide(probs, n, 1, fl.decide_params(rule, 2, 4, lam, f))
        torch.cuda.synchronize()
        for k, (y, s, t, c) in enumerate(zip(ys, ss, to, sc)):
            ref_lev, ref_red = orc.level_decide(y, s, 2, 4, rule, lam=lam, f=np.float32(f))
            lev, score = t.cpu().numpy(), c.cpu().numpy()
            if rule == fl.FL_DECIDE_LADDER:
                dec.check_ladder(lev, score, ref_lev, ref_red, 2, 4, lam, f"step ladder, problem {k}")
            else:
                dec.check_share(lev, score, ref_lev, ref_red, 2, 4, f, f"step share, problem {k}")
    # the residual over the lifted blocks only, as the bench runs it
    res = [(it[0], it[1], it[2], it[3], t, it[5], it[6]) for it, t in zip(items, to)]
    counts = [int(np.floor(np.float64(np.float32(0.16)) * (it[1] // 64))) for it in items]
    for k, (t, u, c) in enumerate(zip(to, up, counts)):
        assert np.array_equal(u.cpu().numpy()[:c], np.flatnonzero(t.cpu().numpy() > 2)), k
    fl.fl_gemv_batched_listed(fl.gemv_problems(res), *fl.block_lists(up, counts), n, 1, 1)
    torch.cuda.synchronize()
    lifted = 0
    for k, (it, t, q, s) in enumerate(zip(items, to, qs, ss)):
        lev = t.cpu().numpy()
        up = np.flatnonzero(lev > 2)
        lifted += len(up)
        blocks = sorted(set(_sample_blocks(len(lev))) | set(up[:2].tolist()))
        rows = np.concatenate([np.arange(64 * b, 64 * b + 64) for b in blocks])
        yref, mass = orc.gemv_depth(q[rows].cpu().numpy(), s[rows], lev[blocks], it[5].cpu().numpy().view(np.uint16),
                                    with_mass=True)
        yk = it[6].cpu().numpy()
        _check(yk[:, rows], yref, mass, f"in-pass step, problem {k}")
        keep_rows = np.repeat(lev <= 2, 64)
        assert np.array_equal(yk[:, keep_rows], ys[k][:, keep_rows]), f"unlifted rows changed, problem {k}"
    assert lifted == sum(int(np.floor(np.float64(np.float32(0.16)) * (it[1] // 64))) for it in items)
