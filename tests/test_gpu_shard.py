"""The read split over ranks, on one GPU, against the CPU oracle through the C-ABI.

Ranks are emulated in one process (their kernels do not wait on one another): each "rank"
reads its block ranges of every layer with fl_gemv_batched on pointer offsets into the plane
store, and the assembled outputs must equal the oracle's at the path's bar; the logits are cut
into pieces, each piece reduced to a partial with fl_logit_gate_partial, and the partials
merged with fl_logit_gate_merge must give the oracle's gate of the whole row (top-2 exact,
entropy and margin within 1e-5 relative, decisions equal outside the band fp32 rounding may
flip).
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
    from variable_precision_weight_b200 import fl, shard
    return torch, fl, shard


def dev(torch, a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


@pytest.mark.parametrize("vocab,batch", [(151936, 1), (151936, 3), (4100, 2)])
@pytest.mark.parametrize("nparts", [1, 2, 3, 8])
def test_gate_partials_merge_to_the_whole_row(env, orc, vocab, batch, nparts):
    torch, fl, shard = env
    z = synth.rng(70, vocab, batch).standard_normal((batch, vocab)).astype(np.float32)
    z[:, vocab // 3] = z[:, vocab // 3 + 1] = z.max() + 1.0            # a tie across the top two
    cut = [vocab * r // nparts // 4 * 4 for r in range(nparts)] + [vocab]
    parts = torch.empty((nparts, batch * fl.GATE_PARTIAL_BYTES), dtype=torch.uint8, device="cuda")
    for r in range(nparts):
        piece = dev(torch, z[:, cut[r]:cut[r + 1]])
        fl.fl_logit_gate_partial(piece, cut[r + 1] - cut[r], batch, cut[r], parts[r])
    H0, M0, t0, _ = orc.logit_gate(z, 1e30, -1.0)
    tau_h, tau_m = float(np.median(H0)), float(np.median(M0))
    ent = torch.empty(batch, device="cuda")
    mar = torch.empty(batch, device="cuda")
    top2 = torch.empty((batch, 2), dtype=torch.int32, device="cuda")
    esc = torch.empty(batch, dtype=torch.uint8, device="cuda")
    fl.fl_logit_gate_merge(parts, nparts, batch, tau_h, tau_m, ent, mar, top2, esc)
    torch.cuda.synchronize()
    H, M, t2, e = orc.logit_gate(z, tau_h, tau_m)
    assert np.array_equal(top2.cpu().numpy(), t2)
    assert np.allclose(ent.cpu().numpy(), H, rtol=1e-5, atol=0)
    assert np.allclose(mar.cpu().numpy(), M, rtol=1e-5, atol=1e-7)
    band = (np.abs(H - tau_h) <= 1e-4 * abs(tau_h)) | (np.abs(M - tau_m) <= 1e-6)
    assert np.array_equal(esc.cpu().numpy()[~band], e[~band])
    # the same as the gate of the whole row in one launch
    ent1, mar1 = torch.empty_like(ent), torch.empty_like(mar)
    top1, esc1 = torch.empty_like(top2), torch.empty_like(esc)
    fl.fl_logit_gate(dev(torch, z), vocab, batch, tau_h, tau_m, ent1, mar1, top1, esc1)
    torch.cuda.synchronize()
    assert np.array_equal(top1.cpu().numpy(), top2.cpu().numpy())
    assert np.allclose(ent1.cpu().numpy(), ent.cpu().numpy(), rtol=1e-5)


@pytest.mark.parametrize("nranks", [2, 3, 5])
@pytest.mark.parametrize("mode", [0, 1])
def test_sharded_read_assembles_to_the_whole_layers(env, orc, nranks, mode):
    torch, fl, shard = env
    batch = 2
    shapes = [(1216, 512), (448, 1664), (3072, 1024)]
    layers, host, lt_dev, lt_host = [], [], [], []
    for li, (out, inn) in enumerate(shapes):
        q, s = synth.int8_layer(out, inn, 71, li)
        lv = synth.seeded_levels(out // 64, 72, li, low=1 if mode else 0)
        lt = np.maximum(lv, synth.seeded_levels(out // 64, 73, li))
        x = synth.bf16_normal((batch, inn), 74, li)
        store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(dev(torch, q), dev(torch, s), out, inn, store)
        layers.append((store, out, inn, dev(torch, lv), dev(torch, x)))
        lt_dev.append(dev(torch, lt))
        host.append((q, s, lv, x))
        lt_host.append(lt)
    plans = shard.plan([h[2] for h in host], [inn for _, inn in shapes], nranks)
    y_full = [np.zeros((batch, out), np.float32) for out, _ in shapes]
    y0 = [synth.rng(75, li).standard_normal((batch, out)).astype(np.float32) for li, (out, _) in enumerate(shapes)]
    for rank in range(nranks):
        rows, total = shard.rank_rows(plans, rank)
        y_local = torch.zeros(max(batch * total, 1), dtype=torch.float32, device="cuda")
        if mode == 1:  # the residual adds to what the rows hold
            off = 0
            for li, r0, n in rows:
                y_local[off:off + batch * n] = dev(torch, y0[li][:, r0:r0 + n].reshape(-1))
                off += batch * n
        items, placed = shard.local_items(layers, plans, rank, y_local, batch, lt_dev if mode else None)
        if items:
            fl.fl_gemv_batched(fl.gemv_problems(items), len(items), batch, mode)
        torch.cuda.synchronize()
        yl = y_local.cpu().numpy()
        for (li, off, n), (lj, r0, nn) in zip(placed, [r for r in rows if r[2] > 0]):
            assert li == lj and n == nn
            y_full[li][:, r0:r0 + n] = yl[off:off + batch * n].reshape(batch, n)
    for li, (q, s, lv, x) in enumerate(host):
        if mode == 0:
            yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
        else:
            d, mass = orc.gemv_residual(q, s, lv, lt_host[li], x, with_mass=True)
            yref = y0[li].astype(np.float64) + d
        err = np.abs(y_full[li].astype(np.float64) - yref)
        assert np.all(err <= REL * mass + ABS), (li, float((err / (REL * mass + ABS)).max()))
    fl.fl_device_status()


@pytest.mark.parametrize("nparts", [1, 3])
def test_fused_gate_partials_merge_to_the_whole_row(env, orc, nparts):
    """The head's logits split into row pieces, each piece its own batched pass with the gate
    fused in partial mode (the rank's share of the vocabulary reduced in the launch that
    computes it); the merged partials equal the oracle's gate of the whole row, and the pieces'
    outputs the oracle's product."""
    torch, fl, shard = env
    out, inn = 64 * 47, 512
    q, s = synth.int8_layer(out, inn, 80)
    lv = np.full(out // 64, 2, np.uint8)
    x = synth.bf16_normal((1, inn), 81)
    store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
    fl.fl_pack_planes(dev(torch, q), dev(torch, s), out, inn, store)
    lvd, xd = dev(torch, lv), dev(torch, x)
    first = fl.fl_shard_blocks(lv, inn, nparts)
    y = torch.zeros((1, out), dtype=torch.float32, device="cuda")
    parts = torch.zeros((nparts, fl.GATE_PARTIAL_BYTES), dtype=torch.uint8, device="cuda")
    wsb = fl.fl_gemv_gate_workspace_bytes(1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    spec = fl.gate_spec(0, 0.0, 0.0, None, None, None, None, ws, wsb)
    for r in range(nparts):
        b0, b1 = first[r], first[r + 1]
        if b1 == b0:
            continue
        item = (store[b0 * 8448 * (inn // 128):], 64 * (b1 - b0), inn, lvd[b0:], None, xd, y[0, 64 * b0:64 * b1])
        fl.fl_gemv_batched_gate_partial(fl.gemv_problems([item]), 1, 1, 0, spec, None, None, 64 * b0, parts[r])
    yref, mass = orc.gemv_depth(q, s, lv, x, with_mass=True)
    H0, M0, _, _ = orc.logit_gate(yref.astype(np.float32), 1e30, -1.0)
    tau_h, tau_m = float(H0[0]), float(M0[0]) / 2
    ent, mar = torch.empty(1, device="cuda"), torch.empty(1, device="cuda")
    top2, esc = torch.empty((1, 2), dtype=torch.int32, device="cuda"), torch.empty(1, dtype=torch.uint8, device="cuda")
    fl.fl_logit_gate_merge(parts, nparts, 1, tau_h, tau_m, ent, mar, top2, esc)
    torch.cuda.synchronize()
    yg = y.cpu().numpy()
    assert np.all(np.abs(yg.astype(np.float64) - yref) <= REL * mass + ABS)
    H, M, t2, _ = orc.logit_gate(yg, tau_h, tau_m)       # the gate of the outputs the passes wrote
    assert np.array_equal(top2.cpu().numpy(), t2)
    assert np.allclose(ent.cpu().numpy(), H, rtol=1e-5, atol=0)
    assert np.allclose(mar.cpu().numpy(), M, rtol=1e-5, atol=1e-7)
    fl.fl_device_status()
