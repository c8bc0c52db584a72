"""Verified speculation on the GPU vs the oracle, through the C-ABI: the acceptance kernel on
every mismatch pattern, and a whole window (k gated D4 draft passes, one gated residual pass
at batch k, acceptance) against the oracle's depth GEMVs and greedy acceptance."""
import itertools

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


def test_accept_kernel_every_pattern(env, orc):
    torch, fl = env
    totals = torch.zeros(2, dtype=torch.int32, device="cuda")
    res = torch.empty(2, dtype=torch.int32, device="cuda")
    want_tot = np.zeros(2, np.int64)
    cases = []
    for k in range(1, 7):
        cases += [(k, bits) for bits in itertools.product((0, 1), repeat=k)]
    g = np.random.default_rng(5)
    cases += [(16, tuple(g.integers(0, 2, 16))) for _ in range(20)] + [(16, (0,) * 16), (16, (0,) * 15 + (1,))]
    for k, bits in cases:
        ver = np.stack([np.arange(k) * 7 + 1, np.arange(k) * 3], axis=1).astype(np.int32)
        dr = ver.copy()
        dr[:, 0] += np.array(bits, np.int32)              # a 1 bit makes that step's draft disagree
        dr[:, 1] = 99                                      # the second column is not compared
        fl.fl_spec_accept(dev(torch, dr), dev(torch, ver), k, res, totals)
        torch.cuda.synchronize()
        a, e = orc.spec_accept(dr[:, 0], ver[:, 0])
        assert res.cpu().numpy().tolist() == [a, e], (k, bits)
        want_tot += (a, e)
    assert totals.cpu().numpy().tolist() == want_tot.tolist()


@pytest.mark.parametrize("K", [4, 8])
def test_spec_window_vs_oracle(env, orc, K):
    torch, fl = env
    shapes = [(1024, 1024), (2048, 1024), (4096, 1024)]      # the last is the logits
    gi = len(shapes) - 1
    layers, stores, keep = [], [], []
    for i, (o, n) in enumerate(shapes):
        q, s = synth.int8_layer(o, n, 500 + K, i)
        x = synth.bf16_normal((K, n), 501 + K, i)
        st = torch.empty(fl.fl_plane_store_bytes(o, n), dtype=torch.uint8, device="cuda")
        fl.fl_pack_planes(dev(torch, q), dev(torch, s), o, n, st)
        layers.append((q, s, x))
        stores.append((st, dev(torch, x), torch.empty((K, o), dtype=torch.float32, device="cuda"),
                       torch.full((o // 64,), 2, dtype=torch.uint8, device="cuda"),
                       torch.full((o // 64,), 4, dtype=torch.uint8, device="cuda")))
    keep.append(stores)
    wsb = fl.fl_gemv_gate_workspace_bytes(K)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    ent = torch.empty(K, dtype=torch.float32, device="cuda")
    mar = torch.empty(K, dtype=torch.float32, device="cuda")
    esc = torch.empty(K, dtype=torch.uint8, device="cuda")
    dtop = torch.empty((K, 2), dtype=torch.int32, device="cuda")
    vtop = torch.empty((K, 2), dtype=torch.int32, device="cuda")
    # drafts: one gated D4 pass per step, batch 1, writing row t of every y
    for t in range(K):
        items = [(st, o, n, d4, None, x[t], y[t]) for (st, x, y, d4, d8), (o, n) in zip(stores, shapes)]
        spec = fl.gate_spec(gi, 0.0, 0.0, ent[t:t + 1], mar[t:t + 1], dtop[t], esc[t:t + 1], ws, wsb)
        fl.fl_gemv_batched_gate(fl.gemv_problems(items), len(items), 1, 0, spec)
    torch.cuda.synchronize()
    y4 = [y.cpu().numpy() for (st, x, y, d4, d8) in stores]
    # verification: one gated residual pass at batch K over the window
    items = [(st, o, n, d4, d8, x, y) for (st, x, y, d4, d8), (o, n) in zip(stores, shapes)]
    spec = fl.gate_spec(gi, 0.0, 0.0, ent, mar, vtop, esc, ws, wsb)
    fl.fl_gemv_batched_gate(fl.gemv_problems(items), len(items), K, 1, spec)
    res = torch.empty(2, dtype=torch.int32, device="cuda")
    fl.fl_spec_accept(dtop, vtop, K, res)
    torch.cuda.synchronize()
    y8 = [y.cpu().numpy() for (st, x, y, d4, d8) in stores]
    for i, ((q, s, x), (o, n)) in enumerate(zip(layers, shapes)):
        for lev, yg in ((2, y4[i]), (4, y8[i])):
            yref, mass = orc.gemv_depth(q, s, np.full(o // 64, lev, np.uint8), x, with_mass=True)
            assert np.all(np.abs(yg - yref) <= REL * mass + ABS), (K, i, lev)
    d_tok, v_tok = dtop.cpu().numpy(), vtop.cpu().numpy()
    assert np.array_equal(d_tok, orc.logit_gate(y4[gi], 0.0, 0.0)[2])
    assert np.array_equal(v_tok, orc.logit_gate(y8[gi], 0.0, 0.0)[2])
    a, e = orc.spec_accept(d_tok[:, 0], v_tok[:, 0])
    assert res.cpu().numpy().tolist() == [a, e]
    # zero KL against the exact D8 model: the emitted tokens are its argmax tokens, except
    # where its two best logits are closer than the product's tolerance
    q, s, x = layers[gi]
    yref, mass = orc.gemv_depth(q, s, np.full(shapes[gi][0] // 64, 4, np.uint8), x, with_mass=True)
    for t in range(e):
        top = np.argsort(-yref[t])[:2]
        close = yref[t, top[0]] - yref[t, top[1]] <= 2 * (REL * mass[t, top].max() + ABS)
        assert close or v_tok[t, 0] == top[0], (K, t)
