"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth used here: hand-worked values written out in tests/golden
(each with its derivation and page citation), closed forms, independent
formulations (a numpy restatement from different algebra, or a library
routine), invariants the pages state, and brute force on tiny inputs.
"""
import math

import numpy as np
import pytest
from scipy.special import entr, softmax

from variable_precision_weight_b200 import synth

DEPTHS = (0, 2, 4, 6, 8)


# ----------------------------------------------------------------------------- quantizer

def test_quantizer_two_implementations_agree(orc):
    w = synth.gaussian_weights(256, 512, 7, 1)
    w[3, 128:256] = 0.0                        # an all-zero group
    w[5, 0] = 0.5                              # a dominant element
    q1, s1 = synth.quantize_int8(w)
    q2, s2 = orc.quantize_int8(w)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_quantizer_invariants(orc):
    w = synth.gaussian_weights(128, 1024, 7, 2)
    w[0, :128] = 0.0
    q, s = orc.quantize_int8(w)
    assert np.all(q[0, :128] == 0) and s[0, 0] == 0.0
    wg = w.reshape(128, 8, 128)
    qg = q.reshape(128, 8, 128).astype(np.int64)
    amax_idx = np.abs(wg).argmax(axis=2)
    top = np.take_along_axis(qg, amax_idx[..., None], axis=2)[..., 0]
    nz = s > 0
    assert np.all(np.abs(top[nz]) == 127)                      # absmax maps to +-127
    err = np.abs(wg - s[..., None] * qg)
    assert np.all(err <= s[..., None] * 0.5 * (1 + 1e-6) + 1e-12)   # round to nearest
    assert q.min() >= -127 and q.max() <= 127


# ----------------------------------------------------------------------------- depth reconstruction

def test_depth_values_hand_worked(orc, golden):
    g = golden("depth_reconstruction.json")
    for case in g["cases"]:
        for d, v in case["w_over_s"].items():
            assert orc.dequant_depth(case["q"], 1.0, int(d)) == v, (case["q"], d)
            assert orc.dequant_depth(case["q"], 0.25, int(d)) == 0.25 * v


def test_d8_equals_int8_dequant(orc):
    for q in range(-127, 128):
        for s in (0.0, 1e-3, 0.0173, 3.0):
            assert orc.dequant_depth(q, s, 8) == float(np.float32(s)) * q


def test_depth_error_bound_all_codes_and_random_weights(orc):
    # |w - w_d| <= s 2^(7-d): worst case over all codes is s (2^(7-d) - 1/2) from truncation,
    # plus at most s/2 from the int8 rounding of w.
    for d in (2, 4, 6, 8):
        errs = [abs(q - orc.dequant_depth(q, 1.0, d)) for q in range(-127, 128)]
        assert max(errs) == 2.0 ** (7 - d) - 0.5
    w = synth.gaussian_weights(64, 1024, 7, 3)
    q, s = synth.quantize_int8(w)
    for d in (2, 4, 6, 8):
        for r in range(0, 64, 7):
            for c in range(0, 1024, 37):
                sc = float(s[r, c // 128])
                assert abs(w[r, c] - orc.dequant_depth(int(q[r, c]), sc, d)) <= sc * 2.0 ** (7 - d) * (1 + 1e-6)


def _independent_depth_gemv(q, s, levels, xf):
    """numpy restatement through the top-d-bit integer U_d = u >> (8-d) and group sums:
    y = sum_g s[r,g] (2^(8-d) sum_c U_d x_c + (c_d - 128) sum_c x_c)."""
    out, inn = q.shape
    u = q.astype(np.int64) + 128
    y = np.zeros((xf.shape[0], out))
    G = inn // 128
    xg = xf.reshape(xf.shape[0], G, 128)
    X = xg.sum(axis=2)                                   # [batch, G]
    for b, lev in enumerate(levels):
        d = 2 * int(lev)
        rows = slice(64 * b, 64 * b + 64)
        if d == 0:
            continue
        U = (u[rows] >> (8 - d)).reshape(64, G, 128).astype(np.float64)
        cd = (2.0 ** (8 - d) - 1) / 2
        part = 2.0 ** (8 - d) * np.einsum("rgc,tgc->trg", U, xg) + (cd - 128.0) * X[:, None, :]
        y[:, rows] = np.einsum("trg,rg->tr", part, s[rows].astype(np.float64))
    return y


def test_gemv_depth_independent_formulation(orc):
    q, s = synth.int8_layer(320, 1024, 7, 4)
    levels = np.array([0, 1, 2, 3, 4], np.uint8)
    x = synth.bf16_normal((3, 1024), 7, 5)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y = orc.gemv_depth(q, s, levels, x)
    y2 = _independent_depth_gemv(q, s, levels, xf)
    assert np.allclose(y, y2, rtol=1e-12, atol=1e-12)
    assert np.all(y[:, :64] == 0.0)                      # ZERO block contributes nothing


def test_gemv_d8_is_plain_dequant_matmul(orc):
    q, s = synth.int8_layer(128, 512, 7, 6)
    x = synth.bf16_normal((2, 512), 7, 7)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    W = np.repeat(s.astype(np.float64), 128, axis=1) * q.astype(np.float64)
    y = orc.gemv_depth(q, s, np.full(2, 4, np.uint8), x)
    assert np.allclose(y, xf @ W.T, rtol=1e-12, atol=1e-12)


def test_zero_block_isolated(orc):
    q, s = synth.int8_layer(192, 256, 7, 8)
    x = synth.bf16_normal((1, 256), 7, 9)
    a = orc.gemv_depth(q, s, np.array([2, 0, 3], np.uint8), x)
    b = orc.gemv_depth(q, s, np.array([2, 4, 3], np.uint8), x)
    assert np.all(a[:, 64:128] == 0.0)
    assert np.array_equal(a[:, :64], b[:, :64]) and np.array_equal(a[:, 128:], b[:, 128:])


def test_residual_identity_d4_to_d8(orc):
    q, s = synth.int8_layer(256, 1024, 7, 10)
    x = synth.bf16_normal((4, 1024), 7, 11)
    lv = lambda v: np.full(4, v, np.uint8)
    y4 = orc.gemv_depth(q, s, lv(2), x)
    y8 = orc.gemv_depth(q, s, lv(4), x)
    res = orc.gemv_residual(q, s, lv(2), lv(4), x)
    assert np.allclose(y4 + res, y8, rtol=1e-12, atol=1e-10)
    assert np.all(orc.gemv_residual(q, s, lv(3), lv(3), x) == 0.0)
    assert np.allclose(orc.gemv_residual(q, s, lv(0), lv(3), x), orc.gemv_depth(q, s, lv(3), x), rtol=1e-12)
    # mixed per-block ranges
    a = np.array([0, 1, 2, 3], np.uint8)
    b = np.array([4, 3, 2, 4], np.uint8)
    ya, yb = orc.gemv_depth(q, s, a, x), orc.gemv_depth(q, s, b, x)
    assert np.allclose(ya + orc.gemv_residual(q, s, a, b, x), yb, rtol=1e-12, atol=1e-10)


# ----------------------------------------------------------------------------- plane store

def test_pack_unpack_bijection_all_codes(orc):
    codes = (np.arange(64 * 256) % 256 - 128).astype(np.int8).reshape(64, 256)
    rng = np.random.default_rng(0)
    s = rng.random((64, 2), dtype=np.float32)
    st = orc.pack_planes(codes, s)
    assert st.size == orc.store_bytes(64, 256) == 2 * 8448
    q2, s2 = orc.unpack_planes(st, 64, 256)
    assert np.array_equal(q2, codes) and np.array_equal(s2, s)


def test_pack_hand_worked_bytes(orc, golden):
    g = golden("plane_store_bytes.json")
    q = np.full((64, 128), -128, np.int8)
    for c, v in zip(g["codes"]["cols"], g["codes"]["q"]):
        q[g["codes"]["row"], c] = v
    s = np.zeros((64, 1), np.float32)
    s[g["scale"]["row"], 0] = g["scale"]["value"]
    st = orc.pack_planes(q, s)
    expect = np.zeros(g["store_bytes"], np.uint8)
    for off, val in g["nonzero_bytes"]:
        expect[off] = val
    assert np.array_equal(st, expect)


def test_store_prefix_is_depth_read(orc):
    # A block read at depth d is the contiguous prefix: scales + planes 0..d/2-1.
    q, s = synth.int8_layer(64, 256, 7, 12)
    st = orc.pack_planes(q, s)
    G = 2
    u = q.astype(np.int64) + 128
    for d in (2, 4, 6, 8):
        pre = st[: 256 * G + 1024 * G * d]
        tail = np.zeros(st.size - pre.size, np.uint8)
        q2, s2 = orc.unpack_planes(np.concatenate([pre, tail]), 64, 256)
        ud = (u >> (8 - d)) << (8 - d)
        assert np.array_equal(q2.astype(np.int64) + 128, ud) and np.array_equal(s2, s)


def test_store_words_give_code_bytes_after_rotation(orc):
    # Property the layout is built for: OR the masked plane-k words of one 16-column word
    # (mask = 0x03030303 rotated left by (6 - 2k + 2i) mod 32), rotate right by 2i, and byte
    # lane L holds the top-d-bit code u_d of column 4i + L.
    q, s = synth.int8_layer(64, 128, 7, 13)
    st = orc.pack_planes(q, s)
    u = q.astype(np.int64) + 128
    rotl = lambda v, n: ((v << n) | (v >> (32 - n))) & 0xFFFFFFFF if n % 32 else v
    rotr = lambda v, n: rotl(v, (32 - n) % 32)
    for r in (0, 17, 63):
        for w in range(8):
            words = [int.from_bytes(bytes(st[256 + 2048 * k + 32 * r + 4 * w: 256 + 2048 * k + 32 * r + 4 * w + 4]),
                                    "little") for k in range(4)]
            for d in (2, 4, 6, 8):
                for i in range(4):
                    acc = 0
                    for k in range(d // 2):
                        acc |= words[k] & rotl(0x03030303, (6 - 2 * k + 2 * i) % 32)
                    acc = rotr(acc, 2 * i)
                    for L in range(4):
                        col = 16 * w + 4 * i + L
                        assert (acc >> (8 * L)) & 0xFF == (u[r, col] >> (8 - d)) << (8 - d)


# ----------------------------------------------------------------------------- lens rule

def test_lens_kappa(orc):
    assert orc.lens_kappa(0.75, 1, 4) == 3        # config with glass D2
    assert orc.lens_kappa(0.75, 3, 4) == 3        # glass D6: floor(0.75) = 0 -> no rings
    assert orc.lens_kappa(1.0, 3, 4) == 4
    assert orc.lens_kappa(0.0, 1, 4) == 1
    assert orc.lens_kappa(1.0, 0, 4) == 4


def test_lens_hand_worked(orc, golden):
    g = golden("lens_hand_maps.json")
    p = g["params"]
    one = g["single_lens"]
    lev = orc.level_map(np.array(one["blocks"]), np.array([one["center"]]), np.array([one["r"]]),
                        p["f"], p["g"], p["gamma"], p["m"], p["stops"], 0)
    assert lev.tolist() == one["levels_sum"]
    two = g["two_lenses"]
    args = (np.array(two["blocks"]), np.array(two["centers"]), np.array(two["r"]), p["f"], p["g"], p["gamma"],
            p["m"], p["stops"])
    assert orc.level_map(*args, 0).tolist() == two["levels_sum"]
    assert orc.level_map(*args, 1).tolist() == two["levels_max"]


def test_lens_degenerate_cases(orc):
    xy, cxy, r = synth.lens_inputs(2000, 8, 7, 14)
    stops = synth.even_stops(3, 1)
    # g = 0: kappa = gamma, every block at the glass
    assert np.all(orc.level_map(xy, cxy, r, 0.3, 0.0, 1, 4, [], 0) == 1)
    # f = 0: R = 0, nothing lifts except a block exactly on a centre
    xy2 = np.concatenate([xy, cxy[:1]])
    lev = orc.level_map(xy2, cxy, r, 0.0, 0.75, 1, 4, stops, 0)
    assert np.all(lev[:-1] == 1) and lev[-1] == 3
    # no lens: glass everywhere
    assert np.all(orc.level_map(xy, cxy[:0], r[:0], 0.3, 0.75, 1, 4, stops, 0) == 1)
    # blocks on a centre reach the ceiling
    lev = orc.level_map(cxy, cxy, r, 0.3, 1.0, 0, 4, synth.even_stops(4, 0), 0)
    assert np.all(lev == 4)
    # sum-clamp never lowers a level relative to max
    a = orc.level_map(xy, cxy * 0.3 + 0.35, r * 4, 0.3, 0.75, 1, 4, stops, 0)
    b = orc.level_map(xy, cxy * 0.3 + 0.35, r * 4, 0.3, 0.75, 1, 4, stops, 1)
    assert np.all(a >= b) and np.any(a > b)


def test_lens_matches_double_evaluation_off_ring_edges(orc):
    """fp32 oracle vs a float64 numpy evaluation of the same rule; they agree except where
    rho* is within 1e-5 (relative) of a stop."""
    xy, cxy, r = synth.lens_inputs(20000, 8, 7, 15)
    cxy = cxy * 0.5 + 0.25
    r = r * 3
    for combine in (0, 1):
        for (f, g, gamma) in ((0.3, 0.75, 1), (0.5, 1.0, 0), (0.2, 0.5, 2)):
            kappa = gamma + math.floor(g * (4 - gamma))
            stops = synth.even_stops(kappa, gamma)
            lev = orc.level_map(xy, cxy, r, f, g, gamma, 4, stops, combine)
            R = r.astype(np.float64) * f / (1 - f)
            dist = np.sqrt(((xy[:, None, :].astype(np.float64) - cxy[None, :, :]) ** 2).sum(-1))
            s_last = float(stops[-1])
            Li = np.maximum(0.0, 1.0 - dist / R[None, :] / s_last)
            L = np.minimum(1.0, Li.sum(1)) if combine == 0 else Li.max(1)
            rho = s_last * (1.0 - L)
            ref = gamma + (rho[:, None] < stops[None, :].astype(np.float64)).sum(1)
            near = (np.abs(rho[:, None] - stops[None, :]) <= 1e-5 * stops[None, :]).any(1) & (L > 0)
            assert np.array_equal(lev[~near], ref[~near])
            assert near.sum() < 5 and (lev > gamma).sum() > 100


def test_memory_bits(orc):
    bits = np.array([0, 2, 4, 6, 8], np.float64)
    for l in range(5):
        assert orc.memory_bits(np.full(10, l, np.uint8), np.ones(10), bits) == 2 * l
    lev = np.array([0, 1, 4, 4], np.uint8)
    wb = np.array([64 * 1024, 64 * 1024, 64 * 2048, 64 * 1024], np.float64)
    # (0 + 2 + 8*2 + 8) / 5 = 26/5
    assert orc.memory_bits(lev, wb, bits) == pytest.approx(26 / 5, rel=1e-15)


# ----------------------------------------------------------------------------- gate

def test_gate_constant_logits(orc):
    V = 151936
    H, M, top2, esc = orc.logit_gate(np.full((1, V), 0.25, np.float32), 11.0, 0.1)
    assert H[0] == pytest.approx(math.log(V), abs=1e-9)
    assert M[0] == 0.0 and top2[0].tolist() == [0, 1] and esc[0] == 1


def test_gate_one_hot(orc):
    z = np.zeros((1, 1000), np.float32)
    z[0, 417] = 200.0
    H, M, top2, esc = orc.logit_gate(z, 1.0, 0.5)
    assert H[0] < 1e-80 and M[0] == 1.0 and top2[0].tolist() == [417, 0] and esc[0] == 0


def test_gate_two_level_closed_form(orc):
    V, k, a = 5000, 7, 3.0
    z = np.zeros((1, V), np.float32)
    z[0, 100:100 + k] = a
    Z = k * math.exp(a) + (V - k)
    H_ref = math.log(Z) - k * a * math.exp(a) / Z
    H, M, top2, _ = orc.logit_gate(z, 0, 0)
    assert H[0] == pytest.approx(H_ref, rel=1e-12)
    assert M[0] == 0.0 and top2[0].tolist() == [100, 101]


def test_gate_random_vs_scipy(orc):
    z = synth.rng(7, 16).standard_normal((4, 151936), dtype=np.float32) * np.float32(2.0)
    H, M, top2, esc = orc.logit_gate(z, 11.5, 1e-3)
    p = softmax(z.astype(np.float64), axis=1)
    Href = entr(p).sum(1)
    assert np.allclose(H, Href, rtol=1e-10)
    srt = np.argsort(-z, axis=1, kind="stable")
    assert np.array_equal(top2, srt[:, :2])
    p1 = np.take_along_axis(p, srt[:, :1], 1)[:, 0]
    p2 = np.take_along_axis(p, srt[:, 1:2], 1)[:, 0]
    assert np.allclose(M, p1 - p2, rtol=1e-9, atol=1e-15)
    assert np.array_equal(esc, ((Href > 11.5) | (p1 - p2 < 1e-3)).astype(np.uint8))


def test_gate_tie_goes_to_lower_index(orc):
    z = np.zeros((1, 64), np.float32)
    z[0, 9] = 5.0
    z[0, 5] = 5.0
    z[0, 30] = 5.0
    H, M, top2, _ = orc.logit_gate(z, 0, 0)
    assert top2[0].tolist() == [5, 9] and M[0] == 0.0


# ----------------------------------------------------------------------------- K-quant

def _record(pairs, n):
    rec = np.zeros(n, np.uint8)
    for off, val in pairs:
        rec[off] = val
    return rec


def test_kquant_hand_built_superblocks(orc, golden):
    g = golden("kquant_superblocks.json")
    w4 = orc.dequant_superblock(_record(g["q4k"]["set_bytes"], 144), orc.Q4_K)
    for i, v in g["q4k"]["expect"].items():
        assert w4[int(i)] == v, i
    assert np.all(w4[2:32] == -0.125) and np.all(w4[64:] == 0.0)
    assert np.all(np.delete(w4[32:64], 16) == -5.625)
    for parity, key in ((0, "set_bytes_even"), (1, "set_bytes_odd")):
        w6 = orc.dequant_superblock(_record(g["q6k"][key], 210), orc.Q6_K, parity)
        for i, v in g["q6k"]["expect"].items():
            assert w6[int(i)] == v, (parity, i)
        assert np.all(w6[1:16] == 48.0) and np.all(w6[16:240] == 0.0)


def test_kquant_saturation_and_zero_scale(orc):
    rec = np.zeros(144, np.uint8)
    rec[0:2] = np.array([1.0], np.float16).view(np.uint8)       # d = 1, dmin = 0
    rec[4:12] = 63                                              # sc_j = 63, mn_j low bits 0
    rec[16:144] = 0xFF                                          # q = 15 everywhere
    assert np.all(orc.dequant_superblock(rec, orc.Q4_K) == 63 * 15)
    rec[2:4] = np.array([0.5], np.float16).view(np.uint8)       # dmin = 0.5
    rec[4:12] = 63 | (3 << 6)                                   # mn_j low bits 3
    rec[12:16] = 0xFF                                           # mn_j high nibbles 15 -> mn = 63
    assert np.all(orc.dequant_superblock(rec, orc.Q4_K) == 63 * 15 - 0.5 * 63)
    rec6 = np.zeros(210, np.uint8)
    rec6[208:210] = np.array([0.0], np.float16).view(np.uint8)  # d = 0
    rec6[:192] = 0xFF
    rec6[192:208] = 127
    assert np.all(orc.dequant_superblock(rec6, orc.Q6_K, 0) == 0.0)
    rec6[208:210] = np.array([2.0], np.float16).view(np.uint8)
    assert np.all(orc.dequant_superblock(rec6, orc.Q6_K, 0) == 2.0 * 127 * 31)   # q = 63 saturated
    odd = np.concatenate([rec6[208:210], rec6[:192], rec6[192:208]])
    assert np.all(orc.dequant_superblock(odd, orc.Q6_K, 1) == 2.0 * 127 * 31)


def _records_by_row(blocks, out, inn, nbytes):
    """Block-tiled records [out / 64][nsb][64][bytes] -> [out][nsb][bytes]."""
    nsb = inn // 256
    return blocks.reshape(out // 64, nsb, 64, nbytes).transpose(0, 2, 1, 3).reshape(out, nsb, nbytes)


def _dequant_tensor(orc, blocks, t, out, inn):
    rec = _records_by_row(blocks, out, inn, orc.RECORD_BYTES[t])
    return np.stack([np.concatenate([orc.dequant_superblock(rec[r, k], t, r) for k in range(inn // 256)])
                     for r in range(out)])


def test_kquant_roundtrip_against_source_weights(orc):
    w = synth.gaussian_weights(64, 2048, 7, 17)
    for t in (orc.Q4_K, orc.Q6_K):
        wr = _dequant_tensor(orc, synth.encode_kquant(w, t), t, 64, 2048)
        rel = np.sqrt(((wr - w) ** 2).mean() / (w ** 2).mean())
        assert rel < (0.12 if t == orc.Q4_K else 0.04)
        sub = 32 if t == orc.Q4_K else 16
        wg = np.abs(w.reshape(-1, sub)).max(1)
        assert np.all(np.abs(wr - w).reshape(-1, sub).max(1) <= wg * (0.2 if t == orc.Q4_K else 0.05) + 1e-7)


def test_kquant_gemv_is_dequant_then_matmul(orc):
    out, inn = 128, 1280
    w = synth.gaussian_weights(out, inn, 7, 18)
    x = synth.bf16_normal((3, inn), 7, 19)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in (orc.Q4_K, orc.Q6_K):
        blocks = synth.encode_kquant(w, t)
        W = _dequant_tensor(orc, blocks, t, out, inn)
        y = orc.gemv_kquant(blocks, t, out, inn, x)
        assert np.allclose(y, xf @ W.T, rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        orc.gemv_kquant(blocks, 13, out, inn, x)


def test_kquant_step_bytes_match_published_footprint():
    # 96 Q4_K + 17 Q6_K tensors of the Llama-3.2-1B mix weigh 799.6 MB resident.
    mix = synth.llama32_kquant_mix()
    assert sum(1 for *_, t in mix if t == synth.Q4_K) == 96
    assert sum(1 for *_, t in mix if t == synth.Q6_K) == 17
    total = sum(o * i // 256 * synth.RECORD_BYTES[t] for _, o, i, t in mix)
    assert round(total / 1e6, 1) == 799.6


# ----------------------------------------------------------------------------- in-pass level decision

def _decide_layer(gd):
    L = gd["layer"]
    out, inn, batch = L["out"], L["in"], L["batch"]
    y = np.zeros((batch, out), np.float32)
    s = np.zeros((out, inn // 128), np.float32)
    for c, b in enumerate(L["blocks"]):
        rows = slice(64 * c, 64 * c + 64)
        s[rows, 0], s[rows, 1] = b["scale_group0"], b["scale_group1"]
        y[0, rows], y[1, rows] = b["y_batch0"], b["y_batch1"]
    return y, s


def test_level_decide_hand_worked(orc, golden):
    gd = golden("level_decide_hand.json")
    E = gd["expect"]
    y, s = _decide_layer(gd)
    lev, red = orc.level_decide(y, s, 2, 4, 0, lam=2.0 ** -14)
    assert red.tolist() == E["reduced_gamma2"]
    assert lev.tolist() == E["ladder_gamma2_kappa4_lambda2e-14"]
    assert orc.level_decide(y, s, 2, 3, 0, lam=2.0 ** -14)[0].tolist() == E["ladder_gamma2_kappa3_lambda2e-14"]
    for f, key in ((0.5, "share_gamma2_kappa4_f0.5"), (0.7, "share_gamma2_kappa4_f0.7"), (1.0, "share_gamma2_kappa4_f1.0")):
        assert orc.level_decide(y, s, 2, 4, 1, f=f)[0].tolist() == E[key], f
    assert orc.level_decide(y, s, 1, 4, 0, lam=1.0)[1][0] == E["reduced_gamma1_block0"]


def test_level_decide_ties_go_to_lower_index(orc):
    y = np.ones((1, 256), np.float32)
    s = np.full((256, 1), 0.01, np.float32)
    lev, red = orc.level_decide(y, s, 2, 4, 1, f=0.5)          # 4 equal scores, 2 rise
    assert len(set(red.tolist())) == 1
    assert lev.tolist() == [4, 4, 2, 2]


def test_level_decide_invariants(orc):
    g = np.random.default_rng(7)
    out, inn, batch = 64 * 40, 512, 3
    y = g.standard_normal((batch, out)).astype(np.float32) * g.uniform(0.1, 10, out).astype(np.float32)
    s = g.uniform(1e-4, 1e-2, (out, inn // 128)).astype(np.float32)
    lev_prev = None
    _, red = orc.level_decide(y, s, 1, 4, 0, lam=1.0)
    for lam in np.geomspace(red.max() * 1e3, red.min() * 1e-6, 12):
        lev, red2 = orc.level_decide(y, s, 1, 4, 0, lam=lam)
        assert np.array_equal(red, red2)
        assert lev.min() >= 1 and lev.max() <= 4
        if lev_prev is not None:
            assert np.all(lev >= lev_prev)                          # a lower lambda never lowers a level
        lev_prev = lev
    assert np.all(lev_prev == 4)                                    # lambda far below every score: all at kappa
    # the reduced score is additive over batch rows
    parts = sum(orc.level_decide(y[t:t + 1], s, 2, 4, 0, lam=1.0)[1] for t in range(batch))
    assert np.allclose(orc.level_decide(y, s, 2, 4, 0, lam=1.0)[1], parts, rtol=1e-12)
    # y x 2^a, s x 2^b scales r by 2^(2a + 4b) exactly; the ladder moves with lambda
    lam = float(np.median(red)) * 4
    base = orc.level_decide(y, s, 2, 4, 0, lam=lam)
    scaled = orc.level_decide(y * np.float32(4), s * np.float32(0.5), 2, 4, 0, lam=lam * 2.0 ** (4 - 4))
    assert np.array_equal(scaled[1], base[1] * 2.0 ** (4 - 4))
    assert np.array_equal(scaled[0], base[0])
    y2 = orc.level_decide(y * np.float32(2), s, 2, 4, 0, lam=lam * 4)
    assert np.array_equal(y2[1], base[1] * 4) and np.array_equal(y2[0], base[0])
    s2 = orc.level_decide(y, s * np.float32(2), 2, 4, 0, lam=lam * 16)
    assert np.array_equal(s2[1], base[1] * 16) and np.array_equal(s2[0], base[0])
    # share: exactly floor(f nb) rise, each lifted score >= every other
    for f in (0.0, 0.1, 0.16, 0.5, 0.99, 1.0):
        lev, r = orc.level_decide(y, s, 2, 3, 1, f=f)
        up = lev == 3
        assert up.sum() == int(np.floor(f * (out // 64)))
        assert set(np.unique(lev).tolist()) <= {2, 3}
        if 0 < up.sum() < len(up):
            assert r[up].min() >= r[~up].max()


def test_level_decide_degenerate(orc):
    y = np.ones((1, 128), np.float32)
    s = np.full((128, 2), 0.5, np.float32)
    assert orc.level_decide(y, s, 3, 3, 0, lam=0.0)[0].tolist() == [3, 3]        # kappa = gamma: no rungs
    assert orc.level_decide(y, s, 3, 3, 1, f=1.0)[0].tolist() == [3, 3]
    assert orc.level_decide(y * 0, s, 2, 4, 0, lam=1e-30)[0].tolist() == [2, 2]   # zero draft stays at base
    assert orc.level_decide(y * 0, s, 2, 4, 0, lam=0.0)[0].tolist() == [4, 4]     # 0 >= 0 at every rung
    for bad in ((0, 4), (3, 2), (2, 5)):
        with pytest.raises(ValueError):
            orc.level_decide(y, s, bad[0], bad[1], 0, lam=1.0)


# ----------------------------------------------------------------------------- verified speculation

def test_spec_accept_hand_cases(orc):
    assert orc.spec_accept([5, 6, 7, 8], [5, 6, 7, 8]) == (4, 4)      # every draft verified
    assert orc.spec_accept([5, 6, 7, 8], [1, 6, 7, 8]) == (0, 1)      # first draft rejected: the correction only
    assert orc.spec_accept([5, 6, 7, 8], [5, 6, 0, 8]) == (2, 3)      # later agreement does not count
    assert orc.spec_accept([5, 6, 7, 8], [5, 6, 7, 0]) == (3, 4)
    assert orc.spec_accept([3], [3]) == (1, 1)
    assert orc.spec_accept([], []) == (0, 0)


def test_spec_emits_the_d8_greedy_tokens(orc):
    """Zero KL: whatever the drafts, the emitted tokens are the D8 argmax tokens of the
    window's first steps, and a D4 draft that matches D8 everywhere is accepted whole."""
    g = np.random.default_rng(11)
    vocab, inn, k = 512, 256, 8
    q, s = synth.int8_layer(vocab, inn, 12)
    x = synth.bf16_normal((k, inn), 13)
    lv4, lv8 = np.full(vocab // 64, 2, np.uint8), np.full(vocab // 64, 4, np.uint8)
    d4 = orc.gemv_depth(q, s, lv4, x)
    d8 = orc.gemv_depth(q, s, lv8, x)
    draft = orc.logit_gate(d4.astype(np.float32), 0.0, 0.0)[2][:, 0]
    verified = orc.logit_gate(d8.astype(np.float32), 0.0, 0.0)[2][:, 0]
    assert np.array_equal(verified, np.argmax(d8, axis=1))
    a, e = orc.spec_accept(draft, verified)
    assert np.all(draft[:a] == verified[:a]) and (a == k or draft[a] != verified[a])
    assert e == min(a + 1, k)
    # a window whose drafts are replaced by the verified tokens is accepted whole
    assert orc.spec_accept(verified, verified) == (k, k)
    # with one row dominating every logit vector, D4 and D8 agree
    q2 = q.copy()
    q2[7] = 127
    xp = synth.f32_to_bf16_bits(np.abs(synth.bf16_bits_to_f32(x)))
    t4 = np.argmax(orc.gemv_depth(q2, s, lv4, xp), axis=1)
    t8 = np.argmax(orc.gemv_depth(q2, s, lv8, xp), axis=1)
    assert np.all(t8 == 7) and orc.spec_accept(t4, t8) == (k, k)
