"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module produces data only: Gaussian weights and their stored encodings
(int8 codes with fp32 absmax scales; Q4_K / Q6_K super-block records), bf16
activation vectors, depth maps, block coordinates and lens parameters. It holds
none of the read path's arithmetic (no depth reconstruction, no product, no lens
rule, no gate). The pages' models and datasets are not available, so every
workload is stood in for by its shapes with N(0, 0.02) weights and N(0, 1)
activations, drawn from ``numpy.random.Generator(PCG64)`` streams keyed by
``SeedSequence`` entropy tuples.

Encodings (the stored formats the read path takes as given):
  * int8: per row, per 128-column group, scale = absmax / 127 (fp32),
    code = clamp(round_half_even(w / scale), -127, 127); an all-zero group has
    scale 0 and codes 0.
  * Q4_K / Q6_K: GGUF-style super-blocks of 256 weights with the GGUF byte
    counts (144 and 210 bytes) in this project's own field layout, quantized by
    absmax per sub-block (asymmetric min/max for Q4_K).
"""
from __future__ import annotations

import numpy as np

Q4_K = 12
Q6_K = 14
RECORD_BYTES = {Q4_K: 144, Q6_K: 210}


def rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


# --------------------------------------------------------------------------- bf16

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_normal(shape, *key: int) -> np.ndarray:
    """bf16 N(0, 1) activations as uint16 bit patterns."""
    return f32_to_bf16_bits(rng(*key).standard_normal(shape, dtype=np.float32))


# --------------------------------------------------------------------------- int8 codes

def gaussian_weights(out: int, inn: int, *key: int, std: float = 0.02) -> np.ndarray:
    w = rng(*key).standard_normal((out, inn), dtype=np.float32)
    w *= np.float32(std)
    return w


def quantize_int8(w: np.ndarray):
    """Symmetric absmax int8 codes, fp32 scale per row per 128 columns."""
    out, inn = w.shape
    assert inn % 128 == 0
    wg = w.reshape(out, inn // 128, 128)
    amax = np.abs(wg).max(axis=2)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    t = np.rint(wg / safe[:, :, None])
    np.clip(t, -127, 127, out=t)
    t[s == 0] = 0
    return t.astype(np.int8).reshape(out, inn), s


def int8_layer(out: int, inn: int, *key: int):
    """Gaussian weights -> (codes int8 [out, in], scales fp32 [out, in/128])."""
    return quantize_int8(gaussian_weights(out, inn, *key))


def seeded_levels(nblocks: int, *key: int, low: int = 0, high: int = 4) -> np.ndarray:
    return rng(*key).integers(low, high + 1, size=nblocks).astype(np.uint8)


# --------------------------------------------------------------------------- K-quant records

def _fp16(a):
    return np.asarray(a, dtype=np.float32).astype(np.float16)


def encode_q4k(w: np.ndarray) -> np.ndarray:
    """Encode rows of weights (out % 64 == 0, in % 256 == 0) as 144-byte Q4_K records in
    block-tiled order (see kquant_tile_order).

    Record: [0,2) d fp16, [2,4) dmin fp16, byte 4 + j = sc_j | (mn_j & 3) << 6,
    nibble j of the word at 12 = mn_j >> 2, byte 16 + 16 j + b = q[32 j + b] | q[32 j + 16 + b] << 4.
    """
    out, inn = w.shape
    assert inn % 256 == 0 and out % 64 == 0
    sb = w.reshape(-1, 8, 32).astype(np.float32)
    n = sb.shape[0]
    lo = np.minimum(sb.min(axis=2), 0.0).astype(np.float32)
    hi = np.maximum(sb.max(axis=2), 0.0).astype(np.float32)
    a = ((hi - lo) / np.float32(15.0)).astype(np.float32)
    b = (-lo).astype(np.float32)
    d16 = _fp16(a.max(axis=1) / np.float32(63.0))
    m16 = _fp16(b.max(axis=1) / np.float32(63.0))
    d = d16.astype(np.float32)[:, None]
    dm = m16.astype(np.float32)[:, None]
    sc = np.where(d > 0, np.rint(a / np.where(d > 0, d, 1)), 0)
    sc = np.clip(sc, 0, 63).astype(np.int64)
    mn = np.where(dm > 0, np.rint(b / np.where(dm > 0, dm, 1)), 0)
    mn = np.clip(mn, 0, 63).astype(np.int64)
    step = (d * sc.astype(np.float32)).astype(np.float32)[:, :, None]
    off = (dm * mn.astype(np.float32)).astype(np.float32)[:, :, None]
    q = np.where(step > 0, np.rint((sb + off) / np.where(step > 0, step, 1)), 0)
    q = np.clip(q, 0, 15).astype(np.uint8)                       # [n, 8, 32]
    rec = np.zeros((n, 144), np.uint8)
    rec[:, 0:2] = d16.view(np.uint8).reshape(n, 2)
    rec[:, 2:4] = m16.view(np.uint8).reshape(n, 2)
    rec[:, 4:12] = (sc | ((mn & 3) << 6)).astype(np.uint8)
    nib = (mn >> 2).astype(np.uint8)
    rec[:, 12:16] = nib[:, 0::2] | (nib[:, 1::2] << 4)
    rec[:, 16:144] = (q[:, :, :16] | (q[:, :, 16:] << 4)).reshape(n, 128)
    return kquant_tile_order(rec, out, inn // 256)


def encode_q6k(w: np.ndarray) -> np.ndarray:
    """Encode rows of weights (out % 64 == 0, in % 256 == 0) as 210-byte Q6_K records in
    block-tiled order (see kquant_tile_order).

    A record's layout depends on the parity of its row: even row -> [0,192) q, [192,208)
    int8 scales, [208,210) d; odd row -> [0,2) d, [2,194) q, [194,210) scales (in the tiled
    order an odd row's record starts 2 bytes past a 4-byte boundary, so its q area is
    4-byte aligned). The q area
    holds, for chunk t (48 bytes) and group m (12 bytes: words A, B, C), with
    W(j, L) = 16 j + 4 t + L: A byte L = lo4 q[W(4m,L)] | lo4 q[W(4m+1,L)] << 4,
    B byte L = lo4 q[W(4m+2,L)] | lo4 q[W(4m+3,L)] << 4, C byte L = hi2 q[W(4m+2,L)]
    | hi2 q[W(4m+3,L)] << 2 | hi2 q[W(4m,L)] << 4 | hi2 q[W(4m+1,L)] << 6.
    """
    out, inn = w.shape
    assert inn % 256 == 0 and out % 64 == 0
    sb = w.reshape(-1, 16, 16).astype(np.float32)
    n = sb.shape[0]
    a = (np.abs(sb).max(axis=2) / np.float32(31.0)).astype(np.float32)
    d16 = _fp16(a.max(axis=1) / np.float32(127.0))
    d = d16.astype(np.float32)[:, None]
    sc = np.where(d > 0, np.rint(a / np.where(d > 0, d, 1)), 0)
    sc = np.clip(sc, -128, 127).astype(np.int64)
    step = (d * sc.astype(np.float32)).astype(np.float32)[:, :, None]
    q = np.where(step > 0, np.rint(sb / np.where(step > 0, step, 1)), 0)
    q = (np.clip(q, -32, 31) + 32).astype(np.uint8)               # [n, 16 j, 16 = 4 t + L]
    qj = q.reshape(n, 4, 4, 4, 4)                                  # [n, m, s, t, L], j = 4 m + s
    lo4 = qj & 15
    hi2 = qj >> 4
    A = lo4[:, :, 0] | (lo4[:, :, 1] << 4)                         # [n, m, t, L]
    B = lo4[:, :, 2] | (lo4[:, :, 3] << 4)
    Cw = hi2[:, :, 2] | (hi2[:, :, 3] << 2) | (hi2[:, :, 0] << 4) | (hi2[:, :, 1] << 6)
    area = np.stack([A, B, Cw], axis=3)                           # [n, m, t, word, L]
    area = area.transpose(0, 2, 1, 3, 4).reshape(n, 192)          # chunk t, group m, word, lane
    rec = np.zeros((n, 210), np.uint8)
    scb = sc.astype(np.int8).view(np.uint8)
    db = d16.view(np.uint8).reshape(n, 2)
    even = ((np.arange(n) // (inn // 256)) % 2) == 0               # record n belongs to row n // (in / 256)
    rec[even, 0:192] = area[even]
    rec[even, 192:208] = scb[even]
    rec[even, 208:210] = db[even]
    odd = ~even
    rec[odd, 0:2] = db[odd]
    rec[odd, 2:194] = area[odd]
    rec[odd, 194:210] = scb[odd]
    return kquant_tile_order(rec, out, inn // 256)


def kquant_tile_order(rec: np.ndarray, out: int, nsb: int) -> np.ndarray:
    """Row-major records [out][nsb][bytes] -> block-tiled [out / 64][nsb][64][bytes], flat.

    A tile of 64 rows x k consecutive super-blocks is then one contiguous byte range."""
    nb = rec.shape[-1]
    return np.ascontiguousarray(rec.reshape(out // 64, 64, nsb, nb).transpose(0, 2, 1, 3)).reshape(-1)


def encode_kquant(w: np.ndarray, ggml_type: int) -> np.ndarray:
    if ggml_type == Q4_K:
        return encode_q4k(w)
    if ggml_type == Q6_K:
        return encode_q6k(w)
    raise ValueError(f"unsupported K-quant type {ggml_type}")


# --------------------------------------------------------------------------- workload shapes

# Qwen3-0.6B-shaped decode step: (name, out, in) per layer, plus the tied head.
QWEN3_06B_LAYER = [("q_proj", 2048, 1024), ("k_proj", 1024, 1024), ("v_proj", 1024, 1024),
                   ("o_proj", 1024, 2048), ("gate_proj", 3072, 1024), ("up_proj", 3072, 1024),
                   ("down_proj", 1024, 3072)]
QWEN3_06B_LAYERS = 28
QWEN3_06B_HEAD = ("lm_head", 151936, 1024)

# Llama-3.2-1B-shaped decode step.
LLAMA32_1B_LAYER = [("q_proj", 2048, 2048), ("k_proj", 512, 2048), ("v_proj", 512, 2048),
                    ("o_proj", 2048, 2048), ("gate_proj", 8192, 2048), ("up_proj", 8192, 2048),
                    ("down_proj", 2048, 8192)]
LLAMA32_1B_LAYERS = 16
LLAMA32_1B_HEAD = ("lm_head", 128256, 2048)


def qwen3_step_shapes():
    """The 197 GEMV shapes of one Qwen3-0.6B decode step, layer order, head last."""
    shapes = []
    for layer in range(QWEN3_06B_LAYERS):
        for name, o, i in QWEN3_06B_LAYER:
            shapes.append((f"layers.{layer}.{name}", o, i))
    shapes.append(QWEN3_06B_HEAD)
    return shapes


def llama32_kquant_mix():
    """(name, out, in, ggml_type) for the Q4_K_M-style mix of the Llama-3.2-1B step.

    Q6_K for v_proj and down_proj in the even-indexed layers and for the tied head,
    Q4_K for everything else: 96 Q4_K and 17 Q6_K tensors.
    """
    mix = []
    for layer in range(LLAMA32_1B_LAYERS):
        for name, o, i in LLAMA32_1B_LAYER:
            t = Q6_K if (layer % 2 == 0 and name in ("v_proj", "down_proj")) else Q4_K
            mix.append((f"layers.{layer}.{name}", o, i, t))
    name, o, i = LLAMA32_1B_HEAD
    mix.append((name, o, i, Q6_K))
    return mix


def lens_stack_layers(nblocks: int = 14708, nlayers: int = 35):
    """Blocks per layer when nblocks are split as evenly as possible over nlayers."""
    base, extra = divmod(nblocks, nlayers)
    return [base + (1 if l < extra else 0) for l in range(nlayers)]


def lens_inputs(nblocks: int, nlenses: int, *key: int, rmin: float = 0.02, rmax: float = 0.08):
    """Block coordinates, lens centres and radii, all uniform in the unit square."""
    g = rng(*key)
    xy = g.random((nblocks, 2), dtype=np.float32)
    cxy = g.random((nlenses, 2), dtype=np.float32)
    r = (np.float32(rmin) + np.float32(rmax - rmin) * g.random(nlenses, dtype=np.float32)).astype(np.float32)
    return xy, cxy, r


def even_stops(kappa: int, gamma: int) -> np.ndarray:
    """Evenly spaced profile stops s_kappa < ... < s_(gamma+1) = 1, ascending."""
    n = kappa - gamma
    return np.array([(j + 1) / n for j in range(n)], dtype=np.float32)
