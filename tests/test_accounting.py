"""The benchmark's algorithmic byte counts against closed forms of the workloads (CPU).

Weight bytes actually read at depth d: d / 8 bytes per weight of the planes read plus 4 bytes
of fp32 scale per 128 weights of every block that is read (ZERO blocks read nothing); K-quant
tensors read their super-block records. These are the numerators of every GB/s and roofline
figure the benchmark prints."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from variable_precision_weight_b200 import synth  # noqa: E402


def test_plane_bytes_closed_form():
    for inn in (128, 1024, 3072, 14336):
        for level in range(5):
            d = 2 * level
            want = 0 if level == 0 else 64 * inn * d // 8 + 64 * (inn // 128) * 4
            assert bench.plane_bytes(inn, level) == want, (inn, level)


def test_decode_step_bytes():
    shapes = synth.qwen3_step_shapes()
    weights = sum(o * i for _, o, i in shapes)
    assert len(shapes) == 197 and weights == 595_984_384
    d4 = sum((o // 64) * bench.plane_bytes(i, 2) for _, o, i in shapes)
    assert d4 == weights // 2 + weights // 128 * 4 == 316_616_704      # 298.0 MB planes + 18.6 MB scales
    # the D4 -> D8 residual reads the two low planes and the scales again: the same count
    res = sum((o // 64) * (256 * (i // 128) + 2048 * (i // 128) * 2) for _, o, i in shapes)
    assert res == d4
    # against an all-D8 read, 100 steps with 16 escalations move 0.58 of the plane bytes
    # ((100 + 16) x 4 bits vs 100 x 8 bits) and 0.598 of all bytes (each pass re-reads the scales)
    d8 = sum((o // 64) * bench.plane_bytes(i, 4) for _, o, i in shapes)
    assert d8 == weights + weights // 128 * 4
    assert (100 + 16) * (weights // 2) / (100 * weights) == 0.58
    assert abs((100 * d4 + 16 * res) / (100 * d8) - 0.5976) < 1e-4


def test_lens_stack_and_large_layer_bytes():
    per = synth.lens_stack_layers(14708, 35)
    assert sum(per) == 14708 and per.count(421) == 8 and per.count(420) == 27
    # config 3 at uniform D6: 44.0 / 44.0 / 12.6 MB of planes + 1.8 / 1.8 / 0.5 MB of scales
    for (o, i), planes, scales in (((14336, 4096), 44_040_192, 1_835_008), ((4096, 14336), 44_040_192, 1_835_008),
                                   ((4096, 4096), 12_582_912, 524_288)):
        assert (o // 64) * bench.plane_bytes(i, 3) == planes + scales


def test_kquant_step_bytes():
    mix = synth.llama32_kquant_mix()
    total = sum(o * (i // 256) * synth.RECORD_BYTES[t] for _, o, i, t in mix)
    assert total == 799_592_448                                        # the page's 799.6 MB
