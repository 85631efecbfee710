"""The seeded input recipe (CPU): row layout of the packed sequence, seeding,
shapes and value distributions of the configured workloads, on reduced sizes
where the full ones would take long to draw."""
import numpy as np
import pytest

import synthetic as S


def test_packed_modality_counts_and_order():
    # non-video rows are round(0.014 M); text takes the odd row; [text | video | audio]
    assert S.packed_modality_counts(4096) == (29, 4039, 28)
    assert S.packed_modality_counts(16384) == (115, 16155, 114)
    segs = S.packed_segments(16384)
    assert [(s.name, s.begin, s.end) for s in segs] == [("text", 0, 115), ("video", 115, 16270),
                                                        ("audio", 16270, 16384)]


def test_layers_are_seeded_and_bf16():
    a = S.make_layer(1, m=256, k=512, n=256)
    b = S.make_layer(1, m=256, k=512, n=256)
    assert a.x.dtype == np.uint16 and a.w.dtype == np.uint16 and a.bias.dtype == np.uint16
    assert np.array_equal(a.x, b.x) and np.array_equal(a.w, b.w) and np.array_equal(a.bias, b.bias)
    c = S.make_layer(2, m=256, k=512, n=256)                  # another config index: another seed
    assert not np.array_equal(a.w, c.w)
    # sweep layers differ from one another, and their width cycles through the sweep's N values
    l0, l4 = S.make_layer(4, m=3 * 64, k=256, layer=0), S.make_layer(4, m=3 * 64, k=256, layer=4)
    assert l0.n == 5120 and l4.n == 15360 and not np.array_equal(l0.x, l4.x)
    assert [s.name for s in l0.segments] == ["text", "video", "audio"]
    assert [s.end - s.begin for s in l0.segments] == [64, 64, 64]


def test_configured_shapes():
    want = {0: (256, 512, 512, 16), 1: (4096, 5120, 5120, 32), 2: (16384, 5120, 20480, 32),
            3: (16384, 20480, 5120, 32)}
    for cfg, (m, k, n, r) in want.items():
        spec = S.CONFIGS[cfg]
        assert (spec["m"], spec["k"], spec["n"], spec["rank"]) == (m, k, n, r)
    assert S.CONFIGS[4]["m"] == 3 * 4096 and S.CONFIGS[4]["layers"] == 48


def test_value_distributions():
    L = S.make_layer(1, m=2048, k=2048, n=1024)
    w = S.bf16_bits_to_f32(L.w).astype(np.float64)
    assert abs(w.std() - 0.02) < 0.0005 and abs(w.mean()) < 0.0005          # N(0, 0.02^2) weights
    x = S.bf16_bits_to_f32(L.x).astype(np.float64)
    video = L.segments[1]
    prof = np.abs(x[video.begin:video.end]).max(axis=0)
    # heavy channels: about 1 % of the channels carry an absmax well above the others'
    top = np.sort(prof)[::-1]
    assert top[:10].min() > 5 * np.median(prof)
    # config 3's activations pass through GELU: nothing below its minimum, about -0.17
    L3 = S.make_layer(3, m=512, k=1024, n=256)
    x3 = S.bf16_bits_to_f32(L3.x)
    assert x3.min() >= -0.1701 and (x3 < 0).mean() > 0.05


@pytest.mark.parametrize("v", [0.0, -0.0, 1.0, -2.5, 3.0e38, 1e-40])
def test_bf16_bits_round_trip(v):
    bits = S.f32_to_bf16_bits(np.array([v], np.float32))
    back = S.bf16_bits_to_f32(bits)
    # half a bf16 step: 2^-8 relative for normal values, 2^-134 absolute among the subnormals
    assert abs(float(back[0]) - float(np.float32(v))) <= max(abs(v) * 2 ** -8, 2.0 ** -134)
    assert np.signbit(back[0]) == np.signbit(np.float32(v))
