"""The seeded input generator: determinism, ranges and distributions."""
import numpy as np
import pytest

import synth


def test_splitmix64_reference_value():
    # First output of SplitMix64 from state 0 (Steele, Lea, Flood 2014; the
    # widely published reference value of the generator).
    assert synth.draw(0, 0) == 0xE220A8397B1DCDAF


def test_codes_deterministic_and_random_access():
    s = synth.MatrixSpec(3, 1, synth.KIND_DOWN, 17, 3, 64, 256)
    a = s.codes()
    assert np.array_equal(a, s.codes())
    assert np.array_equal(a[40:50], s.codes(40, 10))
    assert a.max() == 7 and a.min() == 0
    counts = np.bincount(a.ravel(), minlength=8)
    assert counts.min() > 0.8 * a.size / 8


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_scales_ranges(bits):
    s = synth.MatrixSpec(0, 0, 0, 0, bits, 512, 1024).scales()
    if bits == 4:
        assert set(np.unique(s)) <= {120, 121, 122}        # 2^-7 .. 2^-5
    else:
        v = s.view(np.float16).astype(np.float64)
        assert v.min() >= 0.00999 and v.max() <= 0.04001   # fp16 rounding of the ends
        assert abs(np.median(np.log2(v / 0.02))) < 0.05


def test_x_and_logits_distributions():
    x = synth.bf16_to_f64(synth.x_bf16(0, 0, 8, 4096))
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1) < 0.02
    assert np.array_equal(synth.x_bf16(0, 3, 2, 4096), synth.x_bf16(0, 0, 8, 4096)[3:5])
    b = synth.zipf_bias(0, 0, 256, 1.1)
    assert np.exp(b).sum() == pytest.approx(1.0, rel=1e-12)
    assert np.all(synth.zipf_bias(0, 0, 256, 0.0) == 0.0)
    L = synth.logits(0, 0, 0, 100, 256, 1.1)
    assert L.dtype == np.float32 and L.shape == (100, 256)
    hot = int(np.argmax(b))
    assert np.argmax(np.bincount(np.argsort(-L, axis=1)[:, :6].ravel(), minlength=256)) == hot
