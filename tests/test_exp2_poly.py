"""The minimax polynomial the kernels use for part of their exp2 work:
regenerated from its fit script it matches the committed header, its error
is bounded as stated, and its fp32 range reduction has no overflow path."""
import numpy as np
import pytest

from triangle_biased_attention_b200 import exp2_poly as E


def test_header_matches_fit_script():
    with open(E.HEADER) as f:
        assert f.read() == E.header_text(3)


def test_remez_equioscillates_and_beats_taylor():
    c, err = E.remez(3)
    f = np.linspace(-0.5, 0.5, 100001)
    rel = np.polyval(c[::-1], f) / np.exp2(f) - 1.0
    assert abs(np.abs(rel).max() - err) < 1e-9
    # minimax: the error reaches +-err at degree + 2 points with alternating sign
    peaks = np.sign(rel[np.abs(np.abs(rel) - err) < 1e-3 * err])
    assert (np.diff(peaks) != 0).sum() >= 3
    # a degree-3 Taylor expansion of 2^f about 0 is far worse on the same interval
    ln2 = np.log(2.0)
    taylor = 1 + f * ln2 + (f * ln2) ** 2 / 2 + (f * ln2) ** 3 / 6
    assert np.abs(taylor / np.exp2(f) - 1).max() > 5 * err


@pytest.mark.parametrize("degree,bound", [(3, 8e-5), (4, 3e-6)])
def test_fp32_emulation_error(degree, bound):
    c32, _ = E.coefficients_f32(degree)
    x = np.concatenate([np.linspace(-40, 16, 400001, dtype=np.float32),
                        np.float32(np.random.default_rng(1).uniform(-125, 16, 100000))])
    y = E.exp2_emulated(x, c32).astype(np.float64)
    t = np.exp2(x.astype(np.float64))
    assert np.all(np.abs(y / t - 1) <= bound)


def test_range_reduction_never_overflows():
    """-inf, huge negative values and the clamp boundary give tiny finite
    results (zero once rounded to fp16), never NaN or inf."""
    c32, _ = E.coefficients_f32(3)
    x = np.array([-np.inf, -1e30, -1e9, -5e3, -200, -126.5, -125.5, -125, -124.5], dtype=np.float32)
    y = E.exp2_emulated(x, c32)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -120)
    assert np.all(y.astype(np.float16) == 0)
