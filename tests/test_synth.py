"""The seeded input generators (CPU only)."""
import numpy as np
import pytest

import synth


def test_seeded_and_reproducible():
    a = synth.make_case(synth.config0()[0])
    b = synth.make_case(synth.config0()[0])
    for f in ("q", "s", "z", "x", "theta"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    c = synth.make_case(synth.Linear("other", 512, 512, config_id=1))
    assert not np.array_equal(a.x, c.x)


@pytest.mark.parametrize("bits", [8, 4])
def test_rtn_codes_in_range_and_close_to_w(bits):
    g = synth.rng(7)
    W = synth.gaussian_weights(g, 256, 64)
    q, s, z = synth.rtn_quantize(W, bits)
    assert q.dtype == np.uint8 and q.max() <= (1 << bits) - 1
    assert s.shape == (2, 64) and s.dtype == np.float16
    deq = np.repeat(s.astype(np.float64), 128, 0) * q + np.repeat(z.astype(np.float64), 128, 0)
    err = np.abs(deq - W)
    # half a step, plus the fp16 rounding of s and z
    assert (err <= np.repeat(s.astype(np.float64), 128, 0) * 0.5 + 2e-4).all()


def test_rtn_constant_group_gives_zero_codes():
    W = np.full((128, 16), 0.25, np.float32)
    q, s, z = synth.rtn_quantize(W, 8)
    assert (s == 0).all() and (q == 0).all() and (z == np.float16(0.25)).all()


def test_activation_outliers_and_dtype():
    x = synth.activations(synth.rng(1, 2, 3), 4096)
    assert x.dtype == np.float16
    assert np.sum(np.abs(x.astype(np.float32)) > 8) >= 30  # ~41 planted x20 entries
    t = synth.activations(synth.rng(1, 2, 3), 4096, "student_t")
    assert t.dtype == np.float16 and np.isfinite(t.astype(np.float32)).all()


@pytest.mark.parametrize("target", [2.0, 3.0, 3.3, 4.0])
def test_quantile_thresholds_realize_target(target):
    x = synth.activations(synth.rng(1, 0, 0), 8192)
    fr = synth.level_fractions(target)
    theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), fr)
    assert (np.diff(theta) >= 0).all()
    a = np.abs(x.astype(np.float32))
    b = 2 * (a[:, None] >= theta[None, :]).sum(1)
    assert abs(b.mean() - target) < 0.05


def test_uniform_thresholds():
    assert list(synth.uniform_thresholds(4, 8)) == [0, 0, np.inf, np.inf]
    assert list(synth.uniform_thresholds(0, 4)) == [np.inf, np.inf]


def test_configs_shapes():
    assert [(l.d_in, l.d_out) for l in synth.config0()] == [(512, 512)]
    c1 = synth.config1()
    assert len(c1) == 12 and {(l.d_in, l.d_out) for l in c1} == {
        (4096, 4096), (4096, 12288), (12288, 4096)}
    assert {l.uniform_b for l in synth.config2() if l.uniform_b} == {2, 4, 6, 8}
    assert {(l.d_in, l.d_out) for l in synth.config3()} == {(8192, 28672), (28672, 8192)}
    c4 = synth.config4()
    assert len(c4) == 224
    assert sum(l.d_in * l.d_out for l in c4[:7]) == 218_103_808
