"""Pins of the oracle's small-batch decode step (oracle.union_widths,
oracle.gemv_batch): "GRINQH: Graded Input-Based Quantization Hierarchy for
Efficient LLM Generation", Limitations and outlook -- beyond batch 1 the
requests' active channels differ, so a step that rebuilds each weight once for
the batch reads the union of their planes.

The pins do not re-call the oracle's own per-token path: the union is checked
against one threshold compare of the element-wise largest |x|, and the batch
result against a plane-by-plane numpy computation from the base codes q, in
which each token keeps plane p of row i only where its own width exceeds 2p --
the form a shared-rebuild kernel uses."""
import numpy as np
import pytest

import oracle
import synth


def _case(seed, B, d_in=512, d_out=64, b_max=8):
    g = np.random.default_rng(seed)
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    X = np.stack([synth.activations(g, d_in) for _ in range(B)])
    P = b_max // 2
    theta = synth.quantile_thresholds(np.abs(X.astype(np.float32)).ravel(),
                                      np.full(P + 1, 1.0 / (P + 1)))
    return q, s, z, X, theta


@pytest.mark.parametrize("B", [2, 3, 8])
def test_union_is_the_width_of_the_largest_magnitude(B):
    # b is non-decreasing in |x|, so max_t b(x_t) = b(max_t |x_t|)
    _, _, _, X, theta = _case(10 + B, B)
    X[0, :3] = np.float16(theta[0])           # ties at a threshold
    X[1, 3] = np.float16(-0.0)
    X[-1, 4] = np.float16(np.inf)
    X[0, 5] = np.float16(np.nan)               # NaN has width 0 and adds nothing
    u = oracle.union_widths(X, theta, 8)
    xmax = np.fmax.reduce(np.abs(X.astype(np.float32)), axis=0).astype(np.float16)
    assert np.array_equal(u, oracle.assign(xmax, theta, 8))
    assert u[4] == 8


def test_union_reads_lie_between_the_largest_token_and_the_sum():
    _, _, _, X, theta = _case(3, 8)
    bs = np.stack([oracle.assign(x, theta, 8) for x in X]).astype(np.int64)
    u = oracle.union_widths(X, theta, 8).astype(np.int64)
    assert bs.sum(axis=1).max() <= u.sum() <= bs.sum()
    # identical tokens: the union is each token's own set
    same = np.stack([X[0]] * 4)
    assert np.array_equal(oracle.union_widths(same, theta, 8), oracle.assign(X[0], theta, 8))


def test_union_grows_with_the_batch():
    # the limitation the pages name: more requests, fewer skipped channels
    _, _, _, X, theta = _case(4, 8, d_in=1024)
    eff = [oracle.union_widths(X[:B], theta, 8).mean() for B in range(1, 9)]
    assert all(a <= b for a, b in zip(eff, eff[1:])) and eff[-1] > eff[0]


@pytest.mark.parametrize("B,b_max,use_phi", [(2, 8, False), (5, 8, True), (8, 4, False), (3, 6, True)])
def test_batch_step_by_planes_with_token_masks(B, b_max, use_phi):
    q, s, z, X, theta = _case(100 + B + b_max, B, b_max=b_max)
    P = b_max // 2
    phi = np.array([0.0] + [0.1 * (k + 1) * (-1) ** k for k in range(P)]) if use_phi else None
    planes = oracle.pack(q, b_max)
    Y, bounds, bs = oracle.gemv_batch(planes, s, z, X, theta, b_max, phi=phi)
    phi_t = oracle.phi_default(b_max) if phi is None else phi
    d_in, d_out = q.shape
    s64 = np.repeat(s.astype(np.float64), 128, axis=0)
    z64 = np.repeat(z.astype(np.float64), 128, axis=0)
    digits = [((q.astype(np.int64) >> (2 * (P - 1 - p))) & 3).astype(np.float64) for p in range(P)]
    for t in range(B):
        x = X[t].astype(np.float64)
        b = bs[t].astype(np.int64)
        y = np.zeros(d_out)
        for p in range(P):
            xm = np.where(b > 2 * p, x, 0.0)   # this token's rows that use plane p
            y += (xm[:, None] * s64 * 4.0 ** (P - 1 - p) * digits[p]).sum(axis=0)
        act = b > 0
        y += ((x * act)[:, None] * (s64 * phi_t[b // 2][:, None] + z64)).sum(axis=0)
        assert np.allclose(Y[t], y, rtol=1e-12, atol=1e-12 * np.abs(bounds[t]).max())
    # every token's bound is the sum of |w_hat| |x| over its active rows, so it
    # dominates |y| (a property of the definition, not a re-call)
    assert (np.abs(Y) <= bounds * (1 + 1e-12)).all()


def test_batch_of_one_is_the_single_token_step():
    q, s, z, X, theta = _case(7, 1)
    planes = oracle.pack(q, 8)
    Y, _, bs = oracle.gemv_batch(planes, s, z, X, theta, 8)
    y, _ = oracle.gemv(planes, s, z, X[0], oracle.assign(X[0], theta, 8), 8)
    assert Y.shape == (1, 64) and np.array_equal(Y[0], y)
