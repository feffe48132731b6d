"""GPU parity of the small-batch decode step (grinqh_decode_gemv_batch): B <= 8
tokens through one linear, each with its own widths, against the oracle's
per-token definition (oracle.gemv_batch); the union widths bit-exact against
oracle.union_widths."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import ABS, REL, to_dev
from input_adaptive_bit_b200 import (grinqh_batch_workspace_bytes, grinqh_check_device_error,
                                     grinqh_decode_gemv_batch)
from input_adaptive_bit_b200.layer import GrinqhLinear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


@pytest.fixture(scope="module")
def ws():
    n = grinqh_batch_workspace_bytes()
    return torch.zeros(n, dtype=torch.uint8, device="cuda"), n


def make_inputs(seed, B, d_in, d_out, b_max, same_tokens=False):
    g = np.random.default_rng(seed)
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    X = np.stack([synth.activations(g, d_in) for _ in range(B)])
    if same_tokens:
        X[:] = X[0]
    P = b_max // 2
    theta = synth.quantile_thresholds(np.abs(X.astype(np.float32)).ravel(),
                                      np.full(P + 1, 1.0 / (P + 1)))
    return q, s, z, X, theta


def run_batch(q, s, z, X, theta, b_max, ws, phi=None, lin=None, outs=None):
    B, d_in = X.shape
    d_out = q.shape[1]
    lin = lin or GrinqhLinear(q, s, z, b_max)
    Y = torch.full((B, d_out), float("nan"), dtype=torch.float32, device="cuda")
    u = torch.full((d_in,), 255, dtype=torch.uint8, device="cuda")
    ph = None if phi is None else to_dev(np.asarray(phi, np.float32))
    grinqh_decode_gemv_batch(lin.planes, lin.s, lin.z, to_dev(X), to_dev(np.asarray(theta, np.float32)),
                             ph, B, d_in, d_out, b_max, Y, u, ws[0], ws[1])
    torch.cuda.synchronize()
    grinqh_check_device_error(ws[0])
    assert np.array_equal(u.cpu().numpy(), oracle.union_widths(X, theta, b_max)), "union widths differ"
    Yh = Y.cpu().numpy().astype(np.float64)
    planes = oracle.pack(q, b_max)
    if outs is None:
        Yr, bounds, _ = oracle.gemv_batch(planes, s, z, X, theta, b_max,
                                          phi=None if phi is None else np.asarray(phi, np.float64),
                                          threads=oracle.max_threads())
        ok = oracle.within_tolerance(Yh, Yr, bounds, REL, ABS)
        assert ok.all(), (np.argwhere(~ok)[:5], Yh[~ok][:5], Yr[~ok][:5])
    else:
        for t in range(B):
            b_t = oracle.assign(X[t], theta, b_max)
            yr, bound = oracle.gemv(planes, s, z, X[t], b_t, b_max, outs=outs,
                                    threads=oracle.max_threads())
            ok = oracle.within_tolerance(Yh[t, outs], yr, bound, REL, ABS)
            assert ok.all(), (t, np.flatnonzero(~ok)[:5])
    return lin, Yh


@pytest.mark.parametrize("B,d_in,d_out,b_max", [
    (1, 128, 128, 8),        # one token, one group, one tile
    (2, 512, 256, 8),
    (3, 1024, 2048, 8),
    (8, 1024, 512, 8),       # a full batch
    (5, 2048, 384, 6),
    (8, 1024, 3072, 6),
    (3, 1024, 256, 4),
    (8, 2048, 1024, 4),
    (4, 256, 128, 2),
    (8, 8192, 1024, 8),      # one tile: 148 CTAs share it (cluster pairs, then global memory)
    (4, 2048, 148 * 1024 + 16, 8),  # more tiles than CTAs, the last ragged and not 16-byte aligned
])
def test_batch_matches_the_per_token_oracle(B, d_in, d_out, b_max, ws):
    q, s, z, X, theta = make_inputs(B * 7 + d_in + b_max, B, d_in, d_out, b_max)
    outs = None
    if d_out > 8192:
        rng = np.random.default_rng(1)
        outs = np.unique(np.concatenate([np.arange(64), np.arange(d_out - 80, d_out),
                                         rng.integers(0, d_out, 200)])).astype(np.int32)
    run_batch(q, s, z, X, theta, b_max, ws, outs=outs)


def test_batch_with_an_explicit_phi_table(ws):
    q, s, z, X, theta = make_inputs(3, 4, 1024, 256, 8)
    run_batch(q, s, z, X, theta, 8, ws, phi=[0.0, 0.1, -0.2, 0.3, 0.45])


def test_batch_of_identical_tokens_gives_the_single_token_result(ws):
    q, s, z, X, theta = make_inputs(4, 6, 512, 128, 8, same_tokens=True)
    _, Y = run_batch(q, s, z, X, theta, 8, ws)
    for t in range(1, 6):
        assert np.array_equal(Y[t], Y[0])  # same inputs, same summation order


def test_batch_edge_values_ties_nan_inf(ws):
    # ties at a threshold, -0, NaN (width 0, adds nothing), and +-Inf in one token (that
    # token's outputs are non-finite; the other tokens must not be affected)
    q, s, z, X, theta = make_inputs(5, 4, 512, 256, 8)
    X[0, :4] = np.float16(theta[0])
    X[1, 4] = np.float16(-0.0)
    X[2, 5:9] = np.float16(np.nan)
    X[3, 10] = np.float16(np.inf)
    run_batch(q, s, z, X, theta, 8, ws)


def test_batch_with_every_row_inactive_in_some_tokens(ws):
    # token 1 has no active row (its y is exactly 0); token 0 every row at full width
    q, s, z, X, theta = make_inputs(6, 3, 1024, 1024, 8)
    X[1] = np.float16(0.0)
    theta = np.array([0.25, 0.5, 1.0, 2.0], np.float32)
    X[0] = np.float16(8.0)
    _, Y = run_batch(q, s, z, X, theta, 8, ws)
    assert (Y[1] == 0.0).all()


def test_batch_is_deterministic_and_leaves_the_workspace_zeroed(ws):
    q, s, z, X, theta = make_inputs(7, 8, 4096, 4096, 8)
    lin, Y1 = run_batch(q, s, z, X, theta, 8, ws)
    _, Y2 = run_batch(q, s, z, X, theta, 8, ws, lin=lin)
    assert np.array_equal(Y1, Y2)
    assert not ws[0][256:256 + 8 * 512].any()  # every arrival word is back at zero
