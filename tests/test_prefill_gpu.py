"""GPU parity of the prefill GEMM (grinqh_prefill_gemm): every row at the full
width b_max, a block of T tokens, against the oracle's GEMV of each token with
b_i = b_max for every row (the same tolerance as the decode path)."""
import numpy as np
import pytest
import torch

import oracle
from _gpu_helpers import ABS, REL, to_dev
from input_adaptive_bit_b200 import (grinqh_check_device_error, grinqh_prefill_gemm,
                                     grinqh_prefill_workspace_bytes)
from input_adaptive_bit_b200.layer import GrinqhLinear

pytestmark = pytest.mark.gpu


def run_case(seed, T, d_in, d_out, b_max, phi=None, tokens=None, outs=None):
    """Runs the prefill GEMM on seeded inputs and compares the given tokens (default:
    the first, the last and six random ones) on the given outputs (default: all)
    with the oracle's full-width GEMV."""
    g = np.random.default_rng(seed)
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    X = g.standard_normal((T, d_in)).astype(np.float16)
    lin = GrinqhLinear(q, s, z, b_max)
    Y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = grinqh_prefill_workspace_bytes()
    ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    ph = None if phi is None else to_dev(np.asarray(phi, np.float32))
    grinqh_prefill_gemm(lin.planes, lin.s, lin.z, to_dev(X), ph, T, d_in, d_out, b_max, Y, ws, ws.numel())
    torch.cuda.synchronize()
    grinqh_check_device_error(ws)
    Yh = Y.cpu().numpy().astype(np.float64)
    assert np.isfinite(Yh).all()
    planes = oracle.pack(q, b_max)
    full = np.full(d_in, b_max, np.uint8)
    if tokens is None:
        tokens = sorted(set([0, T - 1] + list(g.integers(0, T, 6))))
    cols = np.arange(d_out) if outs is None else np.asarray(outs, np.int32)
    for t in tokens:
        y_ref, bound = oracle.gemv(planes, s, z, X[t], full, b_max,
                                   phi=None if phi is None else np.asarray(phi, np.float64),
                                   outs=None if outs is None else cols, threads=oracle.max_threads())
        got = Yh[t][cols]
        ok = oracle.within_tolerance(got, y_ref, bound, REL, ABS)
        assert ok.all(), (t, cols[~ok][:5], got[~ok][:5], y_ref[~ok][:5])


@pytest.mark.parametrize("T,d_in,d_out,b_max", [
    (1, 128, 128, 8),          # one token, one group, one tile
    (5, 512, 256, 8),          # ragged token count (padded to 16)
    (64, 1024, 1024, 8),       # several groups per slice
    (130, 2048, 512, 6),       # two token blocks, the second of 2 tokens
    (48, 4096, 384, 4),        # many split-K slices
    (16, 256, 128, 2),         # one plane
])
def test_prefill_matches_the_oracle_at_full_width(T, d_in, d_out, b_max):
    run_case(T + d_in + b_max, T, d_in, d_out, b_max)


def test_prefill_with_an_explicit_phi_table():
    run_case(99, 20, 512, 256, 8, phi=[0.0, 0.1, -0.2, 0.3, 0.45])


def test_prefill_with_many_chunks_per_cta():
    # 16 tiles x 64 chunks = 1024 work units over the GPU's CTAs: every CTA runs
    # pieces of several chunks (the accumulator carried across MMAs, the copy
    # rings wrapping around) and ranges that cross from one tile into the next
    run_case(5, 16, 8192, 2048, 8, tokens=[0, 7, 15])


def test_prefill_with_many_chunks_per_cta_and_phi():
    run_case(6, 24, 4096, 4096, 6, phi=[0.0, 0.2, -0.1, 0.3], tokens=[0, 11, 23])


def test_prefill_at_the_benchmark_shape_on_sampled_outputs():
    # the gate projection of the prefill benchmark (4096 -> 12288, a 128-token
    # block, b_max 8), in the benchmark's launch configuration; 512 sampled
    # outputs (the first and last tile included) of four tokens
    g = np.random.default_rng(8)
    outs = np.unique(np.concatenate([np.arange(128), np.arange(12288 - 128, 12288),
                                     g.integers(0, 12288, 256)]))
    run_case(7, 128, 4096, 12288, 8, tokens=[0, 1, 64, 127], outs=outs)


def test_prefill_explicit_phi_where_the_offset_cancels_the_codes():
    # codes clustered at 128 with z = -128 s, so s q + z nearly cancels, and an
    # explicit phi_P = 0.45: the rebuild must not round z + s phi_P to fp16 (that
    # one error, shared by a group's weights, measures 1.4x the tolerance here)
    g = np.random.default_rng(11)
    T, d_in, d_out = 8, 2048, 256
    q = np.clip(np.round(g.normal(128, 2, size=(d_in, d_out))), 0, 255).astype(np.uint8)
    s = np.full((d_in // 128, d_out), 0.01, np.float16)
    z = (-(s.astype(np.float64) * 128)).astype(np.float16)
    X = g.standard_normal((T, d_in)).astype(np.float16)
    phi = np.array([0.0, 0.1, -0.2, 0.3, 0.45])
    lin = GrinqhLinear(q, s, z, 8)
    Y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(grinqh_prefill_workspace_bytes(), 256), dtype=torch.uint8, device="cuda")
    grinqh_prefill_gemm(lin.planes, lin.s, lin.z, to_dev(X), to_dev(phi.astype(np.float32)), T, d_in, d_out,
                        8, Y, ws, ws.numel())
    torch.cuda.synchronize()
    grinqh_check_device_error(ws)
    Yh = Y.cpu().numpy().astype(np.float64)
    planes = oracle.pack(q, 8)
    full = np.full(d_in, 8, np.uint8)
    for t in range(T):
        y_ref, bound = oracle.gemv(planes, s, z, X[t], full, 8, phi=phi, threads=oracle.max_threads())
        ok = oracle.within_tolerance(Yh[t], y_ref, bound, REL, ABS)
        assert ok.all(), (t, np.flatnonzero(~ok)[:5])
