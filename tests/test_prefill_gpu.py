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


def run_case(seed, T, d_in, d_out, b_max, phi=None):
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
    planes = oracle.pack(q, b_max)
    full = np.full(d_in, b_max, np.uint8)
    rows = sorted(set([0, T - 1] + list(g.integers(0, T, 6))))
    for t in rows:
        y_ref, bound = oracle.gemv(planes, s, z, X[t], full, b_max,
                                   phi=None if phi is None else np.asarray(phi, np.float64),
                                   threads=oracle.max_threads())
        ok = oracle.within_tolerance(Yh[t], y_ref, bound, REL, ABS)
        assert ok.all(), (t, np.flatnonzero(~ok)[:5], Yh[t][~ok][:5], y_ref[~ok][:5])


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
