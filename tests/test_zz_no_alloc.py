"""grinqh_decode_gemv_noalloc: the decode GEMV for callers that cannot allocate
device memory (a host framework that owns all device memory and only lends
its plug-ins streams and tensors, or a path that must never reach the
allocator).  It must give the same y as the workspace-based entry points.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from input_adaptive_bit_b200 import (ERR_UNSUPPORTED_SHAPE, GrinqhError, lib,
                                     grinqh_decode_gemv_noalloc)
from input_adaptive_bit_b200.layer import GrinqhLinear

REL, ABS = 1e-3, 1e-6  # the tolerance of the parity tests


def test_rejects_shapes_beyond_its_scratch():
    # host-side check, no launch: d_in above the fixed scratch's limit
    status = lib().grinqh_decode_gemv_noalloc(1 << 40, 1 << 40, 1 << 40, 1 << 40, 1 << 40, None,
                                              32768 + 128, 4096, 8, 1 << 40, None)
    assert status == ERR_UNSUPPORTED_SHAPE
    assert "32768" in lib().grinqh_last_error().decode()


@pytest.mark.gpu
def test_matches_the_workspace_entry_points_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    g = np.random.default_rng(2024)
    d_in, d_out = 2048, 3072
    W = synth.gaussian_weights(g, d_in, d_out)
    q, s, z = synth.rtn_quantize(W, 8)
    lin = GrinqhLinear(q, s, z, 8)
    planes_ref = oracle.pack(q, 8)
    y_noalloc = torch.empty(d_out, dtype=torch.float32, device="cuda")
    for call in range(2):
        x = synth.activations(np.random.default_rng(call), d_in)
        theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), synth.level_fractions(3.0))
        xd = torch.from_numpy(x).cuda()
        td = torch.from_numpy(theta).cuda()
        y_ref = lin(xd, td).clone()  # grinqh_assign + grinqh_gemv with a caller workspace
        y_noalloc.fill_(float("nan"))
        grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8,
                                   y_noalloc)
        torch.cuda.synchronize()
        a, b = y_noalloc.cpu().numpy(), y_ref.cpu().numpy()
        b_host = oracle.assign(x, theta, 8)
        _, bound = oracle.gemv(planes_ref, s, z, x, b_host, 8, threads=oracle.max_threads())
        assert np.isfinite(a).all()
        assert (np.abs(a - b) <= REL * bound + ABS).all(), f"call {call} differs"


@pytest.mark.gpu
@pytest.mark.parametrize("b_max", [4, 6])
def test_smaller_base_widths(b_max):
    assert torch.cuda.is_available()
    g = np.random.default_rng(77 + b_max)
    d_in, d_out = 1024, 2048
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    lin = GrinqhLinear(q, s, z, b_max)
    x = synth.activations(g, d_in)
    fr = np.full(b_max // 2 + 1, 1.0 / (b_max // 2 + 1))
    theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), fr)
    y = torch.full((d_out,), float("nan"), dtype=torch.float32, device="cuda")
    grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, torch.from_numpy(x).cuda(),
                               torch.from_numpy(theta).cuda(), None, d_in, d_out, b_max, y)
    torch.cuda.synchronize()
    b_host = oracle.assign(x, theta, b_max)
    y_ref, bound = oracle.gemv(oracle.pack(q, b_max), s, z, x, b_host, b_max,
                               threads=oracle.max_threads())
    a = y.cpu().numpy()
    assert (np.abs(a - y_ref) <= REL * bound + ABS).all()
