"""grinqh_decode_gemv_noalloc: the decode GEMV for callers that cannot allocate
device memory (a host framework that owns all device memory and only lends
its plug-ins streams and tensors, or a path that must never reach the
allocator).  It must give the same y as the workspace-based entry points and
as the oracle, keep its device errors until they are read, and allocate
nothing.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from input_adaptive_bit_b200 import (ERR_DEVICE, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE,
                                     GrinqhError, grinqh_decode_gemv_noalloc,
                                     grinqh_noalloc_check_device_error, grinqh_noalloc_scratch, lib)
from input_adaptive_bit_b200.layer import GrinqhLinear

REL, ABS = 1e-3, 1e-6  # the tolerance of the parity tests
FAKE = 1 << 40         # never dereferenced: the host checks fail first


def test_rejects_shapes_beyond_its_limit():
    # host-side check, no launch: d_in above the decode kernel's limit
    status = lib().grinqh_decode_gemv_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                              65536 + 128, 4096, 8, FAKE, None)
    assert status == ERR_UNSUPPORTED_SHAPE
    assert "65536" in lib().grinqh_last_error().decode()


def test_checks_arguments_before_queueing_anything():
    # a NULL x fails the pointer check (before the scratch is looked up or cleared)
    status = lib().grinqh_decode_gemv_noalloc(FAKE, FAKE, FAKE, None, FAKE, None,
                                              4096, 4096, 8, FAKE, None)
    assert status == ERR_INVALID_ARG
    assert "x" in lib().grinqh_last_error().decode()
    assert lib().grinqh_noalloc_scratch(None, None) == ERR_INVALID_ARG


def _within(y, y_ref, bound):
    return bool(np.isfinite(y).all() and (np.abs(y - y_ref) <= REL * bound + ABS).all())


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
        y_ws = lin(xd, td).clone()  # grinqh_assign + grinqh_gemv with a caller workspace
        y_noalloc.fill_(float("nan"))
        grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8,
                                   y_noalloc)
        torch.cuda.synchronize()
        a, b = y_noalloc.cpu().numpy(), y_ws.cpu().numpy()
        b_host = oracle.assign(x, theta, 8)
        y_ref, bound = oracle.gemv(planes_ref, s, z, x, b_host, 8, threads=oracle.max_threads())
        assert _within(a, b, bound), f"call {call}: differs from the workspace entry points"
        assert _within(a, y_ref, bound), f"call {call}: differs from the oracle"
    grinqh_noalloc_check_device_error()  # a correct call records no device error


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
    assert _within(y.cpu().numpy(), y_ref, bound)


@pytest.mark.gpu
def test_largest_d_in_and_no_allocation():
    # the largest accepted d_in; the same call again allocates no device memory
    assert torch.cuda.is_available()
    g = np.random.default_rng(65536)
    d_in, d_out = 65536, 2048
    q = g.integers(0, 256, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    lin = GrinqhLinear(q, s, z, 8)
    x = synth.activations(g, d_in)
    theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), synth.level_fractions(3.0))
    xd, td = torch.from_numpy(x).cuda(), torch.from_numpy(theta).cuda()
    y = torch.full((d_out,), float("nan"), dtype=torch.float32, device="cuda")
    grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8, y)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8, y)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    outs = np.unique(np.concatenate([[0, d_out - 1], g.integers(0, d_out, 200)])).astype(np.int32)
    b_host = oracle.assign(x, theta, 8)
    y_ref, bound = oracle.gemv(oracle.pack(q, 8), s, z, x, b_host, 8, outs=outs,
                               threads=oracle.max_threads())
    assert _within(y.cpu().numpy()[outs], y_ref, bound)
    grinqh_noalloc_check_device_error()


class _DeviceWords:
    """A torch view of device memory the library owns (CUDA array interface)."""

    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"data": (ptr, False), "shape": (n,), "typestr": "<i4",
                                         "version": 3}


@pytest.mark.gpu
def test_device_error_word_is_kept_until_read():
    # An error code left in the scratch's error word (as a failed call would leave
    # it) survives further correct calls, is reported once by the check, and is
    # cleared by it.
    assert torch.cuda.is_available()
    g = np.random.default_rng(9)
    d_in, d_out = 1024, 1024
    q = g.integers(0, 256, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    lin = GrinqhLinear(q, s, z, 8)
    x = synth.activations(g, d_in)
    theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), synth.level_fractions(3.0))
    xd, td = torch.from_numpy(x).cuda(), torch.from_numpy(theta).cuda()
    y = torch.empty(d_out, dtype=torch.float32, device="cuda")
    grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8, y)
    grinqh_noalloc_check_device_error()
    ptr, nbytes = grinqh_noalloc_scratch()
    assert ptr != 0 and 1 << 20 <= nbytes <= 2 << 20
    err = torch.as_tensor(_DeviceWords(ptr, 1), device="cuda")
    err.fill_(3)
    for _ in range(2):
        grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8, y)
    torch.cuda.synchronize()
    with pytest.raises(GrinqhError) as e:
        grinqh_noalloc_check_device_error()
    assert e.value.status == ERR_DEVICE and "code 3" in str(e.value)
    grinqh_noalloc_check_device_error()  # cleared by the check
    b_host = oracle.assign(x, theta, 8)
    y_ref, bound = oracle.gemv(oracle.pack(q, 8), s, z, x, b_host, 8, threads=oracle.max_threads())
    assert _within(y.cpu().numpy(), y_ref, bound)


@pytest.mark.gpu
def test_partial_word_left_nonzero_is_reported_and_cleared():
    # A split-K partial word left non-zero in the fixed array (as a failed call could
    # leave it) is found when the first CTA publishes over it: the call records
    # device error 3, the check reports it and clears the array, and the next call
    # is right and reports nothing.
    assert torch.cuda.is_available()
    g = np.random.default_rng(11)
    d_in, d_out = 1024, 1024
    q = g.integers(0, 256, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    lin = GrinqhLinear(q, s, z, 8)
    x = synth.activations(g, d_in)
    theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), synth.level_fractions(3.0))
    xd, td = torch.from_numpy(x).cuda(), torch.from_numpy(theta).cuda()
    y = torch.empty(d_out, dtype=torch.float32, device="cuda")
    grinqh_noalloc_check_device_error()  # start from a clean array
    ptr, nbytes = grinqh_noalloc_scratch()
    words = torch.as_tensor(_DeviceWords(ptr, nbytes // 4), device="cuda")
    words[64].fill_(0x3f800001)  # the first partial word of CTA 0 (after the 256-byte header)
    grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8, y)
    torch.cuda.synchronize()
    with pytest.raises(GrinqhError) as e:
        grinqh_noalloc_check_device_error()
    assert e.value.status == ERR_DEVICE and "code 3" in str(e.value)
    assert not words.any()  # the check cleared the whole array
    grinqh_decode_gemv_noalloc(lin.planes, lin.s, lin.z, xd, td, None, d_in, d_out, 8, y)
    torch.cuda.synchronize()
    grinqh_noalloc_check_device_error()
    b_host = oracle.assign(x, theta, 8)
    y_ref, bound = oracle.gemv(oracle.pack(q, 8), s, z, x, b_host, 8, threads=oracle.max_threads())
    assert _within(y.cpu().numpy(), y_ref, bound)
    assert not words.any()  # a completed call leaves its partial words at zero
