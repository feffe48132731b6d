"""The C-ABI library loads and exports what include/grinqh.h declares, and its
host-side argument checks answer with the documented status codes (CPU only:
every call here returns before touching a GPU)."""
import ctypes
import os
import re

import pytest

import input_adaptive_bit_b200 as gq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "grinqh.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(grinqh_\w+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for n in ("grinqh_pack", "grinqh_unpack", "grinqh_assign", "grinqh_gemv",
              "grinqh_workspace_bytes", "grinqh_gemv_dense4"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(gq.lib_path)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(gq.EXPORTS)


def test_version():
    assert gq.grinqh_version() == 1000


@pytest.mark.parametrize("d_in,d_out,b_max,ok", [
    (4096, 4096, 8, True), (128, 16, 2, True), (256, 48, 6, True),
    (100, 4096, 8, False), (4096, 40, 8, False), (4096, 4096, 5, False),
    (0, 16, 8, False), ((1 << 24) + 128, 16, 8, False), (128, 8, 8, False),
])
def test_workspace_bytes(d_in, d_out, b_max, ok):
    n = gq.grinqh_workspace_bytes(d_in, d_out, b_max)
    assert (n > 0) == ok
    if ok:
        P = b_max // 2
        assert n >= 256 + 4 * (1 << 15) + 8 * d_in * P and n % 256 == 0


def test_workspace_grows_with_shape():
    assert gq.grinqh_workspace_bytes(8192, 4096, 8) > gq.grinqh_workspace_bytes(4096, 4096, 8)
    assert gq.grinqh_workspace_bytes(4096, 4096, 8) > gq.grinqh_workspace_bytes(4096, 4096, 4)


FAKE = 1 << 40  # never dereferenced: every case below fails a host check first


def _status(fn, *args):
    return getattr(gq.lib(), fn)(*args)


def test_pack_argument_checks():
    assert _status("grinqh_pack", None, 128, 16, 8, FAKE, None) == gq.ERR_INVALID_ARG
    assert _status("grinqh_pack", FAKE, 128, 16, 7, FAKE, None) == gq.ERR_INVALID_ARG
    assert _status("grinqh_pack", FAKE, 120, 16, 8, FAKE, None) == gq.ERR_UNSUPPORTED_SHAPE
    assert _status("grinqh_pack", FAKE, 128, 24, 8, FAKE, None) == gq.ERR_UNSUPPORTED_SHAPE
    assert _status("grinqh_pack", FAKE + 8, 128, 16, 8, FAKE, None) == gq.ERR_INVALID_ARG
    assert "aligned" in gq.grinqh_last_error()


def test_assign_argument_checks():
    args = [FAKE, FAKE, 256, 8, None, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None]
    for k in (0, 1, 5, 6, 7, 8, 9):
        bad = list(args)
        bad[k] = None
        assert _status("grinqh_assign", *bad) == gq.ERR_INVALID_ARG, k
    small = list(args)
    small[10] = 1024
    assert _status("grinqh_assign", *small) == gq.ERR_WORKSPACE_TOO_SMALL
    bad = list(args)
    bad[9] = FAKE + 16  # workspace must be 256-byte aligned
    assert _status("grinqh_assign", *bad) == gq.ERR_INVALID_ARG


def test_gemv_argument_checks():
    need = gq.grinqh_workspace_bytes(256, 64, 8)
    args = [FAKE, FAKE, FAKE, FAKE, 256, 64, 8, FAKE, FAKE, need, None]
    for k in (0, 1, 2, 3, 7, 8):
        bad = list(args)
        bad[k] = None
        assert _status("grinqh_gemv", *bad) == gq.ERR_INVALID_ARG, k
    small = list(args)
    small[9] = need - 1
    assert _status("grinqh_gemv", *small) == gq.ERR_WORKSPACE_TOO_SMALL
    shape = list(args)
    shape[5] = 20
    assert _status("grinqh_gemv", *shape) == gq.ERR_UNSUPPORTED_SHAPE
    bmax = list(args)
    bmax[6] = 3
    assert _status("grinqh_gemv", *bmax) == gq.ERR_INVALID_ARG


def test_decode_argument_checks():
    need = gq.grinqh_workspace_bytes(256, 64, 8)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, None, 256, 64, 8, FAKE, None, None, None, None, FAKE,
            need, None]
    for k in (0, 1, 2, 3, 4, 9, 14):
        bad = list(args)
        bad[k] = None
        assert _status("grinqh_decode_gemv", *bad) == gq.ERR_INVALID_ARG, k
    small = list(args)
    small[15] = need - 1
    assert _status("grinqh_decode_gemv", *small) == gq.ERR_WORKSPACE_TOO_SMALL
    big = list(args)
    big[6] = 65536 + 128
    big[15] = 1 << 40
    assert _status("grinqh_decode_gemv", *big) == gq.ERR_UNSUPPORTED_SHAPE
    assert "65536" in gq.grinqh_last_error()
    unaligned_x = list(args)
    unaligned_x[3] = FAKE + 8
    assert _status("grinqh_decode_gemv", *unaligned_x) == gq.ERR_INVALID_ARG


def test_group_argument_checks():
    need = gq.grinqh_group_workspace_bytes()
    assert need >= 256 + 128 * 1024
    lin = gq.GrinqhLinearDesc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 256, 64, 8, FAKE)
    arr = (gq.GrinqhLinearDesc * 5)(*([lin] * 5))
    p = ctypes.cast(arr, ctypes.c_void_p)
    lib = gq.lib()
    assert lib.grinqh_decode_gemv_group(0, p, FAKE, need, None) == gq.ERR_INVALID_ARG
    assert lib.grinqh_decode_gemv_group(gq.MAX_GROUP + 1, p, FAKE, need, None) == gq.ERR_INVALID_ARG
    assert lib.grinqh_decode_gemv_group(2, None, FAKE, need, None) == gq.ERR_INVALID_ARG
    assert lib.grinqh_decode_gemv_group(2, p, FAKE, need - 1, None) == gq.ERR_WORKSPACE_TOO_SMALL
    assert lib.grinqh_decode_gemv_group(2, p, None, need, None) == gq.ERR_INVALID_ARG
    arr[1].y = None
    assert lib.grinqh_decode_gemv_group(2, p, FAKE, need, None) == gq.ERR_INVALID_ARG
    arr[1].y = FAKE
    arr[1].d_in = 65536 + 128
    assert lib.grinqh_decode_gemv_group(2, p, FAKE, need, None) == gq.ERR_UNSUPPORTED_SHAPE
    assert "65536" in gq.grinqh_last_error()
    arr[1].d_in = 256
    arr[1].b_max = 5
    assert lib.grinqh_decode_gemv_group(2, p, FAKE, need, None) == gq.ERR_INVALID_ARG


def test_dense4_argument_checks():
    need = gq.grinqh_dense4_workspace_bytes(256, 64)
    assert need > 0
    args = [FAKE, FAKE, FAKE, FAKE, 256, 64, FAKE, FAKE, need, None]
    assert _status("grinqh_gemv_dense4", *args[:8], 0, None) == gq.ERR_WORKSPACE_TOO_SMALL
    bad = list(args)
    bad[3] = None
    assert _status("grinqh_gemv_dense4", *bad) == gq.ERR_INVALID_ARG
    assert _status("grinqh_pack_dense4", None, 256, 64, FAKE, None) == gq.ERR_INVALID_ARG


def test_python_binding_raises_with_message():
    with pytest.raises(gq.GrinqhError) as e:
        gq.grinqh_pack(0, 128, 16, 9, FAKE, stream=0)
    assert e.value.status == gq.ERR_INVALID_ARG and "b_max" in str(e.value)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(gq, "_lib", None)
    monkeypatch.setattr(gq, "lib_path", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        gq.grinqh_version()


def test_prefill_argument_checks():
    # planes, s, z, x, phi, T, d_in, d_out, b_max, y, ws, ws_bytes, stream
    ok = [FAKE, FAKE, FAKE, FAKE, None, 128, 4096, 4096, 8, FAKE, FAKE, 4096, None]
    for k in (0, 1, 2, 3, 9, 10):  # every required pointer, null or misaligned
        for bad_ptr in (None, FAKE + 2):
            bad = list(ok)
            bad[k] = bad_ptr
            assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_INVALID_ARG, (k, bad_ptr)
    bad = list(ok)
    bad[4] = FAKE + 2  # phi is fp32
    assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_INVALID_ARG
    for T in (0, -1, 65537):
        bad = list(ok)
        bad[5] = T
        assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_UNSUPPORTED_SHAPE, T
    bad = list(ok)
    bad[7] = 4096 + 16  # a multiple of 16 but not of the 128-output tile
    assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_UNSUPPORTED_SHAPE
    assert "128" in gq.lib().grinqh_last_error().decode()
    bad = list(ok)
    bad[6] = 4096 + 64  # d_in not a whole number of 128-row groups
    assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_UNSUPPORTED_SHAPE
    bad = list(ok)
    bad[8] = 5
    assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_INVALID_ARG
    bad = list(ok)
    bad[11] = gq.grinqh_prefill_workspace_bytes() - 1
    assert _status("grinqh_prefill_gemm", *bad) == gq.ERR_WORKSPACE_TOO_SMALL
    assert gq.grinqh_prefill_workspace_bytes() > 0
