"""Pins of the CPU oracle against things other than itself (CPU only).

Each pin is a value worked by hand from the GRINQH notes' formulas (fixtures
under tests/golden/), a closed form, an invariant, a special case that reduces
to a library routine, or brute force on a tiny input.  They are chosen so that
a plausible slip in the oracle -- a dropped phi, a wrong plane order, a
transposed index, a sign -- fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle

B_MAXES = (2, 4, 6, 8)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---- fp16 decoding -------------------------------------------------------------

def test_f16_decode_exhaustive_matches_numpy():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    # signed zero is kept
    assert np.signbit(oracle.f16_to_f64(0x8000))


# ---- phi (Key design 3) --------------------------------------------------------

@pytest.mark.parametrize("b_max,expected", [
    (8, [32.0, 8.0, 2.0, 0.0]),
    (6, [8.0, 2.0, 0.0]),
    (4, [2.0, 0.0]),
    (2, [0.0]),
])
def test_phi_default_closed_form(b_max, expected):
    # phi_b = 2^(b_max - b - 1) for b < b_max, 0 at full width
    assert list(oracle.phi_default(b_max)[1:]) == expected


# ---- hand-worked fixtures -------------------------------------------------------

def test_reconstruct_hand_worked_q182(golden_dir):
    g = _load(golden_dir, "reconstruct_q182.json")
    b_max = g["b_max"]
    q = np.full((128, 16), 0, np.uint8)
    q[5, 7] = g["q"]
    planes = oracle.pack(q, b_max)
    # the four plane slices, most significant first
    sl = [int((planes[5, p, 0] >> (2 * 7)) & 3) for p in range(4)]
    assert sl == g["planes_msb_first"]
    s = np.full((1, 16), g["s"], np.float16)
    z = np.full((1, 16), g["z"], np.float16)
    phi = oracle.phi_default(b_max)
    for row in g["rows"]:
        assert oracle.truncated_code(planes, 16, b_max, 5, 7, row["b"]) == row["Q"]
        assert phi[row["b"] // 2] == row["phi"]
        assert oracle.reconstruct(planes, s, z, phi, 16, b_max, 5, 7, row["b"]) == row["w_hat"]


def test_pack_hand_worked_words(golden_dir):
    g = _load(golden_dir, "pack_words.json")
    for case in g["cases"]:
        q = np.array(case["codes"], np.uint8).reshape(1, 16)
        planes = oracle.pack(q, g["b_max"])
        assert [int(w) for w in planes[0, :, 0]] == case["words_by_plane"], case["what"]
        assert (oracle.unpack(planes, 16, g["b_max"]) == q).all()


def test_assign_hand_worked(golden_dir):
    g = _load(golden_dir, "assign_cases.json")
    x = np.array([float(v) for v in g["x"]], np.float32).astype(np.float16)
    b = oracle.assign(x, np.array(g["theta"], np.float32), g["b_max"])
    assert list(b) == g["b"]


# ---- assignment -----------------------------------------------------------------

def test_assign_ties_take_higher_level_and_equal_thresholds_skip_a_level():
    theta = np.array([0.5, 1.0, 1.0, 2.0], np.float32)  # two equal thresholds
    x = np.array([0.5, 0.75, 1.0, 1.5, 2.0], np.float16)
    b = oracle.assign(x, theta, 8)
    assert list(b) == [2, 2, 6, 6, 8]  # b = 4 is never produced


def test_assign_scale_invariance():
    g = np.random.default_rng(1)
    x = g.standard_normal(4096)
    x = (np.sign(x) * np.maximum(np.abs(x), 0.01)).astype(np.float16)  # stay clear of subnormals
    theta = np.array([0.2, 0.7, 1.3, 2.1], np.float32)
    b = oracle.assign(x, theta, 8)
    for k in (-3, 2, 4):
        xs = (x.astype(np.float32) * 2.0 ** k).astype(np.float16)
        assert (xs.astype(np.float32) == x.astype(np.float32) * 2.0 ** k).all()  # exact in fp16
        assert (oracle.assign(xs, theta * np.float32(2.0 ** k), 8) == b).all()


def test_assign_uniform_and_infinite_thresholds():
    x = np.random.default_rng(2).standard_normal(256).astype(np.float16)
    for b_max in B_MAXES:
        P = b_max // 2
        for lvl in range(P + 1):
            theta = np.full(P, np.inf, np.float32)
            theta[:lvl] = 0.0
            assert (oracle.assign(x, theta, b_max) == 2 * lvl).all()


# ---- lists ----------------------------------------------------------------------

@pytest.mark.parametrize("b_max", B_MAXES)
def test_lists_ascending_nested_and_exact_membership(b_max):
    g = np.random.default_rng(3)
    P = b_max // 2
    b = (2 * g.integers(0, P + 1, size=1000)).astype(np.uint8)
    lists, counts = oracle.lists(b, b_max)
    prev = None
    for p in range(P):
        lp = lists[p, :counts[p]]
        assert (np.diff(lp) > 0).all()
        assert set(lp.tolist()) == {i for i in range(1000) if b[i] > 2 * p}
        assert (lists[p, counts[p]:] == -1).all()  # untouched past the count
        if prev is not None:
            assert set(lp.tolist()) <= set(prev.tolist())
        prev = lp


# ---- packing --------------------------------------------------------------------

@pytest.mark.parametrize("b_max", B_MAXES)
def test_pack_unpack_round_trip(b_max):
    g = np.random.default_rng(4)
    q = g.integers(0, 1 << b_max, size=(256, 96), dtype=np.uint8)
    q[0] = 0
    q[1] = (1 << b_max) - 1
    planes = oracle.pack(q, b_max)
    assert planes.shape == (256, b_max // 2, 6)
    assert (oracle.unpack(planes, 96, b_max) == q).all()


@pytest.mark.parametrize("b_max", B_MAXES)
def test_pack_single_bit_lands_where_the_layout_says(b_max):
    # Bit k of code (i, o) must set exactly bit 2*(o % 16) + (k % 2) of the word
    # (i, plane P-1-k//2, o//16) and nothing else: catches a swapped plane order,
    # a transposed row/word index or a wrong field position.
    P = b_max // 2
    d_in, d_out = 3, 48
    for i in range(d_in):
        for o in range(0, d_out, 7):
            for k in range(b_max):
                q = np.zeros((d_in, d_out), np.uint8)
                q[i, o] = 1 << k
                planes = oracle.pack(q, b_max)
                nz = np.argwhere(planes != 0)
                assert nz.tolist() == [[i, P - 1 - k // 2, o // 16]]
                assert int(planes[i, P - 1 - k // 2, o // 16]) == 1 << (2 * (o % 16) + k % 2)


# ---- truncation and the midpoint bias (Key design 3) ---------------------------

@pytest.mark.parametrize("b_max", B_MAXES)
def test_truncated_code_is_floor_to_multiple_and_full_width_is_exact(b_max):
    # every code of the width, in one row
    codes = np.arange(1 << b_max, dtype=np.uint8)
    d_out = max(16, len(codes))
    q = np.zeros((1, d_out), np.uint8)
    q[0, :len(codes)] = codes
    planes = oracle.pack(q, b_max)
    for b in range(2, b_max + 1, 2):
        d = b_max - b
        for c in codes:
            Q = oracle.truncated_code(planes, d_out, b_max, 0, int(c), b)
            assert Q == (int(c) >> d) << d  # low d bits cleared
    for c in codes:
        assert oracle.truncated_code(planes, d_out, b_max, 0, int(c), b_max) == int(c)


@pytest.mark.parametrize("b_max", B_MAXES)
def test_bias_closed_forms_exhaustive(b_max):
    """Over uniform codes: floor truncation has mean error -(2^d - 1)/2; with the
    page's phi the reconstruction sits at the midpoint of its cell, mean error
    +1/2 (zero against the cell-centred value q + 1/2); full width is exact."""
    codes = np.arange(1 << b_max)
    d_out = max(16, len(codes))
    q = np.zeros((1, d_out), np.uint8)
    q[0, :len(codes)] = codes
    planes = oracle.pack(q, b_max)
    phi = oracle.phi_default(b_max)
    for b in range(2, b_max + 1, 2):
        d = b_max - b
        Q = np.array([oracle.truncated_code(planes, d_out, b_max, 0, int(c), b) for c in codes])
        if d >= 1:
            assert (Q - codes).mean() == -(2 ** d - 1) / 2
            assert (Q + phi[b // 2] - codes).mean() == 0.5
            assert (Q + phi[b // 2] - (codes + 0.5)).mean() == 0.0
        else:
            assert (Q == codes).all() and phi[b // 2] == 0.0


# ---- the GEMV -------------------------------------------------------------------

def _tiny_case(seed, d_in=256, d_out=48, b_max=8):
    g = np.random.default_rng(seed)
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    G = d_in // 128
    s = (g.uniform(0.001, 0.01, size=(G, d_out))).astype(np.float16)
    z = (g.uniform(-0.5, 0.0, size=(G, d_out))).astype(np.float16)
    x = g.standard_normal(d_in).astype(np.float16)
    return q, s, z, x


def _mask_closed_form_what(q, s, z, b, b_max, phi):
    """w_hat from the integer mask (not from the planes): s*((q>>d)<<d + phi_b) + z."""
    d_in, d_out = q.shape
    W = np.zeros((d_in, d_out))
    for i in range(d_in):
        if b[i] == 0:
            continue
        d = b_max - int(b[i])
        Q = ((q[i].astype(np.int64) >> d) << d).astype(np.float64)
        g = i // 128
        W[i] = s[g].astype(np.float64) * (Q + phi[b[i] // 2]) + z[g].astype(np.float64)
    return W


@pytest.mark.parametrize("b_max", B_MAXES)
def test_gemv_full_width_is_the_textbook_dequant_matvec(b_max):
    q, s, z, x = _tiny_case(5, b_max=b_max)
    planes = oracle.pack(q, b_max)
    b = np.full(q.shape[0], b_max, np.uint8)
    y, _ = oracle.gemv(planes, s, z, x, b, b_max)
    G = q.shape[0] // 128
    deq = (np.repeat(s.astype(np.float64), 128, axis=0) * q
           + np.repeat(z.astype(np.float64), 128, axis=0))
    ref = x.astype(np.float64) @ deq  # library matvec
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert G >= 1


def test_gemv_all_rows_skipped_gives_exact_zero():
    q, s, z, x = _tiny_case(6)
    planes = oracle.pack(q, 8)
    b = oracle.assign(x, np.full(4, np.inf, np.float32), 8)
    assert (b == 0).all()
    y, bound = oracle.gemv(planes, s, z, x, b, 8)
    assert (y == 0).all() and (bound == 0).all()


def test_gemv_ignores_x_of_skipped_rows():
    q, s, z, x = _tiny_case(7)
    planes = oracle.pack(q, 8)
    theta = np.array([0.5, 1.0, 1.5, 2.0], np.float32)
    b = oracle.assign(x, theta, 8)
    assert (b == 0).any() and (b > 0).any()
    y1, _ = oracle.gemv(planes, s, z, x, b, 8)
    x2 = x.copy()
    x2[b == 0] = np.float16(1234.0)
    y2, _ = oracle.gemv(planes, s, z, x2, b, 8)
    assert (y1 == y2).all()


@pytest.mark.parametrize("b_max", B_MAXES)
def test_gemv_one_hot_recovers_a_row(b_max):
    q, s, z, _ = _tiny_case(8, b_max=b_max)
    planes = oracle.pack(q, b_max)
    phi = oracle.phi_default(b_max)
    for i, bw in [(3, 2), (130, b_max), (77, b_max - 2 if b_max > 2 else 2)]:
        x = np.zeros(q.shape[0], np.float16)
        x[i] = 1.0
        b = np.zeros(q.shape[0], np.uint8)
        b[i] = bw
        y, bound = oracle.gemv(planes, s, z, x, b, b_max)
        row = _mask_closed_form_what(q, s, z, b, b_max, phi)[i]
        assert (y == row).all()
        assert (bound == np.abs(row)).all()


def test_gemv_scales_exactly_with_x():
    q, s, z, x = _tiny_case(9)
    planes = oracle.pack(q, 8)
    theta = np.array([0.3, 0.8, 1.2, 1.9], np.float32)
    b = oracle.assign(x, theta, 8)
    y, _ = oracle.gemv(planes, s, z, x, b, 8)
    for k in (-2, 3):
        xs = (x.astype(np.float32) * 2.0 ** k).astype(np.float16)
        bs = oracle.assign(xs, theta * np.float32(2.0 ** k), 8)
        assert (bs == b).all()
        ys, _ = oracle.gemv(planes, s, z, xs, bs, 8)
        assert (ys == y * 2.0 ** k).all()


@pytest.mark.parametrize("b_max", B_MAXES)
def test_gemv_brute_force_tiny_all_level_patterns(b_max):
    # d_in = 128, d_out = 16; every row cycles through every level
    g = np.random.default_rng(10 + b_max)
    P = b_max // 2
    q = g.integers(0, 1 << b_max, size=(128, 16), dtype=np.uint8)
    s = g.uniform(0.001, 0.02, size=(1, 16)).astype(np.float16)
    z = g.uniform(-0.3, 0.1, size=(1, 16)).astype(np.float16)
    x = g.standard_normal(128).astype(np.float16)
    planes = oracle.pack(q, b_max)
    phi = oracle.phi_default(b_max)
    for shift in range(P + 1):
        b = (2 * ((np.arange(128) + shift) % (P + 1))).astype(np.uint8)
        y, bound = oracle.gemv(planes, s, z, x, b, b_max)
        W = _mask_closed_form_what(q, s, z, b, b_max, phi)
        xf = x.astype(np.float64)
        ref = np.array([sum(xf[i] * W[i, o] for i in range(128)) for o in range(16)])
        ref_b = np.abs(xf) @ np.abs(W)
        np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(bound, ref_b, rtol=1e-13, atol=1e-13)


def test_gemv_explicit_phi_table_is_used():
    # phi' = (2^d - 1)/2 makes E[Q + phi' - q] = 0 against the integer code
    q, s, z, x = _tiny_case(11, d_in=128, d_out=16)
    planes = oracle.pack(q, 8)
    b = np.full(128, 4, np.uint8)
    phi_alt = np.array([0.0, 31.5, 7.5, 1.5, 0.0])
    y, _ = oracle.gemv(planes, s, z, x, b, 8, phi=phi_alt)
    W = _mask_closed_form_what(q, s, z, b, 8, phi_alt)
    np.testing.assert_allclose(y, x.astype(np.float64) @ W, rtol=1e-12, atol=1e-12)


def test_gemv_sampled_outputs_match_full():
    q, s, z, x = _tiny_case(12, d_in=384, d_out=64)
    planes = oracle.pack(q, 8)
    b = oracle.assign(x, np.array([0.4, 0.9, 1.4, 2.2], np.float32), 8)
    y, bd = oracle.gemv(planes, s, z, x, b, 8, threads=3)
    outs = np.array([63, 0, 17, 17, 40], np.int32)
    ys, bs = oracle.gemv(planes, s, z, x, b, 8, outs=outs)
    assert (ys == y[outs]).all() and (bs == bd[outs]).all()


def test_gemv_nonfinite_input_poisons_every_output_and_nan_is_skipped():
    q, s, z, x = _tiny_case(13, d_in=128, d_out=16)
    planes = oracle.pack(q, 8)
    theta = np.array([0.5, 1.0, 1.5, 2.0], np.float32)
    xn = x.copy()
    xn[3] = np.float16(np.nan)
    b = oracle.assign(xn, theta, 8)
    assert b[3] == 0
    y, _ = oracle.gemv(planes, s, z, xn, b, 8)
    assert np.isfinite(y).all()
    xi = x.copy()
    xi[3] = np.float16(np.inf)
    b = oracle.assign(xi, theta, 8)
    assert b[3] == 8
    y, bound = oracle.gemv(planes, s, z, xi, b, 8)
    assert (~np.isfinite(y)).all()
    assert oracle.within_tolerance(np.full(16, np.nan), y, bound).all()
    assert not oracle.within_tolerance(np.zeros(16), y, bound).any()


# ---- dense 4-bit comparator ----------------------------------------------------

def test_dense4_hand_worked_and_round_trip():
    q4 = np.array([[0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15]], np.uint8)
    w4 = oracle.pack_dense4(q4)
    # nibble t of word j = output 8j + t, least significant first
    assert [int(w) for w in w4[0]] == [0x76543210, 0xFEDCBA98]
    g = np.random.default_rng(14)
    q4 = g.integers(0, 16, size=(256, 64), dtype=np.uint8)
    assert (oracle.unpack_dense4(oracle.pack_dense4(q4), 64) == q4).all()


def test_dense4_gemv_is_the_textbook_dequant_matvec():
    g = np.random.default_rng(15)
    q4 = g.integers(0, 16, size=(256, 32), dtype=np.uint8)
    s = g.uniform(0.001, 0.1, size=(2, 32)).astype(np.float16)
    z = g.uniform(-1, 0, size=(2, 32)).astype(np.float16)
    x = g.standard_normal(256).astype(np.float16)
    y, bound = oracle.gemv_dense4(oracle.pack_dense4(q4), s, z, x)
    deq = (np.repeat(s.astype(np.float64), 128, axis=0) * q4
           + np.repeat(z.astype(np.float64), 128, axis=0))
    np.testing.assert_allclose(y, x.astype(np.float64) @ deq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(bound, np.abs(x.astype(np.float64)) @ np.abs(deq), rtol=1e-12)


# ---- the acceptance check itself ------------------------------------------------

def test_within_tolerance_semantics():
    y_ref = np.array([1.0, -2.0, 0.0])
    bound = np.array([10.0, 10.0, 0.0])
    assert oracle.within_tolerance(y_ref + [0.0099, -0.0099, 9e-7], y_ref, bound).all()
    assert not oracle.within_tolerance(y_ref + [0.0101, 0, 0], y_ref, bound)[0]
    assert not oracle.within_tolerance(y_ref + [0, 0, 2e-6], y_ref, bound)[2]
