"""GPU parity of the fused decode kernel (grinqh_decode_gemv) in the cases its
own work split creates: ranges spanning several rounds, more tiles than CTAs,
empty groups between active ones, the largest accepted d_in, fewer units than
CTAs, every split-K factor from 144 CTAs per tile down to one (with and
without cluster sums), the optional outputs (bit-exact with grinqh_assign, or
skipped), and a stale split-K counter reported as a device error while y
stays right."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import check_assign, check_y, run_layer, to_dev
from input_adaptive_bit_b200.layer import GrinqhLinear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def cheap_case(seed, d_in, d_out, b_max, fractions=None):
    """Uniform random codes and fp16 s/z (no RTN pass), synthetic x and Theta."""
    g = np.random.default_rng(seed)
    P = b_max // 2
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    x = synth.activations(g, d_in)
    fr = np.full(P + 1, 1.0 / (P + 1)) if fractions is None else np.asarray(fractions)
    theta = synth.quantile_thresholds(np.abs(x.astype(np.float32)), fr)
    return q, s, z, x, theta


def check_fused(q, s, z, x, theta, b_max, outs=None):
    lin, out = run_layer(q, s, z, x, theta, b_max, path="fused")
    b_ref = check_assign(out, x, theta, b_max)
    check_y(out, oracle.pack(q, b_max), s, z, x, b_ref, b_max, outs=outs)
    return lin, out


def test_optional_outputs_match_assign_bit_for_bit_or_are_skipped():
    q, s, z, x, theta = cheap_case(1, 2048, 3072, 8)
    lin = GrinqhLinear(q, s, z, 8)
    xd, th = to_dev(x), to_dev(theta)
    lin.assign(xd, th)
    torch.cuda.synchronize()
    ref = {k: getattr(lin, k).clone() for k in ("b", "lists", "counts", "grp_sums")}
    for k in ref:
        getattr(lin, k).fill_(0)
    y1 = lin.decode(xd, th).clone()
    torch.cuda.synchronize()
    assert torch.equal(lin.b, ref["b"]) and torch.equal(lin.counts, ref["counts"])
    n = ref["counts"].cpu().numpy()
    for p in range(4):
        assert torch.equal(lin.lists[p, :n[p]], ref["lists"][p, :n[p]])
    assert torch.equal(lin.grp_sums.view(torch.int32), ref["grp_sums"].view(torch.int32))
    # outputs skipped: nothing written, y identical
    for k in ref:
        getattr(lin, k).fill_(-3)
    y2 = lin.decode(xd, th, outputs=False)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert (lin.b == 253).all() and (lin.lists == -3).all() and (lin.counts == -3).all()
    assert (lin.grp_sums == -3).all()


def test_more_tiles_than_ctas_and_several_rounds_per_range():
    # d_out = 148 * 1024 + 16: 149 tiles (one CTA takes two), the last ragged and
    # not 16-byte aligned (d_out / 16 odd); 10 groups with ~3.25 planes per row
    # (~4200 units per tile) force rounds cut both by the 8-group window and by
    # the 2048-unit cap (the first window holds ~3300 units)
    d_in, d_out = 1280, 148 * 1024 + 16
    q, s, z, x, theta = cheap_case(2, d_in, d_out, 8, fractions=[0.05, 0.05, 0.1, 0.2, 0.6])
    outs = np.unique(np.concatenate([np.arange(0, 64), np.arange(d_out - 80, d_out),
                                     np.random.default_rng(0).integers(0, d_out, 200)]))
    check_fused(q, s, z, x, theta, 8, outs=outs.astype(np.int32))


@pytest.mark.parametrize("live", [[0, 31], [0, 7, 8, 20, 31], [5], [31]])
def test_empty_groups_between_active_ones(live):
    d_in, d_out = 4096, 2048
    q, s, z, x, theta = cheap_case(3, d_in, d_out, 8)
    keep = np.zeros(d_in, bool)
    for g in live:
        keep[128 * g:128 * (g + 1)] = True
    x = np.where(keep, x, np.float16(0.0)).astype(np.float16)
    theta = np.array([1e-3, 0.5, 1.0, 2.0], np.float32)
    check_fused(q, s, z, x, theta, 8)


def test_largest_accepted_d_in():
    q, s, z, x, theta = cheap_case(4, 65536, 64, 8)
    check_fused(q, s, z, x, theta, 8)


@pytest.mark.parametrize("n_active", [1, 3, 40])
def test_fewer_units_than_ctas(n_active):
    d_in, d_out = 1024, 4096
    q, s, z, x, _ = cheap_case(5, d_in, d_out, 8)
    g = np.random.default_rng(n_active)
    x = (g.standard_normal(d_in) * 0.01).astype(np.float16)
    idx = g.choice(d_in, n_active, replace=False)
    x[idx] = (g.standard_normal(n_active) + 4.0).astype(np.float16)
    theta = np.array([1.0, 2.0, 3.0, 100.0], np.float32)
    check_fused(q, s, z, x, theta, 8)


@pytest.mark.parametrize("b_max", [2, 4, 6])
def test_smaller_base_widths_on_wide_layers(b_max):
    q, s, z, x, theta = cheap_case(6, 2048, 5120, b_max)
    check_fused(q, s, z, x, theta, b_max)


def test_large_activations_use_a_scaled_b_column():
    # |x| * 4^(P-1) beyond the fp16 range: the kernel scales each group's column
    q, s, z, x, theta = cheap_case(7, 1024, 1024, 8)
    x = (x.astype(np.float32) * 900.0).clip(-65504, 65504).astype(np.float16)
    theta = theta * np.float32(900.0)
    check_fused(q, s, z, x, theta, 8)


@pytest.mark.parametrize("d_out", [1024, 2048, 48 * 1024, 72 * 1024, 144 * 1024])
def test_split_k_shares_every_ctas_per_tile(d_out):
    # one tile (every GEMV CTA takes a slice of the same 1024 outputs) down to one
    # CTA per tile: each CTA of a tile waits for the others and adds its share of
    # the partial sums; y must be the same on a second call (fixed order) and the
    # device error word must stay clear
    from input_adaptive_bit_b200 import grinqh_check_device_error
    d_in = 512
    q, s, z, x, theta = cheap_case(8, d_in, d_out, 8)
    rng = np.random.default_rng(d_out)
    outs = np.unique(np.concatenate([np.arange(0, 48), np.arange(d_out - 48, d_out),
                                     rng.integers(0, d_out, 300)])).astype(np.int32)
    lin, out = check_fused(q, s, z, x, theta, 8, outs=outs)
    y2 = lin.decode(to_dev(x), to_dev(theta), outputs=False)
    torch.cuda.synchronize()
    assert np.array_equal(y2.cpu().numpy().astype(np.float64), out["y"])
    grinqh_check_device_error(lin.ws)  # raises if a split-K wait gave up


# The fused decode's split-K partial words in a workspace of grinqh_workspace_bytes:
# after the 256-byte header and grinqh_gemv's arrival counters (one per 512-output
# tile of the largest d_out, 2^24 / 512 of them), one 1024-word partial per CTA.
DPARTIALS = 256 + (1 << 24) // 512 * 4


def test_split_k_reports_a_partial_word_left_nonzero():
    # A workspace whose split-K partial words were not left zeroed (the call requires
    # a zeroed workspace): the first CTA finds its partial's first word non-zero when
    # it publishes, and the call reports device error 3; the check clears the
    # workspace's split-K state, and the next call is right and reports nothing.
    from input_adaptive_bit_b200 import ERR_DEVICE, GrinqhError, grinqh_check_device_error
    q, s, z, x, theta = cheap_case(9, 512, 1024, 8)  # one tile: every GEMV CTA shares it
    lin = GrinqhLinear(q, s, z, 8)
    xd, th = to_dev(x), to_dev(theta)
    lin.ws[DPARTIALS:DPARTIALS + 4].view(torch.int32).fill_(0x3f800001)  # CTA 0's first word
    lin.decode(xd, th, outputs=False)
    torch.cuda.synchronize()
    with pytest.raises(GrinqhError) as err:
        grinqh_check_device_error(lin.ws)
    assert err.value.status == ERR_DEVICE and "code 3" in str(err.value)
    assert not lin.ws[:DPARTIALS + 148 * 4096].any()  # the check cleared the split-K state
    _, out = run_layer(None, None, None, x, theta, 8, lin=lin, path="fused")
    b_ref = check_assign(out, x, theta, 8)
    check_y(out, oracle.pack(q, 8), s, z, x, b_ref, 8)
    grinqh_check_device_error(lin.ws)
    assert not lin.ws[DPARTIALS:DPARTIALS + 256 * 4096].any()  # every partial word is back at zero


def test_y_is_right_while_other_work_holds_some_sms():
    # Other work holds a few SMs (single-thread kernels that sleep ~0.8 s on side
    # streams; the decode kernel's CTAs need a whole SM each, so those SMs are shut
    # to it).  The decode launch is cooperative: it starts once all of its CTAs fit,
    # so the split-K waits between the CTAs of a tile end and y is the oracle's, with
    # no device error.
    from input_adaptive_bit_b200 import grinqh_check_device_error
    q, s, z, x, theta = cheap_case(10, 1024, 4096, 8)  # 4 tiles, 36 CTAs each
    lin = GrinqhLinear(q, s, z, 8)
    xd, th = to_dev(x), to_dev(theta)
    y = torch.full((4096,), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    side = [torch.cuda.Stream() for _ in range(4)]
    for st in side:
        with torch.cuda.stream(st):
            torch.cuda._sleep(int(0.8 * 1.9e9))  # ~0.8 s of clock cycles, one thread
    time.sleep(0.05)  # the sleepers are resident first
    main = torch.cuda.Stream()
    with torch.cuda.stream(main):
        lin.decode(xd, th, y=y, outputs=False, stream=main)
    torch.cuda.synchronize()
    b_ref = oracle.assign(x, theta, 8)
    check_y({"y": y.cpu().numpy().astype(np.float64)}, oracle.pack(q, 8), s, z, x, b_ref, 8)
    grinqh_check_device_error(lin.ws)
    assert not lin.ws[DPARTIALS:DPARTIALS + 256 * 4096].any()  # every partial word is back at zero


@pytest.mark.parametrize("shapes", [
    [(2048, 2048, 8), (2048, 512, 8), (2048, 512, 8)],            # q, k, v of one layer
    [(1024, 4096, 8), (4096, 1024, 8)],                           # different d_in
    [(512, 1040, 6), (1024, 3072, 4), (256, 16, 2), (2048, 1024, 8)],  # mixed widths, a ragged unaligned layout
    [(1024, 2048, 8)],                                            # a group of one
    [(256, 150 * 1024 + 16, 8), (512, 1024, 8)],                  # more tiles than CTAs; a one-CTA tile
])
def test_grouped_launch_matches_the_oracle_per_linear(shapes):
    from input_adaptive_bit_b200 import (grinqh_check_device_error, grinqh_decode_gemv_group,
                                         grinqh_group_workspace_bytes)
    cases, lins = [], []
    for i, (d_in, d_out, b_max) in enumerate(shapes):
        q, s, z, x, theta = cheap_case(20 + i, d_in, d_out, b_max)
        lin = GrinqhLinear(q, s, z, b_max)
        xd, th = to_dev(x), to_dev(theta)
        y = torch.full((d_out,), float("nan"), dtype=torch.float32, device="cuda")
        cases.append((q, s, z, x, theta, b_max, lin, xd, th, y))
    nbytes = grinqh_group_workspace_bytes()
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for _ in range(2):  # twice: the split-K words must come back to zero
        grinqh_decode_gemv_group([(c[6].planes, c[6].s, c[6].z, c[7], c[8], None, c[6].d_in,
                                   c[6].d_out, c[5], c[9]) for c in cases], ws, nbytes)
        torch.cuda.synchronize()
        for q, s, z, x, theta, b_max, lin, xd, th, y in cases:
            out = {"y": y.cpu().numpy().astype(np.float64)}
            check_y(out, oracle.pack(q, b_max), s, z, x, oracle.assign(x, theta, b_max), b_max)
    grinqh_check_device_error(ws)
    assert not ws[256:].any()  # every split-K partial word is back at zero


def test_decode_group_helper_of_the_layer_module():
    from input_adaptive_bit_b200.layer import DecodeGroup
    cases = [cheap_case(30 + i, d_in, d_out, 8) for i, (d_in, d_out) in enumerate([(1024, 2048), (1024, 512)])]
    layers = [GrinqhLinear(q, s, z, 8) for q, s, z, _, _ in cases]
    ys = DecodeGroup(layers)([to_dev(c[3]) for c in cases], [to_dev(c[4]) for c in cases])
    torch.cuda.synchronize()
    for (q, s, z, x, theta), y in zip(cases, ys):
        out = {"y": y.cpu().numpy().astype(np.float64)}
        check_y(out, oracle.pack(q, 8), s, z, x, oracle.assign(x, theta, 8), 8)



def test_grouped_launch_with_an_explicit_phi_table():
    from input_adaptive_bit_b200 import grinqh_decode_gemv_group, grinqh_group_workspace_bytes
    q1, s1, z1, x1, th1 = cheap_case(40, 1024, 2048, 8)
    q2, s2, z2, x2, th2 = cheap_case(41, 512, 1024, 6)
    phi1 = np.array([0.0, 0.37, -1.25, 3.5, 0.0], np.float32)  # any table: levels 0..4
    l1, l2 = GrinqhLinear(q1, s1, z1, 8), GrinqhLinear(q2, s2, z2, 6)
    y1 = torch.empty(2048, dtype=torch.float32, device="cuda")
    y2 = torch.empty(1024, dtype=torch.float32, device="cuda")
    nbytes = grinqh_group_workspace_bytes()
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    grinqh_decode_gemv_group([(l1.planes, l1.s, l1.z, to_dev(x1), to_dev(th1), to_dev(phi1), 1024, 2048, 8, y1),
                              (l2.planes, l2.s, l2.z, to_dev(x2), to_dev(th2), None, 512, 1024, 6, y2)],
                             ws, nbytes)
    torch.cuda.synchronize()
    check_y({"y": y1.cpu().numpy().astype(np.float64)}, oracle.pack(q1, 8), s1, z1, x1,
            oracle.assign(x1, th1, 8), 8, phi=phi1)
    check_y({"y": y2.cpu().numpy().astype(np.float64)}, oracle.pack(q2, 6), s2, z2, x2,
            oracle.assign(x2, th2, 6), 6)
