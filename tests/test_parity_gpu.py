"""GPU <-> oracle parity of the decode path, through the C-ABI.

Bit-exact: planes, unpack(planes), b, the per-plane lists and counts.
Within |y - y_ref| <= 1e-3 * sum_i |w_hat_io||x_i| + 1e-6: y.
Every case runs on both paths: grinqh_assign + grinqh_gemv ("two") and the
fused single-kernel grinqh_decode_gemv ("fused").
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import (ABS, REL, check_assign, check_y, full_case_check, gpu_unpack,
                          planes_host, run_layer, to_dev)
from input_adaptive_bit_b200 import (ERR_DEVICE, GrinqhError, grinqh_check_device_error,
                                     grinqh_gemv)
from input_adaptive_bit_b200.layer import Dense4Linear, GrinqhLinear

pytestmark = pytest.mark.gpu
PATHS = ["two", "fused"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def random_case(seed, d_in, d_out, b_max, x_kind="normal", theta_kind="quantile"):
    g = np.random.default_rng(seed)
    P = b_max // 2
    W = synth.gaussian_weights(g, d_in, d_out)
    q, s, z = synth.rtn_quantize(W, b_max)
    x = synth.activations(g, d_in)
    if x_kind == "special":
        xf = x.astype(np.float32)
        idx = g.choice(d_in, size=min(d_in, 40), replace=False)
        specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 6e-8, -6e-8, 5.9e-5, 65504.0,
                             -65504.0], np.float32)
        xf[idx] = specials[np.arange(idx.size) % specials.size]
        x = xf.astype(np.float16)
    if theta_kind == "quantile":
        fr = np.full(P + 1, 1.0 / (P + 1))
        theta = synth.quantile_thresholds(np.abs(x[np.isfinite(x)].astype(np.float32)), fr)
    elif theta_kind == "ties":  # thresholds equal to input magnitudes, and equal thresholds
        a = np.sort(np.abs(x[np.isfinite(x)].astype(np.float32)))
        theta = np.array([a[len(a) // 4], a[len(a) // 4], a[len(a) // 2], a[3 * len(a) // 4]][:P],
                         np.float32)
    elif theta_kind == "zero":
        theta = np.zeros(P, np.float32)
    elif theta_kind == "inf":
        theta = np.full(P, np.inf, np.float32)
    elif theta_kind == "decreasing":
        theta = np.array([2.0, 1.0, 0.5, 0.25][:P], np.float32)
    elif theta_kind == "nan":
        theta = np.array([0.5, np.nan, 1.0, 2.0][:P], np.float32)
    else:
        raise ValueError(theta_kind)
    return synth.Case(synth.Linear("rand", d_in, d_out, b_max), q, s, z, x, theta)


# ---- the parity workload ----------------------------------------------------------

@pytest.mark.parametrize("path", PATHS)
def test_config0_parity_everything(path):
    case = synth.make_case(synth.config0()[0])
    lin, out = full_case_check(case, path=path)
    assert abs(oracle.effective_bits(out["b"]) - 3.3) < 0.05


@pytest.mark.parametrize("b_max", [2, 4, 6, 8])
@pytest.mark.parametrize("shape", [(128, 16), (256, 48), (384, 592), (1152, 1040), (2048, 512)])
@pytest.mark.parametrize("path", PATHS)
def test_random_shapes(b_max, shape, path):
    d_in, d_out = shape
    full_case_check(random_case(1000 * b_max + d_in + d_out, d_in, d_out, b_max), path=path)


@pytest.mark.parametrize("theta_kind", ["ties", "zero", "inf", "decreasing", "nan"])
@pytest.mark.parametrize("x_kind", ["normal", "special"])
@pytest.mark.parametrize("path", PATHS)
def test_adversarial_thresholds_and_inputs(theta_kind, x_kind, path):
    full_case_check(random_case(7, 1280, 1040, 8, x_kind=x_kind, theta_kind=theta_kind), path=path)


@pytest.mark.parametrize("path", PATHS)
def test_random_shape_sweep(path):
    g = np.random.default_rng(123)
    for k in range(12):
        d_in = 128 * int(g.integers(1, 9))
        d_out = 16 * int(g.integers(1, 65))
        b_max = int(g.choice([2, 4, 6, 8]))
        full_case_check(random_case(5000 + k, d_in, d_out, b_max), path=path)


@pytest.mark.parametrize("path", PATHS)
def test_all_rows_skipped_gives_exact_zeros(path):
    case = random_case(9, 1024, 2048, 8, theta_kind="inf")
    lin, out = run_layer(case.q, case.s, case.z, case.x, case.theta, 8, path=path)
    assert (out["b"] == 0).all() and (out["counts"] == 0).all()
    assert (out["y"] == 0.0).all() and not np.signbit(out["y"]).any()


@pytest.mark.parametrize("path", PATHS)
def test_explicit_phi_table(path):
    case = random_case(10, 1024, 1024, 8)
    phi = np.array([0.0, 31.5, 7.5, 1.5, 0.0], np.float32)
    full_case_check(case, phi=phi, path=path)


@pytest.mark.parametrize("path", PATHS)
def test_one_hot_rows_recover_the_reconstructed_row(path):
    # x = e_i, b_i = 8/6/4/2: y must be the reconstructed row s(Q+phi)+z up to a
    # few fp32 roundings of its terms
    case = random_case(11, 512, 1024, 8)
    lin = GrinqhLinear(case.q, case.s, case.z, 8)
    phi = oracle.phi_default(8)
    for i, lvl in [(0, 4), (130, 3), (257, 2), (511, 1)]:
        x = np.zeros(512, np.float16)
        x[i] = 1.0
        theta = np.array([0.5] * lvl + [np.inf] * (4 - lvl), np.float32)
        _, out = run_layer(None, None, None, x, theta, 8, lin=lin, path=path)
        b = 2 * lvl
        d = 8 - b
        Q = ((case.q[i].astype(np.int64) >> d) << d).astype(np.float64)
        g = i // 128
        row = case.s[g].astype(np.float64) * (Q + phi[lvl]) + case.z[g].astype(np.float64)
        mag = np.abs(case.s[g].astype(np.float64)) * (Q + phi[lvl]) + np.abs(case.z[g].astype(np.float64))
        assert (np.abs(out["y"] - row) <= 8 * 2.0 ** -24 * mag).all()
        assert oracle.within_tolerance(out["y"], row, np.abs(row), REL, ABS).all()


@pytest.mark.parametrize("path", PATHS)
def test_zeroing_skipped_inputs_changes_nothing(path):
    case = random_case(12, 1024, 1536, 8)
    lin, out1 = run_layer(case.q, case.s, case.z, case.x, case.theta, 8, path=path)
    x2 = case.x.copy()
    b = out1["b"]
    # |x| below theta_1 keeps b = 0 when scaled towards zero
    x2[b == 0] = (x2[b == 0].astype(np.float32) * 0.25).astype(np.float16)
    _, out2 = run_layer(None, None, None, x2, case.theta, 8, lin=lin, path=path)
    assert np.array_equal(out2["b"], b)
    assert np.array_equal(out1["y"], out2["y"])


@pytest.mark.parametrize("path", PATHS)
def test_deterministic_across_calls(path):
    case = random_case(13, 4096, 4096, 8)
    lin, out1 = run_layer(case.q, case.s, case.z, case.x, case.theta, 8, path=path)
    for _ in range(3):
        _, out2 = run_layer(None, None, None, case.x, case.theta, 8, lin=lin, path=path)
        assert np.array_equal(out1["y"], out2["y"])
        assert np.array_equal(out1["grp_sums"], out2["grp_sums"])


@pytest.mark.parametrize("path", PATHS)
def test_scaling_x_and_theta_by_power_of_two(path):
    case = random_case(14, 1024, 1024, 8)
    x = case.x.astype(np.float32)
    x = (np.sign(x) * np.maximum(np.abs(x), 0.01)).astype(np.float16)
    lin, out1 = run_layer(case.q, case.s, case.z, x, case.theta, 8, path=path)
    xs = (x.astype(np.float32) * 4).astype(np.float16)
    _, out2 = run_layer(None, None, None, xs, case.theta * np.float32(4), 8, lin=lin, path=path)
    assert np.array_equal(out1["b"], out2["b"])
    assert np.array_equal(out1["y"] * 4, out2["y"])


@pytest.mark.parametrize("path", PATHS)
def test_workspace_shared_by_layers_of_different_shapes(path):
    big = random_case(15, 2048, 4096, 8)
    small = random_case(16, 512, 1024, 6)
    lin_b = GrinqhLinear(big.q, big.s, big.z, 8)
    lin_s = GrinqhLinear(small.q, small.s, small.z, 6)
    lin_s.ws = lin_b.ws  # one workspace sized for the largest layer
    lin_s.ws_bytes = lin_b.ws_bytes
    for case, lin in [(small, lin_s), (big, lin_b), (small, lin_s)]:
        _, out = run_layer(None, None, None, case.x, case.theta, lin.b_max, lin=lin, path=path)
        b_ref = check_assign(out, case.x, case.theta, lin.b_max)
        check_y(out, oracle.pack(case.q, lin.b_max), case.s, case.z, case.x, b_ref, lin.b_max)
    grinqh_check_device_error(lin_b.ws)


def test_stream_of_another_layer_sets_the_device_error_word():
    a = random_case(17, 2048, 512, 8)  # its workspace is large enough for layer b
    b = random_case(18, 1024, 512, 8)
    lin_a = GrinqhLinear(a.q, a.s, a.z, 8)
    lin_b = GrinqhLinear(b.q, b.s, b.z, 8)
    lin_a(to_dev(a.x), to_dev(a.theta))
    # gemv of layer b on the stream that assign wrote for layer a (d_in differs)
    grinqh_gemv(lin_b.planes, lin_b.s, lin_b.z, lin_a.grp_sums, lin_b.d_in, lin_b.d_out, 8,
                lin_b.y, lin_a.ws, lin_a.ws_bytes)
    with pytest.raises(GrinqhError) as e:
        grinqh_check_device_error(lin_a.ws)
    assert e.value.status == ERR_DEVICE
    assert (lin_b.y.cpu() == 0).all()
    grinqh_check_device_error(lin_a.ws)  # cleared by the read


def test_dense4_comparator_parity():
    g = np.random.default_rng(19)
    for d_in, d_out in [(512, 512), (1152, 1040), (4096, 1024)]:
        W = synth.gaussian_weights(g, d_in, d_out)
        q4, s, z = synth.rtn_quantize(W, 4)
        x = synth.activations(g, d_in)
        lin = Dense4Linear(q4, s, z)
        y = lin(to_dev(x))
        torch.cuda.synchronize()
        w4 = lin.w4.cpu().numpy().view(np.uint32)
        assert np.array_equal(w4, oracle.pack_dense4(q4))
        y_ref, bound = oracle.gemv_dense4(oracle.pack_dense4(q4), s, z, x,
                                          threads=oracle.max_threads())
        assert oracle.within_tolerance(y.cpu().numpy(), y_ref, bound, REL, ABS).all()


# ---- full-size workloads (sampled outputs, sampled packed rows) -------------------

@pytest.mark.slow
@pytest.mark.parametrize("idx", range(12))
@pytest.mark.parametrize("path", PATHS)
def test_qwen3_8b_projections(idx, path):
    lin = synth.config1()[idx]
    case = synth.make_case(lin)
    _, out = full_case_check(case, sample_outputs=256, sample_rows=64, path=path)
    assert abs(oracle.effective_bits(out["b"]) - lin.target_bits) < 0.1


@pytest.mark.slow
@pytest.mark.parametrize("idx", range(len(synth.config2())))
@pytest.mark.parametrize("path", PATHS)
def test_uniform_sweep_llama_up_proj(idx, path):
    lin = synth.config2()[idx]
    case = synth.make_case(lin)
    _, out = full_case_check(case, sample_outputs=256, sample_rows=64, path=path)
    if lin.uniform_b is not None:
        assert (out["b"] == lin.uniform_b).all()


@pytest.mark.slow
@pytest.mark.parametrize("idx", range(len(synth.config3())))
@pytest.mark.parametrize("path", PATHS)
def test_70b_shapes_redrawn_inputs(idx, path):
    spec = synth.config3()[idx]
    case = synth.make_case(spec)
    lin, _ = full_case_check(case, sample_outputs=128, sample_rows=32, path=path)
    planes_ref = oracle.pack(case.q, spec.b_max)
    for call in (1, 2):  # a fresh x per call changes the active rows
        x = synth.make_x(spec, call)
        _, out = run_layer(None, None, None, x, case.theta, spec.b_max, lin=lin, path=path)
        b_ref = check_assign(out, x, case.theta, spec.b_max)
        outs = np.random.default_rng(call).integers(0, spec.d_out, 64).astype(np.int32)
        check_y(out, planes_ref, case.s, case.z, x, b_ref, spec.b_max, outs=outs)


@pytest.mark.slow
@pytest.mark.parametrize("layer", [0, 31])
@pytest.mark.parametrize("path", PATHS)
def test_llama3_8b_layers_of_the_decode_step(layer, path):
    # all 7 linears (q, k, v, o, gate, up, down) of the first and the last of the
    # 32 layers of the decode step, each with its own weights, x and theta
    specs = [s for s in synth.config4() if s.name.startswith(f"L{layer}.")]
    assert len(specs) == 7
    for spec in specs:
        case = synth.make_case(spec)
        full_case_check(case, sample_outputs=128, sample_rows=32, path=path)
