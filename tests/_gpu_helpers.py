"""Shared pieces of the GPU parity tests: run the CUDA path through the C-ABI
and compare it with the oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
import synth
from input_adaptive_bit_b200 import grinqh_unpack
from input_adaptive_bit_b200.layer import GrinqhLinear

# The tolerance of the GEMV: |y - y_ref| <= REL * sum_i |w_hat_io||x_i| + ABS.
REL, ABS = 1e-3, 1e-6


def to_dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def run_layer(q, s, z, x, theta, b_max, phi=None, lin=None, path="two"):
    """Runs pack (unless `lin` is given), then assign + gemv (path "two") or the
    fused decode kernel (path "fused"); returns host copies."""
    if lin is None:
        lin = GrinqhLinear(q, s, z, b_max)
    xd = to_dev(x)
    th = to_dev(np.asarray(theta, np.float32))
    ph = None if phi is None else to_dev(np.asarray(phi, np.float32))
    lin.lists.fill_(-7)
    if path == "two":
        y = lin(xd, th, ph)
    elif path == "fused":
        y = lin.decode(xd, th, ph)
    else:
        raise ValueError(path)
    torch.cuda.synchronize()
    return lin, {
        "b": lin.b.cpu().numpy(),
        "lists": lin.lists.cpu().numpy(),
        "counts": lin.counts.cpu().numpy(),
        "grp_sums": lin.grp_sums.cpu().numpy(),
        "y": y.cpu().numpy().astype(np.float64),
    }


def planes_host(lin):
    return lin.planes.cpu().numpy().view(np.uint32)


def gpu_unpack(lin):
    q = torch.empty((lin.d_in, lin.d_out), dtype=torch.uint8, device=lin.device)
    grinqh_unpack(lin.planes, lin.d_in, lin.d_out, lin.b_max, q)
    torch.cuda.synchronize()
    return q.cpu().numpy()


def check_assign(out, x, theta, b_max):
    b_ref = oracle.assign(x, np.asarray(theta, np.float32), b_max)
    assert np.array_equal(out["b"], b_ref), "b differs"
    lists_ref, counts_ref = oracle.lists(b_ref, b_max)
    assert np.array_equal(out["counts"], counts_ref), (out["counts"], counts_ref)
    for p in range(b_max // 2):
        n = counts_ref[p]
        assert np.array_equal(out["lists"][p, :n], lists_ref[p, :n]), f"list {p} differs"
        assert (out["lists"][p, n:] == -7).all(), f"list {p} written past its count"
    return b_ref


def check_y(out, planes_ref, s, z, x, b_ref, b_max, phi=None, outs=None, threads=None):
    threads = threads or oracle.max_threads()
    y_ref, bound = oracle.gemv(planes_ref, s, z, x, b_ref, b_max,
                               phi=None if phi is None else np.asarray(phi, np.float64),
                               outs=outs, threads=threads)
    y = out["y"] if outs is None else out["y"][outs]
    ok = oracle.within_tolerance(y, y_ref, bound, REL, ABS)
    if not ok.all():
        bad = np.flatnonzero(~ok)[:5]
        raise AssertionError(
            f"{(~ok).sum()} outputs out of tolerance, e.g. o={bad}: y={y[bad]}, "
            f"ref={y_ref[bad]}, bound={bound[bad]}")
    return y_ref, bound


def full_case_check(case: synth.Case, phi=None, sample_outputs=None, sample_rows=None, seed=0,
                    path="two"):
    """Parity of one generated case.  Small cases compare everything; large ones
    compare b/lists/counts fully, planes on sampled rows and y on sampled outputs."""
    lin_spec = case.lin
    b_max = lin_spec.b_max
    lin, out = run_layer(case.q, case.s, case.z, case.x, case.theta, b_max, phi, path=path)
    b_ref = check_assign(out, case.x, case.theta, b_max)
    planes = planes_host(lin)
    rng = np.random.default_rng(seed)
    if sample_rows is None:
        planes_ref = oracle.pack(case.q, b_max)
        assert np.array_equal(planes, planes_ref), "planes differ"
        assert np.array_equal(gpu_unpack(lin), case.q), "unpack(planes) != q"
    else:
        rows = np.unique(np.concatenate([[0, case.q.shape[0] - 1],
                                         rng.integers(0, case.q.shape[0], sample_rows)]))
        assert np.array_equal(planes[rows], oracle.pack(case.q[rows], b_max)), "planes differ"
        planes_ref = oracle.pack(case.q, b_max)
    outs = None
    if sample_outputs is not None:
        d_out = case.q.shape[1]
        outs = np.unique(np.concatenate([[0, d_out - 1], rng.integers(0, d_out, sample_outputs)]))
        outs = outs.astype(np.int32)
    check_y(out, planes_ref, case.s, case.z, case.x, b_ref, b_max, phi, outs)
    return lin, out
