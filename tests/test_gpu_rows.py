"""Row-wise alpha-entmax (ent_entmax_rows_fwd / _bwd) against the float64 oracle.

Every row is compared element by element: tau and p with the forward, dz with
the backward, for the three root finders, both dtypes, ragged and maximum n, and
the degenerate rows (one key, constant rows, ties).
"""
import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi
from adaptive_sparse_flash_entmax_b200.inputs import round_to_bf16

pytestmark = pytest.mark.gpu

TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _rows(rows, n, seed, scale=2.0):
    g = np.random.default_rng(seed)
    return (scale * g.standard_normal((rows, n))).astype(np.float32)


def _run(z32, dtype, alpha, solver):
    zq = round_to_bf16(z32) if dtype == "bf16" else z32
    zd = torch.from_numpy(zq).to(TDT[dtype]).cuda()
    p, tau, it = A.entmax_rows_fwd(zd, alpha, solver)
    torch.cuda.synchronize()
    return zq.astype(np.float64), p.float().cpu().numpy(), tau.cpu().numpy(), it.cpu().numpy()


def _check_fwd(z, p, tau, alpha, dtype):
    ttol = 2e-5 if dtype == "f32" else 1e-4
    for r in range(z.shape[0]):
        t_ref = oracle.entmax_tau(z[r], alpha)
        assert abs(tau[r] - t_ref) <= ttol * max(1.0, abs(t_ref)), (r, tau[r], t_ref)
        p_ref = oracle.entmax_probs(z[r], alpha, t_ref)
        if dtype == "f32":
            assert np.abs(p[r] - p_ref).max() <= 2e-5, r
        else:   # bf16 storage of p: half an ulp (8 significant bits) plus the tau error
            assert np.all(np.abs(p[r] - p_ref) <= 2.0 ** -8 * np.abs(p_ref) + 1e-4), r
        # p is the definition evaluated at the returned tau (the solver's accuracy is the
        # tau check above; the stop rule bounds the step, not |sum p - 1|)
        p_own = oracle.entmax_probs(z[r], alpha, float(tau[r]))
        if dtype == "f32":
            assert np.abs(p[r] - p_own).max() <= 1e-6 + 1e-5 * np.abs(p_own).max(), r
        else:
            assert np.all(np.abs(p[r] - p_own) <= 2.0 ** -8 * np.abs(p_own) + 1e-6), r


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("solver", ["hist", "halley", "bisect"])
@pytest.mark.parametrize("n", [1, 7, 300, 1024, 5000])
def test_rows_forward_parity(dtype, solver, n):
    for alpha in (1.25, 1.5, 1.7, 2.0):
        z, p, tau, it = _run(_rows(6, n, seed=n), dtype, alpha, solver)
        _check_fwd(z, p, tau, alpha, dtype)
        assert it.min() >= 1


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rows_forward_max_n(dtype):
    n = capi.ent_entmax_rows_max_n()
    z, p, tau, _ = _run(_rows(3, n, seed=11), dtype, 1.5, "hist")
    _check_fwd(z, p, tau, 1.5, dtype)


@pytest.mark.parametrize("solver", ["hist", "halley", "bisect"])
def test_rows_degenerate(solver):
    n = 257
    z = np.zeros((4, n), np.float32)
    z[1] = 3.0                                   # constant row: p = 1/n
    z[2, :5] = 4.0                               # five tied maxima, the rest far below
    z[2, 5:] = -50.0
    z[3] = np.linspace(-1, 1, n, dtype=np.float32)
    for alpha in (1.5, 2.0):
        zz, p, tau, _ = _run(z, "f32", alpha, solver)
        _check_fwd(zz, p, tau, alpha, "f32")
        # within the stop rule's step (4e-7 max(1,|tau|)) times dp/dtau (1 at alpha = 2)
        assert np.allclose(p[1], 1.0 / n, atol=1e-5)
        assert np.allclose(p[2, :5], 0.2, atol=1e-5) and np.all(p[2, 5:] == 0)


def test_rows_halley_needs_fewer_passes_than_bisection():
    z = _rows(64, 4096, seed=3)
    its = {}
    for solver in ("hist", "halley", "bisect"):
        _, _, _, it = _run(z, "f32", 1.5, solver)
        its[solver] = it.astype(np.float64).mean()
    assert its["bisect"] >= 3 * its["halley"], its
    assert its["hist"] <= its["halley"], its


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 300, 5000])
def test_rows_backward_parity(dtype, n):
    for alpha in (1.25, 1.5, 2.0):
        z32 = _rows(5, n, seed=100 + n)
        dp32 = _rows(5, n, seed=200 + n, scale=1.0)
        if dtype == "bf16":
            z32, dp32 = round_to_bf16(z32), round_to_bf16(dp32)
        zd = torch.from_numpy(z32).to(TDT[dtype]).cuda()
        dpd = torch.from_numpy(dp32).to(TDT[dtype]).cuda()
        _, tau, _ = A.entmax_rows_fwd(zd, alpha, "hist")
        dz = A.entmax_rows_bwd(zd, tau, dpd, alpha).float().cpu().numpy()
        tau = tau.cpu().numpy()
        for r in range(5):
            t_ref = oracle.entmax_tau(z32[r].astype(np.float64), alpha)
            ds, g, _ = oracle.entmax_vjp_row(z32[r].astype(np.float64), alpha, t_ref,
                                              dp32[r].astype(np.float64))
            err = np.linalg.norm(dz[r] - ds) / max(np.linalg.norm(ds), 1e-12)
            assert err <= (1e-4 if dtype == "f32" else 2e-2), (r, err)
            # J 1 = 0: the row of dz sums to zero, up to the storage rounding of dz
            stol = 1e-4 if dtype == "f32" else 2.0 ** -7
            assert abs(dz[r].sum()) <= stol * max(1.0, np.abs(ds).sum())


def test_rows_bad_arguments():
    z = torch.zeros((2, 8), device="cuda")
    with pytest.raises(capi.EntAttnError) as e:
        A.entmax_rows_fwd(z, 2.5)
    assert e.value.status == capi.ENT_EINVAL
    big = torch.zeros((1, capi.ent_entmax_rows_max_n() + 1), device="cuda")
    with pytest.raises(capi.EntAttnError) as e:
        A.entmax_rows_fwd(big, 1.5)
    assert e.value.status == capi.ENT_EUNSUPPORTED
    st = capi.ent_entmax_rows_fwd(z.data_ptr(), 2, 8, capi.ENT_F32, 1.5, 7, z.data_ptr(),
                                  z.data_ptr(), None, 0)
    assert st == capi.ENT_EINVAL
