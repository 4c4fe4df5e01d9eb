"""ent_attn_fwd_otilde / ent_attn_bwd_otilde against the float64 oracle.

The forward with otilde must return exactly what the plain forward returns (same
o, tau, block mask and pass counts, bit for bit) plus otilde_i = sum_j g_ij v_j /
sum_j g_ij; the backward given otilde takes delta_i = dO_i . otilde_i and must
meet the same gradient bound as the plain backward.

otilde bound: max |otilde_gpu - otilde_ref| <= 1e-2 (bfloat16 inputs; g is
rounded to bf16 for the tensor-core product, a relative 2^-9 per weight of a
weighted mean of values of size ~1) or 1e-4 (float32), on rows whose scores all
lie outside the 1e-3 band around tau_ref (inside it g = u^(gamma-1) is steep, and
at alpha = 2 it jumps from 0 to 1, so a score within rounding of tau moves
otilde by a whole support member).  Rows inside the band are counted, not
compared; the gradient check covers them end to end.
"""
import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from parity import BAND, GRAD_RTOL, check_grads, rel_frob, to_dev, to_np

pytestmark = pytest.mark.gpu

OT_TOL = {"f32": 1e-4, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


def _clear_rows(q, k, alpha, causal, rows, tau_ref):
    """Rows (flat ids) whose admissible scores all lie outside the band around tau_ref."""
    B, H, N, d = q.shape
    keep = []
    for flat, tr in zip(rows, tau_ref):
        bh, i = divmod(int(flat), N)
        b, h = divmod(bh, H)
        n = i + 1 if causal else N
        x = (alpha - 1) * (k[b, h, :n].astype(np.float64) @ q[b, h, i].astype(np.float64)) / np.sqrt(d)
        keep.append(np.abs(x - tr).min() > BAND)
    return np.array(keep, bool)


def _run_both(q, k, v, do, alpha, causal, dtype):
    qd, kd, vd, dod = (to_dev(a, dtype) for a in (q, k, v, do))
    wsf = A.workspace(capi.ent_attn_fwd_workspace_size(*q.shape, capi.ENT_BF16), "cuda")
    o0, tau0, m0, it0 = A.entmax_attn_fwd(qd, kd, vd, alpha, causal, with_iters=True)
    ot = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    o1, tau1, m1, it1 = A.entmax_attn_fwd(qd, kd, vd, alpha, causal, with_iters=True, otilde=ot,
                                          ws=wsf)
    cf = A.read_status(wsf)
    wsb = A.workspace(capi.ent_attn_bwd_workspace_size(*q.shape, capi.ENT_BF16), "cuda")
    dq, dk, dv = A.entmax_attn_bwd(qd, kd, vd, None, dod, tau1, m1, alpha, causal, otilde=ot,
                                   ws=wsb)
    cb = A.read_status(wsb)
    g0 = A.entmax_attn_bwd(qd, kd, vd, None, dod, tau0, m0, alpha, causal, ws=wsb)
    cb0 = A.read_status(wsb)
    torch.cuda.synchronize()
    # the otilde forward changes nothing else
    for a0, a1 in ((o0, o1), (tau0, tau1), (m0, m1), (it0, it1)):
        assert torch.equal(a0, a1)
    # the backward given otilde skips exactly the delta phase (S and dP of every live
    # block) and lands where the plain backward does
    live = int(m1.sum().item())
    assert cb0[4] - cb[4] == 2 * live, (cb0[4], cb[4], live)
    for a, b in zip((dq, dk, dv), g0):
        assert rel_frob(to_np(a).astype(np.float64), to_np(b).astype(np.float64)) <= 1e-2
    return dict(o=to_np(o1), tau=to_np(tau1), mask=to_np(m1), ot=to_np(ot), dq=to_np(dq),
                dk=to_np(dk), dv=to_np(dv), cf=cf, cb=cb)


def _check_otilde(gpu, q, k, v, alpha, causal, dtype, rows):
    d = q.shape[-1]
    ot_ref = oracle.attn_otilde_rows(q, k, v, alpha, causal, rows)
    ot = gpu["ot"].reshape(-1, d)[rows]
    assert np.all(np.isfinite(ot))
    _, tau_ref, _ = oracle.attn_fwd_rows(q, k, v, alpha, causal, rows)
    clear = _clear_rows(q, k, alpha, causal, rows, tau_ref)
    assert clear.mean() >= 0.75, clear.mean()
    err = np.abs(ot - ot_ref)[clear].max()
    assert err <= OT_TOL[dtype], err
    return err


@pytest.mark.parametrize("N", [128, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.7, 2.0])
def test_otilde_small_bf16(N, d, causal, alpha):
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=N, d=d, causal=causal, alpha=alpha,
                                         beta=2.0, seed=N + d + 7)
    gpu = _run_both(q, k, v, do, alpha, causal, "bf16")
    _check_otilde(gpu, q, k, v, alpha, causal, "bf16", np.arange(2 * N))
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, alpha, causal)
    check_grads(gpu, (dq, dk, dv))
    # counters: one G.V product per P.V block (the live blocks, and after an unevaluated
    # downward stop the candidates at the final tau)
    live = int(gpu["mask"].sum())
    assert gpu["cf"][5] == gpu["cf"][1] >= live


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_otilde_small_fp32_ragged(alpha):
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=300, d=64, causal=True, alpha=alpha,
                                         beta=1.0, dtype="f32", seed=17)
    gpu = _run_both(q, k, v, do, alpha, True, "f32")
    _check_otilde(gpu, q, k, v, alpha, True, "f32", np.arange(600))
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, alpha, True)
    errs = check_grads(gpu, (dq, dk, dv))
    assert max(errs.values()) <= 1e-3, errs
    assert gpu["cf"][5] == gpu["cf"][1]


def test_otilde_degenerate_rows():
    # one key per row (causal row 0), constant rows (otilde = plain mean of v at every
    # alpha, since every g is equal) and a ragged tail of one row
    g = np.random.default_rng(3)
    N, d = 129, 64
    q = np.zeros((1, 1, N, d), np.float32)
    k = inputs.round_to_bf16(g.standard_normal((1, 1, N, d)).astype(np.float32))
    v = inputs.round_to_bf16(g.standard_normal((1, 1, N, d)).astype(np.float32))
    do = inputs.round_to_bf16(g.standard_normal((1, 1, N, d)).astype(np.float32))
    for causal in (True, False):
        gpu = _run_both(q, k, v, do, 1.5, causal, "bf16")
        ot = gpu["ot"][0, 0]
        for i in (0, 1, 64, 127, 128):
            n = i + 1 if causal else N
            np.testing.assert_allclose(ot[i], v[0, 0, :n].astype(np.float64).mean(axis=0), atol=1e-5)


def test_otilde_workload_iid_sampled():
    # the full iid workload in the launch configuration the bench times: sampled rows of
    # otilde, sampled rows and keys of the gradients, and the sum rules at full size
    w = inputs.WORKLOADS["iid"]
    q, k, v, do = inputs.make_inputs(w, 0)
    gpu = _run_both(q, k, v, do, w.alpha, w.causal, w.dtype)
    B, H, N, d = w.shape
    g = np.random.default_rng(1)
    rows = []
    for bh in (0, B * H - 1):
        rows += [bh * N, bh * N + N - 1] + list(bh * N + g.choice(N, 24, replace=False))
    rows = np.array(sorted(set(rows)))
    _check_otilde(gpu, q, k, v, w.alpha, w.causal, w.dtype, rows)
    qh, kh, vh, doh = (a[0, 0] for a in (q, k, v, do))
    keys = sorted(set(range(N - 64, N)) | set(g.choice(N, 16, replace=False).tolist()))
    qrows = list(range(N - 32, N)) + [0, 1, 2]
    dq_r, dk_k, dv_k = oracle.attn_bwd_head_sampled(qh, kh, vh, doh, w.alpha, w.causal, qrows, keys)
    assert rel_frob(gpu["dq"][0, 0, qrows], dq_r) <= GRAD_RTOL
    assert rel_frob(gpu["dk"][0, 0, keys], dk_k) <= GRAD_RTOL
    assert rel_frob(gpu["dv"][0, 0, keys], dv_k) <= GRAD_RTOL
    dvs = gpu["dv"].astype(np.float64).sum(axis=2)
    assert np.abs(dvs - do.astype(np.float64).sum(axis=2)).max() <= 2e-2 * np.sqrt(N)


def test_otilde_autograd_matches_recompute():
    w, (q, k, v, do) = inputs.small_case(B=2, H=2, N=384, d=128, causal=True, alpha=1.5,
                                         beta=2.0, seed=5)
    grads = {}
    for mode in ("otilde", "recompute"):
        qd, kd, vd = (to_dev(a, "bf16").requires_grad_() for a in (q, k, v))
        o = A.entmax_attention(qd, kd, vd, 1.5, True, delta=mode)
        o.backward(to_dev(do, "bf16"))
        grads[mode] = [to_np(t.grad) for t in (qd, kd, vd)]
    for a, b in zip(grads["otilde"], grads["recompute"]):
        assert rel_frob(a.astype(np.float64), b.astype(np.float64)) <= 1e-2


def test_otilde_bad_arguments():
    z = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    tau = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    m = torch.zeros((1, 1, 1, 1), dtype=torch.uint8, device="cuda")
    ws = A.workspace(capi.ent_attn_bwd_workspace_size(1, 1, 128, 64, capi.ENT_BF16), "cuda")
    st = capi.ent_attn_fwd_otilde(z.data_ptr(), z.data_ptr(), z.data_ptr(), 1, 1, 128, 64,
                                  capi.ENT_BF16, 1.5, 1, z.data_ptr(), tau.data_ptr(), m.data_ptr(),
                                  None, None, ws.data_ptr(), ws.numel(), None)
    assert st == capi.ENT_EINVAL
    st = capi.ent_attn_bwd_otilde(z.data_ptr(), z.data_ptr(), z.data_ptr(), None, z.data_ptr(),
                                  tau.data_ptr(), m.data_ptr(), 1, 1, 128, 64, capi.ENT_BF16, 1.5, 1,
                                  z.data_ptr(), z.data_ptr(), z.data_ptr(), ws.data_ptr(),
                                  ws.numel(), None)
    assert st == capi.ENT_EINVAL
    with pytest.raises(ValueError):
        A.entmax_attn_fwd(z, z, z, 1.5, True, otilde=torch.zeros_like(z))
