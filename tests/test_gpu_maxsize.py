"""The largest sizes the library accepts: one head of N = 130944 (1023 query tiles, the
top of the supported range) and B*H = 65535 heads (the grid's y limit) of a ragged
16-row tile.  The oracle checks sampled rows, whole tiles and whole heads; torch float32
arithmetic checks every row (tests/fullsize.py, and a batched form for the short heads)."""
import math

import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from fullsize import check_forward
from parity import GRAD_RTOL, check_grads, check_mask, check_o, check_tau, rel_frob, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


def test_longest_sequence():
    w = inputs.Workload("longest", 1, 1, 130944, 128, "bf16", True, 1.5, 1.0, "iid")
    q, k, v, do = inputs.make_inputs(w, seed=4)
    qd, kd, vd, dod = (to_dev(a, "bf16") for a in (q, k, v, do))
    o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal)
    dq, dk, dv = A.entmax_attn_bwd(qd, kd, vd, o, dod, tau, mask, w.alpha, w.causal)
    torch.cuda.synchronize()
    N = w.N
    # every row: tau in its bracket and at its root, the mask, O
    check_forward(qd, kd, vd, tau, mask, o, w.alpha, w.causal)
    # oracle: sampled rows and the first and last tiles
    g = np.random.default_rng(4)
    rows = np.unique(np.r_[0, 1, N - 1, g.choice(N, 16, replace=False)])
    o_r, tau_r, _ = oracle.attn_fwd_rows(q, k, v, w.alpha, w.causal, rows)
    check_tau(to_np(tau).reshape(-1)[rows], tau_r)
    check_o(to_np(o).reshape(-1, w.d)[rows], o_r, "bf16")
    for t in (0, N // 128 - 1):
        r = np.arange(t * 128, t * 128 + 128)
        _, tau_t, bm = oracle.attn_fwd_rows(q, k, v, w.alpha, w.causal, r)
        check_tau(to_np(tau).reshape(-1)[r], tau_t)
        check_mask(to_np(mask)[0, 0, t][None], bm.max(axis=0)[None])
    # backward: the last rows and keys against the oracle, sum rules over the head
    qrows, keys = list(range(N - 32, N)), list(range(N - 64, N))
    dq_r, dk_k, dv_k = oracle.attn_bwd_head_sampled(q[0, 0], k[0, 0], v[0, 0], do[0, 0], w.alpha,
                                                    w.causal, qrows, keys)
    assert rel_frob(to_np(dq)[0, 0, qrows], dq_r) <= GRAD_RTOL
    assert rel_frob(to_np(dk)[0, 0, keys], dk_k) <= GRAD_RTOL
    assert rel_frob(to_np(dv)[0, 0, keys], dv_k) <= GRAD_RTOL
    dvs = to_np(dv).astype(np.float64).sum(axis=2)
    assert np.abs(dvs - do.astype(np.float64).sum(axis=2)).max() <= 2e-2 * np.sqrt(N)


def _check_short_heads(q, k, v, tau, mask, o, alpha):
    """Every head of a [BH, n <= 128] problem at once (causal): bracket, Newton distance,
    O against exact p, and the single block of each head marked live."""
    BH, n, d = q.shape
    gamma, cx = 1.0 / (alpha - 1.0), (alpha - 1.0) / math.sqrt(d)
    x = cx * torch.bmm(q.float(), k.float().transpose(1, 2))
    causal = torch.tril(torch.ones(n, n, dtype=torch.bool, device=q.device))
    x = x.masked_fill(~causal, -math.inf)
    t = tau.float()
    m = x.amax(dim=2)
    cnt = torch.arange(1, n + 1, device=q.device, dtype=torch.float32)[None, :]
    slack = 1e-4 * torch.clamp(m.abs(), min=1.0)
    assert bool(((t >= m - 1.0 - slack) & (t <= m - cnt ** (1.0 - alpha) + slack)).all())
    u = x - t[..., None]
    up = torch.clamp(u, min=0)
    f = torch.pow(up, gamma).sum(dim=2) - 1.0
    gs = torch.where(u > 0, torch.pow(up, gamma - 1.0), torch.zeros_like(up)).sum(dim=2)
    assert float((f.abs() / (gamma * gs) / torch.clamp(t.abs(), min=1.0)).max()) <= 1e-3
    o_ref = torch.bmm(torch.pow(up, gamma), v.float())
    ax = torch.clamp(o_ref.abs(), min=torch.finfo(torch.float32).tiny)
    err = (o.float() - o_ref).abs() - torch.exp2(torch.floor(torch.log2(ax)) - 8)
    assert float(err.max()) <= 1e-2
    assert bool((mask.reshape(BH) == 1).all())


def test_most_heads():
    w = inputs.Workload("most-heads", 65535, 1, 16, 64, "bf16", True, 1.5, 2.0, "iid")
    q, k, v, do = inputs.make_inputs(w, seed=5)
    qd, kd, vd, dod = (to_dev(a, "bf16") for a in (q, k, v, do))
    for with_ot in (False, True):
        ot = torch.empty(qd.shape, dtype=torch.float32, device="cuda") if with_ot else None
        o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal, otilde=ot)
        dq, dk, dv = A.entmax_attn_bwd(qd, kd, vd, o, dod, tau, mask, w.alpha, w.causal, otilde=ot)
        torch.cuda.synchronize()
        BH = w.B * w.H
        _check_short_heads(qd.view(BH, w.N, w.d), kd.view(BH, w.N, w.d), vd.view(BH, w.N, w.d),
                           tau.view(BH, w.N), mask, o.view(BH, w.N, w.d), w.alpha)
        # whole heads against the oracle: first, middle, last
        sel = [0, BH // 2, BH - 1]
        pick = lambda a: np.ascontiguousarray(a.reshape(BH, w.N, w.d)[sel][None])
        qs, ks, vs, dos = (pick(a) for a in (q, k, v, do))
        o_ref, tau_ref, _ = oracle.attn_fwd(qs, ks, vs, w.alpha, w.causal)
        check_tau(to_np(tau).reshape(BH, w.N)[sel][None], tau_ref)
        check_o(pick(to_np(o)), o_ref, "bf16")
        ref = oracle.attn_bwd(qs, ks, vs, dos, w.alpha, w.causal)[:3]
        check_grads({"dq": pick(to_np(dq)), "dk": pick(to_np(dk)), "dv": pick(to_np(dv))}, ref)
        # every head: the rows of dV sum to those of dO (p sums to 1 per row)
        dvs = dv.float().view(BH, w.N, w.d).sum(dim=1)
        dos_all = dod.float().view(BH, w.N, w.d).sum(dim=1)
        assert float((dvs - dos_all).abs().max()) <= 2e-2 * math.sqrt(w.N)
