"""Whole heads against the oracle at the full workload sizes: every head of the
LM-shaped workload, and heads (0, 0) and (B-1, H-1) of the iid and alpha workloads
(the rest of their heads are covered by the every-row checks of test_gpu_fullsize.py).
The GPU runs the whole workload in the launch configuration the bench times; the
oracle computes the selected heads in full, forward and backward, and both backward
paths (delta recomputed, delta from otilde) are compared."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from parity import check_grads, check_mask, check_o, check_tau, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


def _run(w, heads):
    q, k, v, do = inputs.make_inputs(w, seed=2)
    qd, kd, vd, dod = (to_dev(a, w.dtype) for a in (q, k, v, do))
    o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal)
    grads = A.entmax_attn_bwd(qd, kd, vd, o, dod, tau, mask, w.alpha, w.causal)
    ot = torch.empty(qd.shape, dtype=torch.float32, device="cuda")
    A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal, otilde=ot)
    grads_ot = A.entmax_attn_bwd(qd, kd, vd, None, dod, tau, mask, w.alpha, w.causal, otilde=ot)
    torch.cuda.synchronize()
    sel = lambda a: np.ascontiguousarray(np.stack([a[b, h] for b, h in heads])[None])
    gpu = {"o": sel(to_np(o)), "tau": sel(to_np(tau)), "mask": sel(to_np(mask))}
    qs, ks, vs, dos = (sel(a) for a in (q, k, v, do))
    o_ref, tau_ref, marg = oracle.attn_fwd(qs, ks, vs, w.alpha, w.causal)
    check_tau(gpu["tau"], tau_ref)
    check_o(gpu["o"], o_ref, w.dtype, label=f"{w.name} alpha {w.alpha} beta {w.beta} (whole heads)")
    check_mask(gpu["mask"], marg)
    ref = oracle.attn_bwd(qs, ks, vs, dos, w.alpha, w.causal)[:3]
    for g in (grads, grads_ot):
        check_grads({key: sel(to_np(t)) for key, t in zip(("dq", "dk", "dv"), g)}, ref)


def test_lm_every_head():
    w = inputs.WORKLOADS["lm"]
    _run(w, [(b, h) for b in range(w.B) for h in range(w.H)])


@pytest.mark.parametrize("change", [{}, {"beta": 8.0}])
def test_iid_first_and_last_head(change):
    w = inputs.WORKLOADS["iid"].replace(**change) if change else inputs.WORKLOADS["iid"]
    _run(w, [(0, 0), (w.B - 1, w.H - 1)])


@pytest.mark.parametrize("alpha", [1.25, 2.0])
def test_alpha_first_and_last_head(alpha):
    w = inputs.WORKLOADS["alpha"].replace(alpha=alpha)
    _run(w, [(0, 0), (w.B - 1, w.H - 1)])
