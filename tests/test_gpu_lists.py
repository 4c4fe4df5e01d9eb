"""Support-list pair (ent_attn_fwd_lists / ent_attn_bwd_lists) against the float64 oracle.

The forward records, per query row, the keys with p > 0 and their u = x - tau (up to 16;
list_n = 255 beyond that); the backward does every query tile whose rows all have lists
from the lists alone and the other tiles by the block kernels.  Checked: the forward's
outputs are bit-identical to ent_attn_fwd's, each list is the row's support (outside
the 1e-3 band around tau) with u = x - tau, and the gradients meet the oracle on small
cases (all-list, mixed and all-block tiles) and on sampled rows and keys at full size."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from parity import BAND, GRAD_RTOL, check_grads, check_o, check_tau, rel_frob, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


def run_lists(q, k, v, do, alpha, causal):
    qd, kd, vd, dod = (to_dev(a, "bf16") for a in (q, k, v, do))
    lists = A.alloc_lists(qd)
    o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, alpha, causal, lists=lists)
    o0, tau0, mask0, _ = A.entmax_attn_fwd(qd, kd, vd, alpha, causal)
    torch.cuda.synchronize()
    assert torch.equal(o, o0) and torch.equal(tau, tau0) and torch.equal(mask, mask0)
    B, H, N, d = q.shape
    ws = A.workspace(capi.ent_attn_bwd_lists_workspace_size(B, H, N, d, capi.ENT_BF16), qd.device)
    dq, dk, dv = A.entmax_attn_bwd(qd, kd, vd, o, dod, tau, mask, alpha, causal, lists=lists, ws=ws)
    torch.cuda.synchronize()
    T = -(-N // 128)
    L = capi.ent_attn_bwd_workspace_size(B, H, N, d, capi.ENT_BF16)
    tiles = ws[L:L + B * H * T].view(B, H, T).cpu().numpy()   # tiles the list kernel covered
    return ({"o": to_np(o), "tau": to_np(tau), "mask": to_np(mask), "dq": to_np(dq),
             "dk": to_np(dk), "dv": to_np(dv)},
            tuple(to_np(x) for x in lists), tiles)


def check_lists(q, k, tau, lists, alpha, causal, rows=None):
    """Each listed row: its keys are {j : x_ij > tau_i} outside the band, u = x - tau."""
    lk, lu, ln = lists
    B, H, N, d = q.shape
    cap = capi.ent_attn_list_cap()
    flat = range(B * H * N) if rows is None else rows
    listed = 0
    for f in flat:
        bh, i = divmod(int(f), N)
        b, h = divmod(bh, H)
        n_adm = i + 1 if causal else N
        x = (alpha - 1) * (k[b, h, :n_adm].astype(np.float64) @ q[b, h, i].astype(np.float64)) / np.sqrt(d)
        t = float(tau[b, h, i])
        n = int(ln[b, h, i])
        if n == 255:        # more nonzeros than a list holds (up to scores within the band)
            assert (x > t - BAND).sum() > cap
            continue
        listed += 1
        keys = lk[b, h, i, :n]
        assert len(set(keys.tolist())) == n and np.all((keys >= 0) & (keys < n_adm))
        clear = np.abs(x - t) > BAND
        assert set(keys[clear[keys]].tolist()) == set(np.flatnonzero((x > t) & clear).tolist())
        assert np.abs(lu[b, h, i, :n] - (x[keys] - t)).max() <= 1e-3
    return listed


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_small_all_list_tiles(d, causal, alpha):
    # beta 8: a few nonzeros per row, so every tile is done from its lists
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=300, d=d, causal=causal, alpha=alpha,
                                         beta=8.0, seed=40 + d)
    gpu, lists, tiles = run_lists(q, k, v, do, alpha, causal)
    o_ref, tau_ref, _ = oracle.attn_fwd(q, k, v, alpha, causal)
    check_tau(gpu["tau"], tau_ref)
    check_o(gpu["o"], o_ref, "bf16")
    assert check_lists(q, k, gpu["tau"], lists, alpha, causal) > 0
    assert tiles.any()
    if alpha >= 1.5:       # alpha 1.25 keeps more than 16 nonzeros in some rows
        assert tiles.all()
    check_grads(gpu, oracle.attn_bwd(q, k, v, do, alpha, causal)[:3])


def test_small_mixed_tiles():
    # query tile 0 sharp (beta 8: lists), tile 1 flat (beta 1/4: > 16 nonzeros, block
    # kernels), tile 2 sharp again: the two backward paths meet in dK and dV
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=384, d=64, causal=False, beta=1.0, seed=77)
    q[:, :, :128] *= 8.0
    q[:, :, 128:256] *= 0.25
    q[:, :, 256:] *= 8.0
    q = inputs.round_to_bf16(q).reshape(q.shape)
    gpu, lists, tiles = run_lists(q, k, v, do, 1.5, False)
    assert tiles[:, :, 0].all() and not tiles[:, :, 1].any() and tiles[:, :, 2].all()
    check_lists(q, k, gpu["tau"], lists, 1.5, False)
    check_grads(gpu, oracle.attn_bwd(q, k, v, do, 1.5, False)[:3])


@pytest.mark.parametrize("name,change", [("iid", {"beta": 8.0}), ("iid", {"beta": 4.0}),
                                         ("alpha", {}), ("alpha", {"alpha": 2.0})])
def test_fullsize_sampled(name, change):
    w = inputs.WORKLOADS[name].replace(**change)
    q, k, v, do = inputs.make_inputs(w, seed=1)
    gpu, lists, tiles = run_lists(q, k, v, do, w.alpha, w.causal)
    B, H, N, d = w.shape
    assert tiles.mean() > 0.5       # most query tiles done from their lists
    g = np.random.default_rng(1)
    rows = np.array(sorted(set([0, N - 1] + list(g.choice(B * H * N, 24, replace=False)))))
    o_r, tau_r, _ = oracle.attn_fwd_rows(q, k, v, w.alpha, w.causal, rows)
    check_tau(gpu["tau"].reshape(-1)[rows], tau_r)
    check_lists(q, k, gpu["tau"], lists, w.alpha, w.causal, rows=rows)
    # gradients of the first head on sampled rows and keys
    qh, kh, vh, doh = (a[0, 0] for a in (q, k, v, do))
    keys = sorted(set(range(N - 64, N)) | set(g.choice(N, 16, replace=False).tolist()))
    qrows = list(range(N - 32, N)) + [0, 1, 2]
    dq_r, dk_k, dv_k = oracle.attn_bwd_head_sampled(qh, kh, vh, doh, w.alpha, w.causal, qrows, keys)
    assert rel_frob(gpu["dq"][0, 0, qrows], dq_r) <= GRAD_RTOL
    assert rel_frob(gpu["dk"][0, 0, keys], dk_k) <= GRAD_RTOL
    assert rel_frob(gpu["dv"][0, 0, keys], dv_k) <= GRAD_RTOL
    # and everywhere against the block-kernel backward of the same forward
    qd, kd, vd, dod = (to_dev(a, "bf16") for a in (q, k, v, do))
    o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal)
    ref = A.entmax_attn_bwd(qd, kd, vd, o, dod, tau, mask, w.alpha, w.causal)
    for key, r in zip(("dq", "dk", "dv"), ref):
        assert rel_frob(gpu[key].astype(np.float64), to_np(r).astype(np.float64)) <= 1e-2


def test_lists_argument_errors():
    z = torch.zeros((1, 1, 128, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(capi.EntAttnError) as e:
        A.entmax_attn_fwd(z, z, z, 1.5, True, lists=A.alloc_lists(z))
    assert e.value.status == capi.ENT_EUNSUPPORTED


def test_autograd_lists_matches_recompute():
    # beta 8: every query tile has lists, so the backward runs the list kernel alone
    w, (q, k, v, do) = inputs.small_case(B=2, H=2, N=384, d=64, causal=True, alpha=1.5,
                                         beta=8.0, seed=6)
    grads = {}
    for mode in ("lists", "recompute"):
        qd, kd, vd = (to_dev(a, "bf16").requires_grad_() for a in (q, k, v))
        o = A.entmax_attention(qd, kd, vd, 1.5, True, delta=mode)
        o.backward(to_dev(do, "bf16"))
        grads[mode] = [to_np(t.grad) for t in (qd, kd, vd)]
    for a, b in zip(grads["lists"], grads["recompute"]):
        assert rel_frob(a.astype(np.float64), b.astype(np.float64)) <= 1e-2
