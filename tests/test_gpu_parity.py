"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases run the whole oracle; the full-size workloads are checked on
sampled rows, keys and whole tiles that the oracle computes one by one, plus
sum rules that hold at any size.  Tolerances are in tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from parity import (check_grads, check_mask, check_o, check_support, check_tau, run_gpu, to_dev,
                    to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


def full_parity(q, k, v, do, alpha, causal, dtype, bwd=True):
    gpu = run_gpu(q, k, v, do, alpha, causal, dtype, with_bwd=bwd)
    o_ref, tau_ref, marg = oracle.attn_fwd(q, k, v, alpha, causal)
    check_tau(gpu["tau"], tau_ref)
    check_o(gpu["o"], o_ref, dtype, label=f"small cases {dtype} (whole oracle)")
    check_mask(gpu["mask"], marg)
    B, H, N, d = q.shape
    rows = np.unique(np.r_[0, N - 1, np.arange(0, B * H * N, max(1, B * H * N // 64))])
    check_support(q, k, gpu["tau"].reshape(-1)[rows], tau_ref.reshape(-1)[rows], alpha, causal, rows)
    assert gpu["iters"].max() <= 24
    if bwd:
        dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, alpha, causal)
        check_grads(gpu, (dq, dk, dv))
    return gpu


def test_tiny_fp32_workload():
    w = inputs.WORKLOADS["tiny"]
    q, k, v, do = inputs.make_inputs(w, seed=0)
    full_parity(q, k, v, do, w.alpha, w.causal, "f32")


@pytest.mark.parametrize("N", [128, 300, 384])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.7, 2.0])
def test_small_bf16(N, d, causal, alpha):
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=N, d=d, causal=causal, alpha=alpha,
                                         beta=2.0, seed=N + d)
    full_parity(q, k, v, do, alpha, causal, "bf16")


@pytest.mark.parametrize("causal", [False, True])
def test_small_f32_d32(causal):
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=200, d=32, dtype="f32", causal=causal,
                                         alpha=1.5, beta=2.0, seed=32)
    full_parity(q, k, v, do, 1.5, causal, "f32")


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_small_fp32_ragged(alpha):
    w, (q, k, v, do) = inputs.small_case(B=2, H=1, N=200, d=64, dtype="f32", causal=True,
                                         alpha=alpha, seed=5)
    full_parity(q, k, v, do, alpha, True, "f32")


def test_clustered_block_sparse():
    """Clustered keys: most 128x128 blocks are dead; parity and mask still exact."""
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=2048, d=128, causal=True, alpha=1.5,
                                         beta=4.0, kind="clustered", seed=2)
    gpu = full_parity(q, k, v, do, 1.5, True, "bf16")
    T = 16
    live = gpu["mask"][:, :, np.tril_indices(T)[0], np.tril_indices(T)[1]]
    assert 0 < live.mean() < 0.7   # a good share of the causal blocks is skipped


# ------------------------------------------------------------- edge cases
def test_single_key():
    q = np.ones((1, 1, 1, 64), np.float32)
    k = np.full((1, 1, 1, 64), 0.5, np.float32)
    v = np.arange(64, dtype=np.float32).reshape(1, 1, 1, 64)
    do = np.ones_like(v)
    for dtype in ("f32", "bf16"):
        gpu = run_gpu(q, k, v, do, 1.5, True, dtype)
        np.testing.assert_allclose(gpu["o"], v, atol=1e-6)
        x = 0.5 * 0.5 * 64 / 8.0
        assert gpu["tau"][0, 0, 0] == pytest.approx(x - 1.0, abs=1e-5)
        assert gpu["mask"].tolist() == [[[[1]]]]
        np.testing.assert_allclose(gpu["dv"], do, atol=1e-6)   # p = 1
        np.testing.assert_allclose(gpu["dq"], 0, atol=1e-6)    # dS = 0 with one key
        np.testing.assert_allclose(gpu["dk"], 0, atol=1e-6)


def test_causal_row0_and_constant_rows():
    w, (q, k, v, do) = inputs.small_case(B=1, H=1, N=256, d=64, causal=True, seed=3)
    q[:] = 0.0     # all scores 0: row i is uniform over its i+1 keys
    gpu = full_parity(q, k, v, do, 1.5, True, "bf16")
    np.testing.assert_allclose(gpu["o"][0, 0, 0], v[0, 0, 0], atol=1e-2)
    want = np.cumsum(v[0, 0].astype(np.float64), axis=0) / np.arange(1, 257)[:, None]
    np.testing.assert_allclose(gpu["o"][0, 0], want, atol=1e-2)


def test_ties():
    w, (q, k, v, do) = inputs.small_case(B=1, H=1, N=256, d=64, causal=False, beta=4.0, seed=4)
    k[0, 0, 128:] = k[0, 0, :128]          # every key duplicated in the other block
    full_parity(q, k, v, do, 1.5, False, "bf16")


def test_empty_inputs_are_noops():
    for shape in ((0, 2, 128, 64), (1, 0, 128, 64), (1, 2, 0, 64)):
        z = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        o, tau, mask, _ = A.entmax_attn_fwd(z, z, z, 1.5, True)
        dq, dk, dv = A.entmax_attn_bwd(z, z, z, o, z, tau, mask, 1.5, True)
        assert o.shape == shape and dq.shape == shape


def test_guard_bands_untouched():
    """Outputs are views into larger buffers whose margins hold a canary."""
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=300, d=64, causal=True, seed=6)
    qd, kd, vd, dod = (to_dev(a, "bf16") for a in (q, k, v, do))
    n = q.size
    G = 4096

    def guarded(numel, dtype):
        buf = torch.full((numel + 2 * G,), 7, dtype=dtype, device="cuda")
        return buf, buf[G:G + numel]

    ob, o = guarded(n, torch.bfloat16)
    tb, tau = guarded(2 * 300, torch.float32)
    mb, mask = guarded(2 * 9, torch.uint8)
    ib, it = guarded(2 * 300, torch.uint8)
    A.entmax_attn_fwd(qd, kd, vd, 1.5, True, with_iters=True,
                      out=(o.view(q.shape), tau.view(1, 2, 300), mask.view(1, 2, 3, 3),
                           it.view(1, 2, 300)))
    grads = [guarded(n, torch.bfloat16) for _ in range(3)]
    A.entmax_attn_bwd(qd, kd, vd, o.view(q.shape), dod, tau.view(1, 2, 300), mask.view(1, 2, 3, 3),
                      1.5, True, out=tuple(g.view(q.shape) for _, g in grads))
    torch.cuda.synchronize()
    for buf in [ob, tb, mb, ib] + [b for b, _ in grads]:
        assert torch.all(buf[:G] == 7) and torch.all(buf[-G:] == 7)


def test_counters_and_status():
    w, (q, k, v, do) = inputs.small_case(B=2, H=2, N=512, d=64, causal=True, seed=7)
    qd, kd, vd = (to_dev(a, "bf16") for a in (q, k, v))
    ws = A.workspace(capi.ent_attn_fwd_workspace_size(2, 2, 512, 64, capi.ENT_BF16), "cuda")
    o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, 1.5, True, ws=ws)
    ctr = A.read_status(ws)
    assert ctr[3] == 2 * 2 * 4                           # query tiles
    assert ctr[1] >= int(mask.sum())                     # P.V blocks: the live ones and, after
                                                         # an unevaluated downward stop, candidates
    causal_blocks = 2 * 2 * (1 + 2 + 3 + 4)
    assert ctr[0] >= 2 * causal_blocks                   # stats pass + at least one solver pass
    assert ctr[2] >= ctr[3]                              # every tile ran >= 1 solver pass


def test_bad_arguments_on_gpu():
    z = torch.zeros((1, 1, 128, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(capi.EntAttnError) as e:
        A.entmax_attn_fwd(z, z, z, 1.5, True)
    assert e.value.status == capi.ENT_EUNSUPPORTED
    z = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(capi.EntAttnError) as e:
        A.entmax_attn_fwd(z, z, z, 2.5, True)
    assert e.value.status == capi.ENT_EINVAL


# ------------------------------------------------------------- full-size workloads
def _sampled_parity(w, seed=0, n_rows=48, tiles=(0, -1), late_keys=64, early_keys=0):
    q, k, v, do = inputs.make_inputs(w, seed)
    gpu = run_gpu(q, k, v, do, w.alpha, w.causal, w.dtype)
    B, H, N, d = w.shape
    T = -(-N // 128)
    g = np.random.default_rng(seed)
    heads = [(0, 0), (B - 1, H - 1)]
    rows = []
    for b, h in heads:
        base = (b * H + h) * N
        rows += [base, base + N - 1] + list(base + g.choice(N, n_rows // 2, replace=False))
    rows = np.array(sorted(set(rows)))
    o_r, tau_r, bmax = oracle.attn_fwd_rows(q, k, v, w.alpha, w.causal, rows)
    check_tau(gpu["tau"].reshape(-1)[rows], tau_r)
    check_o(gpu["o"].reshape(-1, d)[rows], o_r, w.dtype,
            label=f"{w.name} alpha {w.alpha} beta {w.beta} (sampled rows)")
    check_support(q, k, gpu["tau"].reshape(-1)[rows], tau_r, w.alpha, w.causal, rows)
    # whole tiles: the mask row needs every row of the tile
    for b, h in heads:
        for t in tiles:
            t = t % T
            r = (b * H + h) * N + np.arange(t * 128, min(N, t * 128 + 128))
            _, tau_t, bm = oracle.attn_fwd_rows(q, k, v, w.alpha, w.causal, r)
            check_tau(gpu["tau"].reshape(-1)[r], tau_t)
            check_mask(gpu["mask"][b, h, t][None], bm.max(axis=0)[None])
    # backward on sampled rows and keys of the first head
    qh, kh, vh, doh = (a[0, 0] for a in (q, k, v, do))
    keys = sorted(set(range(N - late_keys, N)) | set(g.choice(N, early_keys, replace=False).tolist()))
    qrows = list(range(N - 32, N)) + ([0, 1, 2] if early_keys else [])
    dq_r, dk_k, dv_k = oracle.attn_bwd_head_sampled(qh, kh, vh, doh, w.alpha, w.causal,
                                                    qrows, keys)
    from parity import rel_frob, GRAD_RTOL
    assert rel_frob(gpu["dq"][0, 0, qrows], dq_r) <= GRAD_RTOL
    assert rel_frob(gpu["dk"][0, 0, keys], dk_k) <= GRAD_RTOL
    assert rel_frob(gpu["dv"][0, 0, keys], dv_k) <= GRAD_RTOL
    # sum rules at full size: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head
    dvs = gpu["dv"].astype(np.float64).sum(axis=2)
    dos = do.astype(np.float64).sum(axis=2)
    assert np.abs(dvs - dos).max() <= 2e-2 * np.sqrt(N)
    dks = gpu["dk"].astype(np.float64).sum(axis=2)
    assert np.abs(dks).max() <= 2e-2 * np.abs(gpu["dk"]).astype(np.float64).sum(axis=2).max() + 1e-3
    return gpu


def test_workload_iid_beta_sweep():
    for beta in (1.0, 2.0, 4.0, 8.0):
        _sampled_parity(inputs.WORKLOADS["iid"].replace(beta=beta), early_keys=16)


def test_workload_alpha_sweep():
    for alpha in (1.25, 1.5, 2.0):
        gpu = _sampled_parity(inputs.WORKLOADS["alpha"].replace(alpha=alpha), early_keys=8)
        it = gpu["iters"]
        assert it.max() <= 24 and it.min() >= 1


def test_workload_long_clustered():
    gpu = _sampled_parity(inputs.WORKLOADS["long"], n_rows=32, late_keys=128)
    T = 256
    tri = np.tril_indices(T)
    sparsity = 1.0 - gpu["mask"][:, :, tri[0], tri[1]].mean()
    assert sparsity > 0.6, sparsity


def test_workload_lm():
    _sampled_parity(inputs.WORKLOADS["lm"], early_keys=16)


def test_workload_head_dim_32():
    # the iid shape at d = 32 (run by the d = 64 kernels on zero-filled upper columns)
    _sampled_parity(inputs.WORKLOADS["iid"].replace(d=32, beta=2.0), early_keys=16)
    _sampled_parity(inputs.WORKLOADS["clustered4k"].replace(d=32, span=128), n_rows=32, early_keys=8)


def test_workload_clustered4k_span_sweep():
    # supplementary block-sparsity sweep at the iid shape (cluster span sets the sparsity)
    for span in (128, 2048):
        _sampled_parity(inputs.WORKLOADS["clustered4k"].replace(span=span), n_rows=32, early_keys=8)


@pytest.mark.parametrize("budget", ["-1", "6144"])
def test_histogram_start(monkeypatch, budget):
    # the histogram start of the statistics pass (selected by ENTATTN_HIST_BUDGET, read at
    # each forward call): the same results as the plain-bracket default
    monkeypatch.setenv("ENTATTN_HIST_BUDGET", budget)
    for N, d, causal, alpha in [(300, 64, True, 1.5), (384, 128, False, 2.0),
                                (128, 64, True, 1.25), (384, 128, True, 1.7)]:
        w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=N, d=d, causal=causal, alpha=alpha,
                                             beta=2.0, seed=N + d + 1)
        full_parity(q, k, v, do, alpha, causal, "bf16")
    w, (q, k, v, do) = inputs.small_case(B=1, H=2, N=1000, d=128, causal=True, beta=4.0,
                                         kind="clustered", seed=5)
    full_parity(q, k, v, do, w.alpha, w.causal, "bf16", bwd=False)
    _sampled_parity(inputs.WORKLOADS["alpha"], early_keys=8)
