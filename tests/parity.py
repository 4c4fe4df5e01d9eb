"""Helpers for the GPU-vs-oracle parity tests (test infrastructure).

Tolerances (stated once, used by every parity test):
  tau      |tau_gpu - tau_ref| <= 1e-3 * max(|tau_ref|, 1)
  O        max |O_gpu - O_ref| <= 1e-4 (float32 inputs), 1e-2 (bfloat16) plus
           the bf16 storage half-ulp of O_ref (one contract, `o_excess`, used by
           these tests, the full-size checker and smoke())
  dQ,dK,dV relative Frobenius error <= 2e-2
  support  {x > tau} agrees except where |x - tau_ref| <= 1e-3
  mask     bit-exact except for blocks whose max(x - tau_ref) lies within 1e-3 of 0
"""
from __future__ import annotations

import numpy as np
import torch

TAU_RTOL = 1e-3
O_TOL = {"f32": 1e-4, "bf16": 1e-2}
GRAD_RTOL = 2e-2
BAND = 1e-3

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(TORCH_DTYPE[dtype]).contiguous()


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy() if t.is_floating_point() else t.cpu().numpy()


def run_gpu(q, k, v, do, alpha, causal, dtype, with_bwd=True):
    """Run the CUDA forward (and backward) through the binding; numpy outputs."""
    from adaptive_sparse_flash_entmax_b200 import attention as A
    qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    o, tau, mask, iters = A.entmax_attn_fwd(qd, kd, vd, alpha, causal, with_iters=True)
    out = {"o": to_np(o), "tau": to_np(tau), "mask": to_np(mask), "iters": to_np(iters)}
    if with_bwd:
        dod = to_dev(do, dtype)
        dq, dk, dv = A.entmax_attn_bwd(qd, kd, vd, o, dod, tau, mask, alpha, causal)
        out.update(dq=to_np(dq), dk=to_np(dk), dv=to_np(dv))
    torch.cuda.synchronize()
    return out


def check_tau(tau_gpu, tau_ref):
    err = np.abs(tau_gpu - tau_ref) / np.maximum(np.abs(tau_ref), 1.0)
    assert np.all(np.isfinite(tau_gpu))
    assert err.max() <= TAU_RTOL, f"tau rel err {err.max():.3g}"


def storage_half_ulp(x, dtype):
    """Half a unit in the last place of the output dtype at |x| (0 for float32,
    whose rounding is far below the 1e-4 bound).  bfloat16 keeps 8 significant
    bits: for |x| in [2^e, 2^(e+1)) its half-ulp is 2^(e-8), which is 0.0078 on
    [2, 4) and exceeds the 1e-2 bound from |x| >= 4 on (0.0156), so a bf16 O
    there cannot be stored within 1e-2 at all; its bound is 1e-2 plus this
    storage rounding.  Works on numpy arrays and torch tensors."""
    if dtype != "bf16":
        return x * 0
    if isinstance(x, torch.Tensor):
        ax = torch.clamp(x.abs(), min=torch.finfo(torch.float32).tiny)
        return torch.exp2(torch.floor(torch.log2(ax)) - 8)
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 8)


def o_excess(o_gpu, o_ref, dtype):
    """|O_gpu - O_ref| with the bf16 storage rounding of O_ref taken out: the part
    of the error the computation made.  The contract is o_excess <= O_TOL[dtype]."""
    return abs(o_gpu - o_ref) - storage_half_ulp(o_ref, dtype)


# worst o_excess per label over the session (reported when ENT_PARITY_REPORT is set)
O_REPORT: dict = {}


def check_o(o_gpu, o_ref, dtype, label=None):
    if not o_ref.size:
        return 0.0
    worst = float(o_excess(o_gpu, o_ref, dtype).max())
    if label is not None:
        O_REPORT[label] = max(O_REPORT.get(label, -1.0), worst)
    assert worst <= O_TOL[dtype], f"max |ΔO| beyond storage rounding {worst:.3g} > {O_TOL[dtype]}"
    return worst


def check_mask(mask_gpu, margin_ref):
    """margin_ref: oracle max(x - tau) per block (-inf where nothing is admissible)."""
    want = margin_ref > 0
    decided = np.abs(margin_ref) > BAND
    bad = (mask_gpu.astype(bool) != want) & decided
    assert not bad.any(), f"{bad.sum()} mask entries differ outside the band"
    assert not mask_gpu[np.isneginf(margin_ref)].any(), "mask set on an inadmissible block"


def rel_frob(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / nb if nb > 0 else np.linalg.norm(a)


def check_grads(gpu, ref):
    errs = {}
    for key, r in zip(("dq", "dk", "dv"), ref):
        e = rel_frob(gpu[key].astype(np.float64), r)
        errs[key] = e
        assert e <= GRAD_RTOL, f"{key} rel Frobenius {e:.3g}"
    return errs


def check_support(q, k, tau_gpu_rows, tau_ref_rows, alpha, causal, rows):
    """Support {x > tau} of sampled rows (flat ids): GPU tau vs oracle tau."""
    B, H, N, d = q.shape
    for flat, tg, tr in zip(rows, tau_gpu_rows, tau_ref_rows):
        bh, i = divmod(int(flat), N)
        b, h = divmod(bh, H)
        n = i + 1 if causal else N
        x = (alpha - 1) * (k[b, h, :n].astype(np.float64) @ q[b, h, i].astype(np.float64)) / np.sqrt(d)
        bad = ((x > tg) != (x > tr)) & (np.abs(x - tr) > BAND)
        assert not bad.any(), f"support differs at row {flat}"
