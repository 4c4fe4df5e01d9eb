"""Full-size self-consistency of a forward on every row and block of every head.

Test infrastructure (torch arithmetic in float32 on the device of the inputs; no
oracle).  The oracle checks sampled rows and whole tiles at the full sizes; this
checks properties that hold at any size, for all of them, in the tolerances of
tests/parity.py:
  bracket  m - 1 <= tau <= m - n^(1-alpha) (tau of the kernel, m the row maximum of x)
  tau      the Newton distance |f(tau)| / |f'(tau)| to the root is <= 1e-3 max(1, |tau|)
           (the tau tolerance, to first order), f(tau) = sum_j (x_j - tau)_+^gamma - 1
  mask     bit-exact against max(x - tau) > 0 per 128 x 128 block except inside the
           1e-3 band, and 0 on every block with no admissible pair
  O        |O - sum_j p_j v_j| <= 1e-2 plus the bf16 storage half-ulp of the reference
  otilde   |otilde - sum_j g_j v_j / sum_j g_j| <= 2 * 2^-8 * (max over the support of
           |v_j|_inf + |otilde|_inf) + 1e-3 (g is rounded to bf16 for the product:
           2^-8 relative per weight, redistributed by the normalisation), on rows with
           no score inside the band
Scores are x = (alpha - 1) q.k / sqrt(d) in float32 (no TF32) from the same bf16 or
float32 inputs.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F

BLK = 128
BAND = 1e-3


from parity import O_TOL, o_excess


def check_forward(q, k, v, tau, mask, o, alpha, causal, otilde=None, chunk=512):
    """Worst values of every check over all heads (see the module docstring); raises
    AssertionError on the first violation."""
    assert chunk % BLK == 0
    prev_tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        return _check(q, k, v, tau, mask, o, alpha, causal, otilde, chunk)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev_tf32


def _check(q, k, v, tau, mask, o, alpha, causal, otilde, chunk):
    B, H, N, d = q.shape
    T = -(-N // BLK)
    gamma = 1.0 / (alpha - 1.0)
    cx = (alpha - 1.0) / math.sqrt(d)
    dev = q.device
    cols = torch.arange(N, device=dev)
    worst = {"bracket": 0.0, "newton": 0.0, "o": 0.0, "otilde": 0.0, "band_rows": 0,
             "rows": 0, "nnz": 0, "admissible": 0}
    for b in range(B):
        for h in range(H):
            K, V = k[b, h].float(), v[b, h].float()
            vinf = V.abs().amax(dim=1)                       # |v_j|_inf per key
            bm = torch.full((T, T), -math.inf, device=dev)
            for r0 in range(0, N, chunk):
                r1 = min(N, r0 + chunk)
                R = r1 - r0
                rows = torch.arange(r0, r1, device=dev)
                x = cx * (q[b, h, r0:r1].float() @ K.T)
                if causal:
                    x = x.masked_fill(cols[None, :] > rows[:, None], -math.inf)
                t = tau[b, h, r0:r1].float()
                n = (rows + 1).float() if causal else torch.full_like(t, float(N))
                m = x.amax(dim=1)
                # bracket
                slack = 1e-4 * torch.clamp(m.abs(), min=1.0)
                lo, hi = m - 1.0, m - torch.pow(n, 1.0 - alpha)
                viol = torch.clamp(lo - slack - t, min=0) + torch.clamp(t - hi - slack, min=0)
                worst["bracket"] = max(worst["bracket"], viol.max().item())
                assert viol.max().item() == 0.0, f"tau outside its bracket (head {b},{h})"
                # Newton distance to the root
                u = x - t[:, None]
                sup = u > 0
                up = torch.clamp(u, min=0)
                f = torch.pow(up, gamma).sum(dim=1) - 1.0
                g = torch.where(sup, torch.pow(up, gamma - 1.0), torch.zeros_like(up))
                sg = g.sum(dim=1)
                dist = f.abs() / (gamma * sg) / torch.clamp(t.abs(), min=1.0)
                worst["newton"] = max(worst["newton"], dist.max().item())
                assert dist.max().item() <= 1e-3, f"tau off its root (head {b},{h}): {dist.max().item()}"
                worst["nnz"] += int(sup.sum().item())
                worst["admissible"] += int(n.sum().item())
                worst["rows"] += R
                # block maxima of x - tau, rows gathered into their tiles
                upad = F.pad(u, (0, T * BLK - N), value=-math.inf).view(R, T, BLK).amax(dim=2)
                rpad = -(-R // BLK) * BLK - R
                tmax = F.pad(upad, (0, 0, 0, rpad), value=-math.inf).view(-1, BLK, T).amax(dim=1)
                bm[r0 // BLK: r0 // BLK + tmax.shape[0]] = tmax
                # O = P V with exact p
                o_ref = torch.pow(up, gamma) @ V
                odt = "bf16" if o.dtype == torch.bfloat16 else "f32"
                err = o_excess(o[b, h, r0:r1].float(), o_ref, odt)
                worst["o"] = max(worst["o"], err.max().item())
                assert err.max().item() <= O_TOL[odt], f"O off (head {b},{h}): {err.max().item()}"
                if otilde is not None:
                    ot_ref = (g @ V) / sg[:, None]
                    ot = otilde[b, h, r0:r1]
                    clear = ~((u.abs() <= BAND).any(dim=1))
                    vmax = torch.where(sup, vinf[None, :], torch.zeros_like(u)).amax(dim=1)
                    bound = 2.0 * 2.0 ** -8 * (vmax + ot.abs().amax(dim=1)) + 1e-3
                    if o.dtype != torch.bfloat16:
                        bound = torch.full_like(bound, 1e-4)
                    e = (ot - ot_ref).abs().amax(dim=1)
                    worst["band_rows"] += int((~clear).sum().item())
                    if clear.any():
                        worst["otilde"] = max(worst["otilde"], (e - bound)[clear].max().item())
                        assert bool((e <= bound)[clear].all()), f"otilde off (head {b},{h})"
            mk = mask[b, h].bool()
            decided = bm.abs() > BAND
            bad = ((mk != (bm > 0)) & decided) | (mk & torch.isneginf(bm))
            assert not bool(bad.any()), f"{int(bad.sum())} mask entries differ (head {b},{h})"
    return worst
