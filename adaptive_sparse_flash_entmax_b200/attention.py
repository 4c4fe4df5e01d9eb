"""PyTorch-facing wrappers of the C ABI (argument marshalling only).

PyTorch supplies device memory and the current stream; every step of the
alpha-entmax attention runs inside libentattn.so.  Tensors are [B, H, N, d],
contiguous, float32 or bfloat16, on one CUDA device.
"""
from __future__ import annotations

import torch

from . import capi

_DTYPES = {torch.float32: capi.ENT_F32, torch.bfloat16: capi.ENT_BF16}


def _stream_handle(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


# The library launches on the calling thread's current CUDA device; every call below
# runs with the tensors' device made current, so tensors on another GPU than the
# current one are handled on theirs.


def _check(*ts):
    t0 = ts[0]
    if t0.dim() != 4:
        raise ValueError(f"expected [B, H, N, d] tensors, got shape {tuple(t0.shape)}")
    if t0.dtype not in _DTYPES:
        raise ValueError(f"dtype {t0.dtype} not supported (float32 or bfloat16)")
    for t in ts:
        if t.shape != t0.shape or t.dtype != t0.dtype or t.device != t0.device:
            raise ValueError("q, k, v (and o, dout) must share shape, dtype and device")
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _raise(st: int, where: str):
    if st != capi.ENT_OK:
        raise capi.EntAttnError(st, where, capi.ent_attn_last_error())


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device workspace of at least ``nbytes`` bytes (256-byte aligned by torch)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def alloc_lists(q):
    """Support-list buffers for ``entmax_attn_fwd(..., lists=)``: (key int32, u float32
    [B, H, N, cap], n uint8 [B, H, N])."""
    B, H, N, _ = q.shape
    cap = capi.ent_attn_list_cap()
    return (torch.empty((B, H, N, cap), dtype=torch.int32, device=q.device),
            torch.empty((B, H, N, cap), dtype=torch.float32, device=q.device),
            torch.empty((B, H, N), dtype=torch.uint8, device=q.device))


def entmax_attn_fwd(q, k, v, alpha: float = 1.5, causal: bool = False, *, with_iters=False,
                    ws: torch.Tensor | None = None, out=None, otilde=None, lists=None):
    """Forward: returns (o, tau, block_mask, iters_or_None).

    ``otilde``: a float32 tensor shaped like q to call ``ent_attn_fwd_otilde`` instead,
    which also fills it with sum_j g_ij v_j / sum_j g_ij (the backward's delta is then
    dO . otilde, see ``entmax_attn_bwd``).  ``lists``: the buffers of ``alloc_lists`` to
    call ``ent_attn_fwd_lists``, which also records every row's (key, u) support list."""
    _check(q, k, v)
    B, H, N, d = q.shape
    dt = _DTYPES[q.dtype]
    T = -(-N // capi.ent_attn_block_size()) if N else 0
    if out is None:
        o = torch.empty_like(q)
        tau = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        mask = torch.empty((B, H, T, T), dtype=torch.uint8, device=q.device)
        iters = torch.empty((B, H, N), dtype=torch.uint8, device=q.device) if with_iters else None
    else:
        o, tau, mask, iters = out
    need = capi.ent_attn_fwd_workspace_size(B, H, N, d, dt)
    if ws is None or ws.numel() < need:
        ws = workspace(need, q.device)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, dt, alpha, causal, o.data_ptr(),
            tau.data_ptr(), mask.data_ptr(), iters.data_ptr() if iters is not None else None)
    tail = (ws.data_ptr(), ws.numel(), _stream_handle(q.device))
    if lists is not None:
        if otilde is not None:
            raise ValueError("otilde and lists are separate forward variants")
        lk, lu, ln = lists
        with torch.cuda.device(q.device):
            st = capi.ent_attn_fwd_lists(*args, lk.data_ptr(), lu.data_ptr(), ln.data_ptr(), *tail)
        _raise(st, "ent_attn_fwd_lists")
    elif otilde is None:
        with torch.cuda.device(q.device):
            st = capi.ent_attn_fwd(*args, *tail)
        _raise(st, "ent_attn_fwd")
    else:
        _check_otilde(otilde, q)
        with torch.cuda.device(q.device):
            st = capi.ent_attn_fwd_otilde(*args, otilde.data_ptr(), *tail)
        _raise(st, "ent_attn_fwd_otilde")
    return o, tau, mask, iters


def _check_otilde(otilde, q):
    if (otilde.dtype != torch.float32 or otilde.shape != q.shape or otilde.device != q.device
            or not otilde.is_contiguous()):
        raise ValueError("otilde must be a contiguous float32 tensor shaped like q, on its device")


def entmax_attn_bwd(q, k, v, o, dout, tau, block_mask, alpha: float = 1.5, causal: bool = False,
                    *, ws: torch.Tensor | None = None, out=None, otilde=None, lists=None):
    """Backward: returns (dq, dk, dv).

    ``otilde``: the tensor a forward with ``otilde=`` filled; the call then goes to
    ``ent_attn_bwd_otilde`` (delta = dO . otilde, no delta pass over the keys).
    ``lists``: the support lists a forward with ``lists=`` filled; the call then goes to
    ``ent_attn_bwd_lists`` (query tiles whose rows all have lists are done from them)."""
    _check(q, k, v, dout)
    B, H, N, d = q.shape
    dt = _DTYPES[q.dtype]
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = out
    need = (capi.ent_attn_bwd_lists_workspace_size if lists is not None
            else capi.ent_attn_bwd_workspace_size)(B, H, N, d, dt)
    if ws is None or ws.numel() < need:
        ws = workspace(need, q.device)
    tail = (dout.data_ptr(), tau.data_ptr(), block_mask.data_ptr(), B, H, N, d, dt, alpha, causal,
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel(),
            _stream_handle(q.device))
    if lists is not None:
        if otilde is not None:
            raise ValueError("otilde and lists are separate backward variants")
        lk, lu, ln = lists
        with torch.cuda.device(q.device):
            st = capi.ent_attn_bwd_lists(q.data_ptr(), k.data_ptr(), v.data_ptr(), lk.data_ptr(),
                                         lu.data_ptr(), ln.data_ptr(), *tail)
        _raise(st, "ent_attn_bwd_lists")
    elif otilde is None:
        with torch.cuda.device(q.device):
            st = capi.ent_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                   o.data_ptr() if o is not None else None, *tail)
        _raise(st, "ent_attn_bwd")
    else:
        _check_otilde(otilde, q)
        with torch.cuda.device(q.device):
            st = capi.ent_attn_bwd_otilde(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          otilde.data_ptr(), *tail)
        _raise(st, "ent_attn_bwd_otilde")
    return dq, dk, dv


def read_status(ws: torch.Tensor) -> list[int]:
    """Counters of the last call that used ``ws`` (synchronises); raises on a timeout flag."""
    with torch.cuda.device(ws.device):
        st, ctr = capi.ent_attn_read_status(ws.data_ptr(), _stream_handle(ws.device))
    _raise(st, "ent_attn_read_status")
    return ctr


class EntmaxAttention(torch.autograd.Function):
    """Autograd wrapper: O = entmax_alpha(Q K^T / sqrt(d)) V.

    With ``delta="otilde"`` the forward also computes otilde (float32, shaped like q:
    B*H*N*d*4 bytes kept for the backward) and the backward takes delta = dO . otilde
    instead of a delta pass over the keys (faster where most blocks are live);
    ``delta="recompute"`` keeps nothing extra and recomputes delta from the scores
    (faster at high block sparsity, and the choice when activation memory is tight);
    ``delta="lists"`` keeps each row's support list (16 keys and u values, 128 bytes per
    row, bf16 inputs) and the backward does every query tile whose rows all have lists
    from them (faster where nearly every row has at most 16 nonzeros)."""

    @staticmethod
    def forward(ctx, q, k, v, alpha, causal, delta):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        if delta not in ("otilde", "recompute", "lists"):
            raise ValueError(f"delta must be 'otilde', 'recompute' or 'lists', not {delta!r}")
        grad = any(ctx.needs_input_grad[:3])
        ot = (torch.empty(q.shape, dtype=torch.float32, device=q.device)
              if delta == "otilde" and grad else None)
        lists = alloc_lists(q) if delta == "lists" and grad else None
        o, tau, mask, _ = entmax_attn_fwd(q, k, v, alpha, causal, otilde=ot, lists=lists)
        lk, lu, ln = lists if lists is not None else (None, None, None)
        ctx.save_for_backward(q, k, v, o, tau, mask, ot, lk, lu, ln)
        ctx.alpha, ctx.causal = alpha, causal
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, tau, mask, ot, lk, lu, ln = ctx.saved_tensors
        lists = (lk, lu, ln) if lk is not None else None
        dq, dk, dv = entmax_attn_bwd(q, k, v, o, do.contiguous(), tau, mask, ctx.alpha, ctx.causal,
                                     otilde=ot, lists=lists)
        return dq, dk, dv, None, None, None


def entmax_attention(q, k, v, alpha: float = 1.5, causal: bool = False, delta: str = "otilde"):
    """Differentiable fused alpha-entmax attention (``delta``: see EntmaxAttention)."""
    return EntmaxAttention.apply(q, k, v, alpha, causal, delta)


# ------------------------------------------------------------ row-wise entmax
SOLVERS = {"hist": capi.ENT_SOLVE_HIST, "halley": capi.ENT_SOLVE_HALLEY,
           "bisect": capi.ENT_SOLVE_BISECT}


def _check_rows(*ts):
    t0 = ts[0]
    if t0.dim() != 2:
        raise ValueError(f"expected [rows, n] tensors, got shape {tuple(t0.shape)}")
    if t0.dtype not in _DTYPES:
        raise ValueError(f"dtype {t0.dtype} not supported (float32 or bfloat16)")
    for t in ts:
        if t.shape != t0.shape or t.dtype != t0.dtype or t.device != t0.device:
            raise ValueError("z, dp must share shape, dtype and device")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")


def entmax_rows_fwd(z, alpha: float = 1.5, solver: str = "hist", *, out=None):
    """Row-wise alpha-entmax of z [rows, n]: returns (p, tau [rows], iters [rows] uint8)."""
    _check_rows(z)
    rows, n = z.shape
    if out is None:
        p = torch.empty_like(z)
        tau = torch.empty(rows, dtype=torch.float32, device=z.device)
        iters = torch.empty(rows, dtype=torch.uint8, device=z.device)
    else:
        p, tau, iters = out
    with torch.cuda.device(z.device):
        st = capi.ent_entmax_rows_fwd(z.data_ptr(), rows, n, _DTYPES[z.dtype], alpha,
                                      SOLVERS[solver], p.data_ptr(), tau.data_ptr(),
                                      iters.data_ptr() if iters is not None else None,
                                      _stream_handle(z.device))
    _raise(st, "ent_entmax_rows_fwd")
    return p, tau, iters


def entmax_rows_bwd(z, tau, dp, alpha: float = 1.5, *, out=None):
    """Gradient w.r.t. z of sum(dp * entmax(z)) for the tau the forward returned."""
    _check_rows(z, dp)
    rows, n = z.shape
    dz = torch.empty_like(z) if out is None else out
    with torch.cuda.device(z.device):
        st = capi.ent_entmax_rows_bwd(z.data_ptr(), tau.data_ptr(), dp.data_ptr(), rows, n,
                                      _DTYPES[z.dtype], alpha, dz.data_ptr(),
                                      _stream_handle(z.device))
    _raise(st, "ent_entmax_rows_bwd")
    return dz
