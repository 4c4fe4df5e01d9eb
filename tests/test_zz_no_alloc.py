"""ent_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (memory planned ahead of time, or no allocator at hand).  Called through
the C ABI and compared with ent_attn_bwd (which takes a caller workspace) on
two calls in a row.  Both run the same deterministic kernels (no cross-CTA
atomics on the outputs), so the gradients must agree bit for bit; a scratch
array left stale by the previous call would show up as a difference.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = capi.load()
    fn = lib.ent_attn_bwd_noalloc
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp, vp, vp]
    fn.restype = ci
    return fn


@pytest.mark.parametrize("dtype,shape,causal", [("bf16", (2, 3, 384, 128), True),
                                                ("bf16", (1, 2, 300, 64), False),
                                                ("f32", (1, 2, 256, 64), False)])
def test_noalloc_matches_workspace_backward(dtype, shape, causal):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fn = _noalloc_fn()
    B, H, N, d = shape
    w = inputs.Workload("noalloc", B, H, N, d, dtype, causal, 1.5, 2.0, "iid")
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q, k, v, do = (torch.from_numpy(x).to("cuda").to(tdt) for x in inputs.make_inputs(w, seed=11))
    o, tau, mask, _ = A.entmax_attn_fwd(q, k, v, 1.5, causal)
    code = capi.ENT_BF16 if dtype == "bf16" else capi.ENT_F32
    ws = A.workspace(capi.ent_attn_bwd_workspace_size(B, H, N, d, code), q.device)
    ref = A.entmax_attn_bwd(q, k, v, o, do, tau, mask, 1.5, causal, ws=ws)
    ref_counters = A.read_status(ws)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):   # two calls in a row share the library's scratch
        dq, dk, dv = torch.full_like(q, 3.0), torch.full_like(k, 3.0), torch.full_like(v, 3.0)
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                tau.data_ptr(), mask.data_ptr(), B, H, N, d, code, 1.5, int(causal),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), stream)
        assert st == capi.ENT_OK, capi.ent_attn_last_error()
        torch.cuda.synchronize()
        for got, want in zip((dq, dk, dv), ref):
            assert torch.equal(got, want)
        # the fixed array's header: no bounded wait gave up, and the same work was counted
        st, counters = capi.ent_attn_noalloc_read_status(stream)
        assert st == capi.ENT_OK, capi.ent_attn_last_error()
        assert counters == list(ref_counters)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fn = _noalloc_fn()
    fake = 1 << 20   # never dereferenced: the size check comes first
    st = fn(fake, fake, fake, None, fake, fake, fake, 64, 64, 4096, 64, capi.ENT_BF16, 1.5, 1,
            fake, fake, fake, None)
    assert st == capi.ENT_EUNSUPPORTED
    assert "fixed" in capi.ent_attn_last_error()
