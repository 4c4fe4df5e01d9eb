"""Every row and block of every head of the full-size workloads (tests/fullsize.py):
tau in its bracket and at its root, the block mask, O and otilde, in the launch
configuration the bench times.  Complements the oracle's sampled rows and tiles."""
import pytest
import torch

from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from fullsize import check_forward
from parity import O_REPORT, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


CASES = [("iid", {}, True), ("iid", {"beta": 8.0}, False), ("alpha", {"alpha": 1.25}, False),
         ("alpha", {"alpha": 2.0}, True), ("alpha", {}, True), ("long", {}, False),
         ("long", {}, True), ("lm", {}, True), ("clustered4k", {"span": 128}, False),
         ("iid", {"d": 32}, True), ("clustered4k", {"span": 128, "d": 32}, False)]


@pytest.mark.parametrize("name,change,with_otilde", CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in c.items()) or 'default'}"
                              f"-{'otilde' if ot else 'plain'}" for n, c, ot in CASES])
def test_fullsize_every_row(name, change, with_otilde):
    w = inputs.WORKLOADS[name].replace(**change) if change else inputs.WORKLOADS[name]
    q, k, v, _ = inputs.make_inputs(w, seed=3)
    qd, kd, vd = (to_dev(a, w.dtype) for a in (q, k, v))
    del q, k, v
    ot = torch.empty(qd.shape, dtype=torch.float32, device="cuda") if with_otilde else None
    o, tau, mask, _ = A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal, otilde=ot)
    torch.cuda.synchronize()
    res = check_forward(qd, kd, vd, tau, mask, o, w.alpha, w.causal, otilde=ot)
    assert res["rows"] == w.B * w.H * w.N
    key = f"{w.name} alpha {w.alpha} beta {w.beta} (every row, exact p at the kernel's tau)"
    O_REPORT[key] = max(O_REPORT.get(key, -1.0), res["o"])
    print(name, change, res)
