"""Statistics-pass skipping by key-block bounds (bf16 forward; query tiles of at least
64 key blocks).

A key block whose centroid bound lies at or below (lower bound of the row maximum) - 1
for every row of a tile is left out of the statistics pass and of everything after
it.  Such a block holds no p > 0 and no row maximum, so the later passes see the same
blocks and sums: the outputs must be bit-identical with the bound switched off
(ENTATTN_BOUND=0), while the work counters show the blocks it saved."""
import pytest
import torch

from adaptive_sparse_flash_entmax_b200 import attention as A
from adaptive_sparse_flash_entmax_b200 import capi, inputs

from parity import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.load()


# the bound pass runs in query tiles of at least 64 key blocks, so N >= 8192
CASES = [
    ("clustered4k", {"span": 128, "B": 1, "H": 2, "N": 8192}, True),
    ("clustered4k", {"span": 128, "B": 1, "H": 2, "d": 64, "N": 8492}, True),       # ragged tail, d 64
    ("clustered4k", {"span": 64, "B": 1, "H": 1, "causal": False, "N": 8192}, True),  # non-causal
    ("clustered4k", {"span": 128, "B": 1, "H": 2, "d": 32, "N": 8300}, True),       # d 32
    ("long", {"H": 2}, True),
    ("iid", {"B": 1, "H": 2, "N": 8192}, False),
]


def _fwd(w, qd, kd, vd, otilde):
    B, H, N, d = w.shape
    ws = A.workspace(capi.ent_attn_fwd_workspace_size(B, H, N, d, capi.ENT_BF16), qd.device)
    ot = torch.empty(qd.shape, dtype=torch.float32, device=qd.device) if otilde else None
    o, tau, mask, it = A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal, ws=ws, with_iters=True,
                                         otilde=ot)
    ctr = A.read_status(ws)
    return (o, tau, mask, it, ot), ctr


@pytest.mark.parametrize("name,change,skips", CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in c.items())}" for n, c, _ in CASES])
@pytest.mark.parametrize("otilde", [False, True])
def test_bound_changes_work_not_results(name, change, skips, otilde, monkeypatch):
    w = inputs.WORKLOADS[name].replace(**change)
    q, k, v, _ = inputs.make_inputs(w, seed=5)
    qd, kd, vd = (to_dev(a, "bf16") for a in (q, k, v))
    monkeypatch.delenv("ENTATTN_BOUND", raising=False)
    with_bound, c1 = _fwd(w, qd, kd, vd, otilde)
    monkeypatch.setenv("ENTATTN_BOUND", "0")
    without, c0 = _fwd(w, qd, kd, vd, otilde)
    for a, b in zip(with_bound, without):
        if a is not None:
            assert torch.equal(a, b)
    assert c0[6] == 0
    if skips:
        assert c1[6] > 0
        if name == "long":   # long rows: far fewer score products, the bound's own included
            assert c1[0] < 0.5 * c0[0]
    else:
        assert c1[6] == 0
    assert c1[1] == c0[1] and c1[2] == c0[2]   # same live blocks, same solver passes


def test_forward_workspace_guard_bands():
    """The forward writes its key-block bounds inside the workspace it asked for, no further."""
    w = inputs.WORKLOADS["clustered4k"].replace(span=128, B=1, H=3, N=8300)
    q, k, v, _ = inputs.make_inputs(w, seed=9)
    qd, kd, vd = (to_dev(a, "bf16") for a in (q, k, v))
    need = capi.ent_attn_fwd_workspace_size(*w.shape, capi.ENT_BF16)
    G = 4096
    buf = torch.full((need + 2 * G,), 7, dtype=torch.uint8, device="cuda")
    ws = buf[G:G + need]
    assert ws.data_ptr() % 256 == 0
    A.entmax_attn_fwd(qd, kd, vd, w.alpha, w.causal, ws=ws)
    ctr = A.read_status(ws)
    assert ctr[6] > 0
    assert torch.all(buf[:G] == 7) and torch.all(buf[-G:] == 7)
