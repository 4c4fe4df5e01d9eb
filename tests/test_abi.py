"""The C-ABI library on a machine without a GPU: it builds, loads, exports every
symbol the header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import shutil
import subprocess

import pytest

from adaptive_sparse_flash_entmax_b200 import build, capi


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.load()


def test_exports_every_header_symbol(lib):
    names = capi.header_symbols()
    assert {"ent_attn_fwd", "ent_attn_bwd", "ent_attn_fwd_workspace_size",
            "ent_attn_bwd_workspace_size", "ent_attn_read_status", "ent_attn_last_error",
            "ent_attn_block_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_sizes(lib):
    assert capi.ent_attn_block_size() == 128
    assert capi.ent_attn_fwd_workspace_size(4, 16, 4096, 128, capi.ENT_BF16) >= 256
    B, H, N, d = 4, 16, 4096, 128
    # the backward's workspace is its header plus delta (one float per query row), no more
    for (B, H, N, d) in ((4, 16, 4096, 128), (1, 1, 1, 64), (3, 5, 300, 64), (0, 4, 128, 128)):
        rows = B * H * N * 4
        assert capi.ent_attn_bwd_workspace_size(B, H, N, d, capi.ENT_BF16) == 256 + -(-rows // 256) * 256
    assert capi.ent_attn_bwd_workspace_size(-1, 1, 128, 64, capi.ENT_BF16) == 0
    # sequences of >= 64 query tiles also hold the calibrated start's scores: 8 sampled rows
    # of N floats per head, which shorter ones do not need
    short = capi.ent_attn_fwd_workspace_size(2, 3, 63 * 128, 64, capi.ENT_BF16)
    long_ = capi.ent_attn_fwd_workspace_size(2, 3, 64 * 128, 64, capi.ENT_BF16)
    assert long_ - short >= 2 * 3 * 8 * 64 * 128 * 4
    assert long_ % 256 == 0 and short % 256 == 0


FAKE = 1 << 20   # a 16-byte-aligned non-null value; never dereferenced on argument errors


def fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, B=1, H=1, N=128, d=64, dtype=capi.ENT_BF16, alpha=1.5,
             causal=1, o=FAKE, tau=FAKE, block_mask=FAKE, iters=None, ws=FAKE, ws_bytes=1 << 30,
             stream=None)
    a.update(kw)
    return capi.ent_attn_fwd(**a)


def bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=None, dout=FAKE, tau=FAKE, block_mask=FAKE, B=1, H=1,
             N=128, d=64, dtype=capi.ENT_BF16, alpha=1.5, causal=1, dq=FAKE, dk=FAKE, dv=FAKE,
             ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return capi.ent_attn_bwd(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(alpha=1.0), capi.ENT_EINVAL),
    (dict(alpha=2.5), capi.ENT_EINVAL),
    (dict(alpha=float("nan")), capi.ENT_EINVAL),
    (dict(d=96), capi.ENT_EUNSUPPORTED),
    (dict(dtype=7), capi.ENT_EINVAL),
    (dict(N=-1), capi.ENT_EINVAL),
    (dict(causal=2), capi.ENT_EINVAL),
    (dict(q=None), capi.ENT_EINVAL),
    (dict(o=FAKE + 4), capi.ENT_EINVAL),
    (dict(ws=None), capi.ENT_EINVAL),
    (dict(ws_bytes=16), capi.ENT_EINVAL),
    (dict(N=200000), capi.ENT_EUNSUPPORTED),
])
def test_fwd_argument_errors(lib, kw, code):
    assert fwd(**kw) == code
    assert capi.ent_attn_last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(alpha=0.5), capi.ENT_EINVAL),
    (dict(d=256), capi.ENT_EUNSUPPORTED),
    (dict(tau=None), capi.ENT_EINVAL),
    (dict(dq=FAKE + 8), capi.ENT_EINVAL),
    (dict(ws_bytes=512), capi.ENT_EINVAL),   # needs 256 + 128 * 4
])
def test_bwd_argument_errors(lib, kw, code):
    assert bwd(**kw) == code
    assert capi.ent_attn_last_error()


def test_missing_library_fails_loudly(tmp_path):
    saved = capi._lib
    try:
        capi._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            capi.load(str(tmp_path / "libentattn.so"))
    finally:
        capi._lib = saved


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """include/entattn.h is plain C99: a C program using every entry point compiles,
    links against libentattn.so and gets the argument errors without a GPU."""
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(capi.LIB_PATH)
    exe = tmp_path / "abi_from_c"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic",
                    "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c", "abi_from_c.c"),
                    "-L", libdir, "-lentattn", "-Wl,-rpath," + libdir, "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "abi from C ok" in r.stdout


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_otilde_argument_errors(lib, which):
    if which == "fwd":
        args = dict(q=FAKE, k=FAKE, v=FAKE, B=1, H=1, N=128, d=64, dtype=capi.ENT_BF16,
                    alpha=1.5, causal=1, o=FAKE, tau=FAKE, block_mask=FAKE, iters=None,
                    otilde=None, ws=FAKE, ws_bytes=1 << 30, stream=None)
        call = capi.ent_attn_fwd_otilde
    else:
        args = dict(q=FAKE, k=FAKE, v=FAKE, otilde=None, dout=FAKE, tau=FAKE, block_mask=FAKE,
                    B=1, H=1, N=128, d=64, dtype=capi.ENT_BF16, alpha=1.5, causal=1, dq=FAKE,
                    dk=FAKE, dv=FAKE, ws=FAKE, ws_bytes=1 << 30, stream=None)
        call = capi.ent_attn_bwd_otilde
    assert call(**args) == capi.ENT_EINVAL                 # null otilde
    assert "otilde" in capi.ent_attn_last_error()
    assert call(**dict(args, otilde=FAKE + 4)) == capi.ENT_EINVAL   # misaligned
    assert call(**dict(args, d=48, otilde=FAKE)) == capi.ENT_EUNSUPPORTED
