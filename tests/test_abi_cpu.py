"""CPU-only checks of the C ABI: the library loads, exports every declared symbol, and rejects bad
arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "entmax_attn.h")


@pytest.fixture(scope="module")
def L():
    from adaptive_sparse_flash_b200 import binding, build
    build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)
    keep = [n for n in names if n.startswith(("entmax_", "softmax_")) and n not in ("entmax_status", "entmax_dtype")]
    return sorted(set(keep))


def test_header_declares_the_binding_exports():
    from adaptive_sparse_flash_b200 import binding
    assert sorted(binding.EXPORTS) == declared_functions()


def test_library_exports_every_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_version_and_status_strings(L):
    from adaptive_sparse_flash_b200 import binding as b
    assert L.entmax_attn_version() == 3
    for s in range(7):
        assert len(b.entmax_status_str(s)) > 0
    assert b.entmax_status_str(99) == "unknown status"


def test_workspace_size(L):
    from adaptive_sparse_flash_b200 import binding as b
    n, d = 16384, 64
    ws = b.entmax_attn_workspace_size(1, 16, n, d)
    rows = 16 * n
    assert ws >= rows * d * 4 + 2 * rows * 4
    assert ws % 256 == 0
    assert b.entmax_attn_workspace_size(1, 16, n, 96) == 0     # d unsupported
    assert b.entmax_attn_workspace_size(0, 16, n, 64) == 0     # empty batch
    assert b.entmax_attn_workspace_size(1, 1, 0, 64) == 0      # empty sequence


def _a256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("B,H,n,d,dt,alpha,with_uv,with_h16", [
    (1, 16, 16384, 64, 0, 1.5, False, True),   # fp16 kernels: no U V, fp16 copies in the scratch
    (1, 16, 16384, 64, 0, 3.0, True, True),    # alpha > 2: bf16 kernels keep U V
    (1, 16, 16384, 64, 0, 0.0, True, True),    # alpha unknown: sized for any alpha
    (2, 16, 4096, 128, 0, 1.5, True, False),   # d = 128: bf16 kernels, no fp16 copies
    (1, 1, 256, 64, 1, 1.5, True, False),      # fp32 inputs: FMA kernel, no fp16 copies
    (3, 5, 1000, 64, 0, 2.0, False, True),     # ragged n
])
def test_workspace_parts(L, B, H, n, d, dt, alpha, with_uv, with_h16):
    """The saved and scratch parts hold exactly the buffers the header lists for the call's kernels."""
    from adaptive_sparse_flash_b200 import binding as b
    o = b.make_opts(alpha=alpha)
    o.mask_block = 32 if dt == 1 else 0
    mb = 32 if dt == 1 else 64
    rows, nb = B * H * n, (n + mb - 1) // mb
    rows_pad = B * H * ((n + 63) // 64) * 64
    saved = (_a256(rows * d * 4) if with_uv else 0) + _a256(rows * 4) + _a256(B * H * nb * ((nb + 31) // 32) * 4)
    scratch = 2 * _a256(rows_pad * 4) + _a256(8 * 4) + (4 * _a256(rows * d * 2) if with_h16 else 0)
    assert b.entmax_attn_saved_size(B, H, n, d, dt, o) == saved
    assert b.entmax_attn_scratch_size(B, H, n, d, dt, o) == scratch
    assert b.entmax_attn_workspace_size(B, H, n, d, dt, o) == saved + scratch
    saved_sm = saved - (_a256(rows * d * 4) if with_uv else 0)  # the dense baseline keeps no U V
    assert b.softmax_attn_workspace_size(B, H, n, d, dt, o) == saved_sm + scratch


def _fwd(L, ptr=16, n=64, d=64, alpha=1.5, causal=1, dt=0, ws=True, mask_block=0, bins=0, init_mode=0,
         num_events=0):
    from adaptive_sparse_flash_b200 import binding as b
    o = b.EntmaxOpts()
    o.num_events = num_events
    o.mask_block = mask_block
    o.hist_bins = bins
    o.init_mode = init_mode
    if ws:
        o.workspace = 256
        o.workspace_bytes = 1 << 40
    p = ctypes.c_void_p(ptr) if ptr is not None else None
    return L.entmax_attn_fwd(p, p, p, p, p, p, 1, 1, n, d, alpha, causal, dt, ctypes.byref(o), None)


def test_validation_errors_return_before_launch(L):
    from adaptive_sparse_flash_b200 import binding as b
    # all of these are rejected by host checks; no device call happens
    assert _fwd(L, ptr=None) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, alpha=1.0) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, alpha=float("nan")) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, causal=2) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, n=0) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, d=80) == b.ENTMAX_ERR_UNSUPPORTED
    assert _fwd(L, n=65535 * 128 + 1) == b.ENTMAX_ERR_UNSUPPORTED  # beyond the grid's tile extent
    assert _fwd(L, dt=7) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, mask_block=32) == b.ENTMAX_ERR_UNSUPPORTED      # bf16 path uses 64
    assert _fwd(L, bins=100) == b.ENTMAX_ERR_UNSUPPORTED
    assert _fwd(L, init_mode=5) == b.ENTMAX_ERR_INVALID
    assert _fwd(L, ptr=18) == b.ENTMAX_ERR_ALIGN
    assert _fwd(L, ws=False) == b.ENTMAX_ERR_WORKSPACE
    assert _fwd(L, num_events=3) == b.ENTMAX_ERR_INVALID     # events count without an events array
    assert _fwd(L, num_events=-1) == b.ENTMAX_ERR_INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from adaptive_sparse_flash_b200 import binding as b
    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        b.lib()
