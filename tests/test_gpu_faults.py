"""Failure detection without a GPU fault: bounded device waits report a status, bad arguments are
rejected on the host. Nothing here faults, traps or hangs the GPU."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_sparse_flash_b200 import binding as b, build
    build.build()
    b.lib()
    return b


def test_bounded_wait_reports_timeout(lib):
    b = lib
    assert b.entmax_attn_check() == b.ENTMAX_OK
    b.entmax_attn_selftest_timeout(2000)       # waits 2 ms on a barrier nobody arrives at
    assert b.entmax_attn_check() == b.ENTMAX_ERR_TIMEOUT
    assert b.entmax_attn_check() == b.ENTMAX_OK  # the status word is cleared by the read


def test_context_usable_after_timeout(lib):
    import torch
    b = lib
    b.entmax_attn_selftest_timeout(1000)
    assert b.entmax_attn_check() == b.ENTMAX_ERR_TIMEOUT
    q = torch.randn(1, 1, 64, 64, device="cuda").to(torch.bfloat16)
    f = b.forward(q, q, q, 1.5, True)
    torch.cuda.synchronize()
    assert b.entmax_attn_check() == b.ENTMAX_OK
    assert torch.isfinite(f.O.float()).all()


def test_workspace_and_alignment_errors(lib):
    import torch
    b = lib
    q = torch.randn(1, 1, 128, 64, device="cuda").to(torch.bfloat16)
    O = torch.empty_like(q)
    tau = torch.empty(1, 1, 128, device="cuda")
    mask = torch.empty(b.mask_shape(1, 1, 128), dtype=torch.int32, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(b.EntmaxError) as e:
        b.entmax_attn_fwd(q, q, q, O, tau, mask, 1.5, True, b.make_opts(small))
    assert e.value.status == b.ENTMAX_ERR_WORKSPACE
    ws = b.alloc_workspace(1, 1, 128, 64)
    buf = torch.empty(128 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    mis = buf[1:1 + 128 * 64].view(1, 1, 128, 64)   # 2-byte offset: not 16-byte aligned
    with pytest.raises(b.EntmaxError) as e:
        b.entmax_attn_fwd(mis, q, q, O, tau, mask, 1.5, True, b.make_opts(ws))
    assert e.value.status == b.ENTMAX_ERR_ALIGN
    torch.cuda.synchronize()
    assert b.entmax_attn_check() == b.ENTMAX_OK
