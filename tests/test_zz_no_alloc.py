"""The forward that allocates nothing (entmax_attn_fwd_noalloc), for callers that cannot allocate device
memory: it must give the same outputs as entmax_attn_fwd with a caller workspace, call after call.

Kept in a file of its own that pytest collects last, so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest

from adaptive_sparse_flash_b200 import inputs

from _parity import to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_sparse_flash_b200 import binding as b, build
    build.build()
    b.lib()
    return torch, b


def _outputs(torch, b, Q, shape):
    B, H, n, d = shape
    O = torch.empty_like(Q)
    tau = torch.empty((B, H, n), dtype=torch.float32, device=Q.device)
    mask = torch.empty(b.mask_shape(B, H, n), dtype=torch.int32, device=Q.device)
    return O, tau, mask


def test_noalloc_forward_matches_workspace_forward(env):
    torch, b = env
    L = b.lib()
    shape = (1, 4, 1000, 64)
    arr = inputs.clustered(*shape, centres=32, beta_q=4.0, seed=41, with_dO=False)
    t = to_torch(arr, torch.bfloat16)
    # reference: the regular entry point with a caller-owned workspace
    ws = b.alloc_workspace(*shape)
    O0, tau0, mask0 = _outputs(torch, b, t["Q"], shape)
    b.entmax_attn_fwd(t["Q"], t["K"], t["V"], O0, tau0, mask0, 1.5, True, b.make_opts(ws))
    torch.cuda.synchronize()
    assert b.entmax_attn_check() == 0
    ref = (O0.float().cpu().numpy(), tau0.cpu().numpy(), mask0.cpu().numpy())
    # two calls in a row through the C ABI, no workspace and no opts
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        O1, tau1, mask1 = _outputs(torch, b, t["Q"], shape)
        st = L.entmax_attn_fwd_noalloc(ctypes.c_void_p(t["Q"].data_ptr()), ctypes.c_void_p(t["K"].data_ptr()),
                                       ctypes.c_void_p(t["V"].data_ptr()), ctypes.c_void_p(O1.data_ptr()),
                                       ctypes.c_void_p(tau1.data_ptr()), ctypes.c_void_p(mask1.data_ptr()),
                                       *shape, 1.5, 1, b.ENTMAX_BF16, None, stream)
        assert st == b.ENTMAX_OK, b.entmax_status_str(st)
        torch.cuda.synchronize()
        assert b.entmax_attn_check() == 0
        # the same kernels on the same inputs: identical outputs, whichever memory holds the scratch
        O = O1.float().cpu().numpy()
        assert np.array_equal(O, ref[0]), (call, float(np.abs(O - ref[0]).max()))
        assert np.array_equal(tau1.cpu().numpy(), ref[1]), call
        assert np.array_equal(mask1.cpu().numpy(), ref[2]), call


def test_noalloc_rejects_sizes_beyond_its_scratch(env):
    torch, b = env
    L = b.lib()
    # 1 x 16 x 16384 x 64 needs ~200 MB of workspace, more than the 32 MiB scratch array
    need = b.entmax_attn_workspace_size(1, 16, 16384, 64)
    assert need > b.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = L.entmax_attn_fwd_noalloc(p, p, p, p, p, p, 1, 16, 16384, 64, 1.5, 1, b.ENTMAX_BF16, None, None)
    assert st == b.ENTMAX_ERR_WORKSPACE
