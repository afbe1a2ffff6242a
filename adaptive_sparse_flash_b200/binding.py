"""Thin ctypes binding over libentmax_attn.so (the C ABI in include/entmax_attn.h).

Functions here have the same names as the C entry points. They marshal torch
tensors into pointers and sizes, pick the current CUDA stream, and raise
`EntmaxError` on a non-OK status. Every step of the computation runs in the
library's CUDA kernels; there is no other code path. Loading fails loudly when
the library is missing.
"""
from __future__ import annotations

import ctypes
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libentmax_attn.so")

ENTMAX_OK = 0
ENTMAX_ERR_INVALID = 1
ENTMAX_ERR_UNSUPPORTED = 2
ENTMAX_ERR_ALIGN = 3
ENTMAX_ERR_CUDA = 4
ENTMAX_ERR_TIMEOUT = 5
ENTMAX_ERR_WORKSPACE = 6
ENTMAX_BF16 = 0
ENTMAX_FP32 = 1

# every symbol the header declares
EXPORTS = (
    "entmax_attn_workspace_size",
    "entmax_attn_fwd",
    "entmax_attn_bwd",
    "softmax_attn_fwd",
    "softmax_attn_bwd",
    "entmax_attn_check",
    "entmax_attn_selftest_timeout",
    "entmax_status_str",
    "entmax_attn_version",
    "entmax_attn_fwd_noalloc",
    "entmax_attn_saved_size",
    "entmax_attn_scratch_size",
    "softmax_attn_workspace_size",
)


class EntmaxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {entmax_status_str(status)} (status {status})")


class EntmaxStats(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_ulonglong),
        ("steps", ctypes.c_ulonglong),
        ("fallbacks", ctypes.c_ulonglong),
        ("step_hist", ctypes.c_ulonglong * 9),
        ("causal_blocks", ctypes.c_ulonglong),
        ("candidate_blocks", ctypes.c_ulonglong),
        ("nonzero_blocks", ctypes.c_ulonglong),
        ("sweeps", ctypes.c_ulonglong),
        ("overflow_rows", ctypes.c_ulonglong),
        ("support", ctypes.c_ulonglong),
    ]


STATS_WORDS = ctypes.sizeof(EntmaxStats) // 8


class EntmaxOpts(ctypes.Structure):
    _fields_ = [
        ("scale", ctypes.c_float),
        ("mask_block", ctypes.c_int),
        ("hist_bins", ctypes.c_int),
        ("init_mode", ctypes.c_int),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("stats", ctypes.c_void_p),
        ("tau_hist", ctypes.c_void_p),
        ("steps", ctypes.c_void_p),
        ("events", ctypes.c_void_p),
        ("num_events", ctypes.c_int),
        ("scratch", ctypes.c_void_p),
        ("scratch_bytes", ctypes.c_size_t),
        ("alpha", ctypes.c_float),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once). Raises if the shared object is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m adaptive_sparse_flash_b200.build` "
            "(or __graft_entry__.build()); there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    op = ctypes.POINTER(EntmaxOpts)
    for nm in ("entmax_attn_workspace_size", "entmax_attn_saved_size", "entmax_attn_scratch_size",
               "softmax_attn_workspace_size"):
        getattr(L, nm).argtypes = [i, i, i, i, i, op]
        getattr(L, nm).restype = sz
    L.entmax_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, op, vp]
    L.entmax_attn_fwd.restype = i
    L.entmax_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, op, vp]
    L.entmax_attn_bwd.restype = i
    L.softmax_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, op, vp]
    L.softmax_attn_fwd.restype = i
    L.softmax_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, op, vp]
    L.softmax_attn_bwd.restype = i
    L.entmax_attn_check.argtypes = [vp]
    L.entmax_attn_check.restype = i
    L.entmax_attn_selftest_timeout.argtypes = [i, vp]
    L.entmax_attn_selftest_timeout.restype = i
    L.entmax_status_str.argtypes = [i]
    L.entmax_status_str.restype = ctypes.c_char_p
    L.entmax_attn_version.argtypes = []
    L.entmax_attn_version.restype = i
    L.entmax_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, op, vp]
    L.entmax_attn_fwd_noalloc.restype = i

    _lib = L
    return L


def entmax_status_str(status: int) -> str:
    return lib().entmax_status_str(int(status)).decode()


def _check(status: int, where: str):
    if status != ENTMAX_OK:
        raise EntmaxError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return ENTMAX_BF16
    if t.dtype == torch.float32:
        return ENTMAX_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_opts(workspace=None, *, scale=0.0, mask_block=0, hist_bins=0, init_mode=0,
              stats=None, tau_hist=None, steps=None, events=None, scratch=None, alpha=0.0) -> EntmaxOpts:
    """Options block. `events`: torch.cuda.Event objects (already recorded once, so that their CUDA handles
    exist) that the call records around its kernel launches (include/entmax_attn.h, per-kernel timing)."""
    o = EntmaxOpts()
    o.scale = float(scale)
    o.mask_block = int(mask_block)
    o.hist_bins = int(hist_bins)
    o.init_mode = int(init_mode)
    o.alpha = float(alpha)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    if scratch is not None:
        o.scratch = scratch.data_ptr()
        o.scratch_bytes = scratch.numel() * scratch.element_size()
    o.stats = None if stats is None else stats.data_ptr()
    o.tau_hist = None if tau_hist is None else tau_hist.data_ptr()
    o.steps = None if steps is None else steps.data_ptr()
    if events:
        arr = (ctypes.c_void_p * len(events))(*[int(e.cuda_event) for e in events])
        o.events = ctypes.cast(arr, ctypes.c_void_p)
        o.num_events = len(events)
        o._keep = arr  # the handle array must outlive the call
    return o


def entmax_attn_workspace_size(B, H, n, d, dtype_code=ENTMAX_BF16, opts: EntmaxOpts | None = None) -> int:
    return int(lib().entmax_attn_workspace_size(B, H, n, d, dtype_code,
                                                 None if opts is None else ctypes.byref(opts)))


def entmax_attn_saved_size(B, H, n, d, dtype_code=ENTMAX_BF16, opts: EntmaxOpts | None = None) -> int:
    return int(lib().entmax_attn_saved_size(B, H, n, d, dtype_code, None if opts is None else ctypes.byref(opts)))


def entmax_attn_scratch_size(B, H, n, d, dtype_code=ENTMAX_BF16, opts: EntmaxOpts | None = None) -> int:
    return int(lib().entmax_attn_scratch_size(B, H, n, d, dtype_code, None if opts is None else ctypes.byref(opts)))


def softmax_attn_workspace_size(B, H, n, d, dtype_code=ENTMAX_BF16, opts: EntmaxOpts | None = None) -> int:
    return int(lib().softmax_attn_workspace_size(B, H, n, d, dtype_code,
                                                  None if opts is None else ctypes.byref(opts)))


def alloc_workspace(B, H, n, d, dtype_code=ENTMAX_BF16, device="cuda", opts=None, part="whole"):
    """Device buffer for the workspace: part "whole" (saved + scratch in one buffer), "saved" or "scratch";
    "softmax" for the dense baseline's calls (no U V)."""
    import torch
    size_fn = {"whole": entmax_attn_workspace_size, "saved": entmax_attn_saved_size,
               "scratch": entmax_attn_scratch_size, "softmax": softmax_attn_workspace_size}[part]
    nbytes = size_fn(B, H, n, d, dtype_code, opts)
    if nbytes == 0:
        raise EntmaxError(ENTMAX_ERR_INVALID, size_fn.__name__)
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def mask_shape(B, H, n, mask_block=64):
    nb = (n + mask_block - 1) // mask_block
    return (B, H, nb, (nb + 31) // 32)


def entmax_attn_fwd(Q, K, V, O, tau, block_mask, alpha, causal, opts: EntmaxOpts, stream=None):
    """Raw forward: all tensors preallocated by the caller ([B,H,n,d], tau fp32 [B,H,n], mask int32)."""
    B, H, n, d = Q.shape
    st = lib().entmax_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(tau), _ptr(block_mask),
                               B, H, n, d, float(alpha), int(causal), _dtype_code(Q),
                               ctypes.byref(opts), _stream(stream))
    _check(st, "entmax_attn_fwd")


def entmax_attn_bwd(Q, K, V, O, dO, tau, block_mask, dQ, dK, dV, alpha, causal, opts: EntmaxOpts, stream=None):
    B, H, n, d = Q.shape
    st = lib().entmax_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(tau), _ptr(block_mask),
                               _ptr(dQ), _ptr(dK), _ptr(dV), B, H, n, d, float(alpha), int(causal),
                               _dtype_code(Q), ctypes.byref(opts), _stream(stream))
    _check(st, "entmax_attn_bwd")


def softmax_attn_fwd(Q, K, V, O, lse, causal, opts: EntmaxOpts | None = None, stream=None):
    B, H, n, d = Q.shape
    st = lib().softmax_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), B, H, n, d, int(causal),
                                _dtype_code(Q), None if opts is None else ctypes.byref(opts), _stream(stream))
    _check(st, "softmax_attn_fwd")


def softmax_attn_bwd(Q, K, V, O, dO, lse, dQ, dK, dV, causal, opts: EntmaxOpts, stream=None):
    B, H, n, d = Q.shape
    st = lib().softmax_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse), _ptr(dQ), _ptr(dK),
                                _ptr(dV), B, H, n, d, int(causal), _dtype_code(Q), ctypes.byref(opts),
                                _stream(stream))
    _check(st, "softmax_attn_bwd")


NOALLOC_SCRATCH_BYTES = 32 << 20  # size of the library's scratch array used by entmax_attn_fwd_noalloc


def entmax_attn_fwd_noalloc(Q, K, V, O, tau, block_mask, alpha, causal, opts: EntmaxOpts | None = None, stream=None):
    """Forward that allocates nothing: the library's fixed scratch array replaces the workspace."""
    B, H, n, d = Q.shape
    st = lib().entmax_attn_fwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(tau), _ptr(block_mask),
                                       B, H, n, d, float(alpha), int(causal), _dtype_code(Q),
                                       None if opts is None else ctypes.byref(opts), _stream(stream))
    _check(st, "entmax_attn_fwd_noalloc")


def entmax_attn_check(stream=None) -> int:
    return int(lib().entmax_attn_check(_stream(stream)))


def entmax_attn_selftest_timeout(limit_us: int, stream=None):
    _check(lib().entmax_attn_selftest_timeout(int(limit_us), _stream(stream)), "entmax_attn_selftest_timeout")


# ---------------------------------------------------------------------------------------------
# Allocating helpers (torch owns the memory; the library only computes)
# ---------------------------------------------------------------------------------------------

class EntmaxForward:
    """Outputs of `forward` plus what `backward` needs (workspace, options)."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def forward(Q, K, V, alpha, causal=True, *, scale=0.0, mask_block=0, hist_bins=0, init_mode=0,
            with_stats=False, with_debug=False, separate_scratch=False, stream=None) -> EntmaxForward:
    """Forward with buffers from torch. With separate_scratch, only the workspace's saved part is kept for the
    backward (the scratch is a transient buffer of this call, and the backward takes its own)."""
    import torch
    B, H, n, d = Q.shape
    dev = Q.device
    mb = mask_block or 64
    code = _dtype_code(Q)
    probe = make_opts(scale=scale, mask_block=mask_block, hist_bins=hist_bins, init_mode=init_mode, alpha=alpha)
    ws = alloc_workspace(B, H, n, d, code, dev, probe, part="saved" if separate_scratch else "whole")
    scratch = alloc_workspace(B, H, n, d, code, dev, probe, part="scratch") if separate_scratch else None
    O = torch.empty_like(Q)
    tau = torch.empty((B, H, n), dtype=torch.float32, device=dev)
    mask = torch.empty(mask_shape(B, H, n, mb), dtype=torch.int32, device=dev)
    stats = torch.zeros(STATS_WORDS, dtype=torch.int64, device=dev) if with_stats else None
    tau_hist = torch.empty((B, H, n), dtype=torch.float32, device=dev) if with_debug else None
    steps = torch.empty((B, H, n), dtype=torch.uint8, device=dev) if with_debug else None
    opts = make_opts(ws, scale=scale, mask_block=mask_block, hist_bins=hist_bins, init_mode=init_mode,
                     stats=stats, tau_hist=tau_hist, steps=steps, scratch=scratch)
    entmax_attn_fwd(Q, K, V, O, tau, mask, alpha, causal, opts, stream)
    if separate_scratch:
        opts = make_opts(ws, scale=scale, mask_block=mask_block, hist_bins=hist_bins, init_mode=init_mode)
    return EntmaxForward(O=O, tau=tau, mask=mask, workspace=ws, opts=opts, stats=stats, tau_hist=tau_hist,
                         steps=steps, alpha=alpha, causal=causal, separate=separate_scratch,
                         keep=(stats, tau_hist, steps))


def backward(Q, K, V, fwd: EntmaxForward, dO, stream=None):
    import torch
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    dK = torch.empty(K.shape, dtype=torch.float32, device=K.device)
    dV = torch.empty(V.shape, dtype=torch.float32, device=V.device)
    opts = fwd.opts
    if getattr(fwd, "separate", False):
        B, H, n, d = Q.shape
        scratch = alloc_workspace(B, H, n, d, _dtype_code(Q), Q.device, fwd.opts, part="scratch")
        opts = EntmaxOpts.from_buffer_copy(fwd.opts)
        opts.scratch = scratch.data_ptr()
        opts.scratch_bytes = scratch.numel()
    entmax_attn_bwd(Q, K, V, fwd.O, dO, fwd.tau, fwd.mask, dQ, dK, dV, fwd.alpha, fwd.causal, opts, stream)
    return dQ, dK, dV


def stats_dict(stats_tensor) -> dict:
    v = [int(x) for x in stats_tensor.cpu().tolist()]
    names = ["rows", "steps", "fallbacks"] + [f"step_hist_{i}" for i in range(9)] + \
        ["causal_blocks", "candidate_blocks", "nonzero_blocks", "sweeps", "overflow_rows", "support"]
    return dict(zip(names, v))


def softmax_forward(Q, K, V, causal=True, workspace=None, stream=None):
    """Dense softmax baseline forward. With a workspace (allocated here when None) d = 64 runs on the
    fp16 kernels; pass workspace=False for the bf16 kernel."""
    import torch
    B, H, n, d = Q.shape
    O = torch.empty_like(Q)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = alloc_workspace(B, H, n, d, _dtype_code(Q), Q.device, part="softmax")
    opts = make_opts(workspace) if workspace is not False else None
    softmax_attn_fwd(Q, K, V, O, lse, causal, opts, stream)
    return O, lse


def softmax_backward(Q, K, V, O, lse, dO, causal=True, workspace=None, stream=None):
    import torch
    B, H, n, d = Q.shape
    if workspace is None:
        workspace = alloc_workspace(B, H, n, d, _dtype_code(Q), Q.device, part="softmax")
    opts = make_opts(workspace)
    dQ, dK, dV = (torch.empty(Q.shape, dtype=torch.float32, device=Q.device) for _ in range(3))
    softmax_attn_bwd(Q, K, V, O, dO, lse, dQ, dK, dV, causal, opts, stream)
    return dQ, dK, dV


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
