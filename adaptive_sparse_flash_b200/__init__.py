"""alpha-entmax attention (AdaSplash-2 hot path) for NVIDIA B200, sm_100a.

The compute path lives in the CUDA library `libentmax_attn.so` built from
`csrc/`; `binding` is a thin ctypes layer over its C ABI. Importing this
package does not load the library; `binding.lib()` does, and raises if it is
missing.
"""
__all__ = ["binding", "inputs"]
