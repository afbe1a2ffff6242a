"""Host-side checks of the PyTorch front end (adaptive_sparse_flash_b200.module): argument validation that
happens before any device call."""
import pytest


def test_module_rejects_unsupported_shapes_and_options():
    import torch
    from adaptive_sparse_flash_b200.module import EntmaxMultiheadAttention
    with pytest.raises(ValueError, match="head size"):
        EntmaxMultiheadAttention(96, 1)               # head size 96
    with pytest.raises(ValueError, match="divisible"):
        EntmaxMultiheadAttention(129, 2)
    with pytest.raises(ValueError, match="num_kv_heads"):
        EntmaxMultiheadAttention(192, 3, num_kv_heads=2)
    with pytest.raises(ValueError, match="alpha"):
        EntmaxMultiheadAttention(128, 2, alpha=1.0)
    m = EntmaxMultiheadAttention(128, 2, num_kv_heads=1)
    assert m.k_proj.out_features == 64 and m.q_proj.out_features == 128
    x = torch.zeros(1, 8, 128)
    with pytest.raises(ValueError, match="key_padding_mask"):
        m(x, x, x, key_padding_mask=torch.zeros(1, 8, dtype=torch.bool))
    with pytest.raises(ValueError, match="need_weights"):
        m(x, x, x, need_weights=True)
    with pytest.raises(ValueError, match="attn_mask"):
        m(x, x, x, attn_mask=torch.zeros(8, 8))
    with pytest.raises(ValueError, match="same sequence length"):
        m(x, torch.zeros(1, 9, 128), torch.zeros(1, 9, 128))


def test_function_rejects_host_tensors():
    import torch
    from adaptive_sparse_flash_b200.module import entmax_attention
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="bf16 CUDA"):
        entmax_attention(q, q, q)
