"""Argument checks of the drop-in interfaces (no GPU needed: they fail before any call)."""
import pytest
import torch

import quantized_attention_fine_b200 as sage


def test_sage_attention_module_configuration_checks():
    with pytest.raises(ValueError):
        sage.SageAttention(head_dim=96)
    with pytest.raises(ValueError):
        sage.SageAttention(quant_mode="qk_int4_pv_fp8")
    with pytest.raises(ValueError):
        sage.SageAttention(tensor_layout="BHND")
    a = sage.SageAttention(head_dim=64, is_causal=True, quant_mode="qk_int8_pv_fp16")
    assert a.quant_mode == "qk_int8_pv_fp16" and a.is_causal
    q = torch.zeros(1, 2, 8, 128)
    with pytest.raises(ValueError):   # head dim differs from the configured one
        a(q, q, q)


def test_sdpa_signature_refuses_what_the_method_does_not_define():
    q = torch.zeros(1, 4, 8, 64)
    k = torch.zeros(1, 2, 8, 64)
    with pytest.raises(NotImplementedError):
        sage.scaled_dot_product_attention(q, q, q, attn_mask=torch.ones(8, 8, dtype=torch.bool))
    with pytest.raises(NotImplementedError):
        sage.scaled_dot_product_attention(q, q, q, dropout_p=0.1)
    with pytest.raises(ValueError):   # fewer key heads without enable_gqa, as in torch
        sage.scaled_dot_product_attention(q, k, k)
    with pytest.raises(ValueError):
        sage.scaled_dot_product_attention(q, q, q, quant_mode="fp4")
