"""Host logic of MetisLinear (no GPU): default rank, sample sizes and shape checks."""

import pytest
import torch


def test_default_rank_is_one_and_a_half_percent(metis_lib):
    from spectral_quantized_gemm_b200.linear import default_rank
    assert default_rank(768, 3072) == 12        # GPT-2 small: 1.5% of 768, rounded up to 4
    assert default_rank(4096, 14336) == 64      # LLaMA-3 8B: 61.4 rounded up to 64
    assert default_rank(14336, 4096) == 64
    assert default_rank(256, 256) == 4
    assert default_rank(8192, 8192) == 64       # capped at the library's maximum rank


def test_sample_sizes(metis_lib):
    from spectral_quantized_gemm_b200.linear import MetisLinear
    layer = MetisLinear(768, 3072)
    assert layer._l_k(8192, sampled=True) == 82          # ceil(1% of 8192)
    assert layer._l_k(768, sampled=False) == 768          # the weight: every row
    assert layer._l_k(1024, sampled=True) == layer.k + layer.s   # never fewer than k + s rows
    assert layer.weight.dtype == torch.float32 and layer.weight.shape == (768, 3072)


def test_shape_and_argument_checks(metis_lib):
    from spectral_quantized_gemm_b200.linear import MetisLinear
    with pytest.raises(ValueError):
        MetisLinear(700, 3072)
    with pytest.raises(ValueError):
        MetisLinear(768, 3072, rounding="down")
    layer = MetisLinear(256, 256)
    with pytest.raises(ValueError):
        layer._check_rows(300)
    with pytest.raises(ValueError):
        layer(torch.zeros(256, 512))              # wrong feature size, caught before any GPU work
