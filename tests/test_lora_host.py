"""Host logic of LoRASVDLinear (no GPU): parameters, argument checks, checkpoint state."""

import pytest
import torch


def test_parameters_and_defaults(metis_lib):
    from spectral_quantized_gemm_b200.lora_svd import LoRASVDLinear
    layer = LoRASVDLinear(768, 3072)
    assert layer.k == 12                                   # 1.5% of the hidden size, as MetisLinear
    assert layer.realign_every == 2048 and layer.beta == 1.0
    shapes = {name: tuple(p.shape) for name, p in layer.named_parameters()}
    assert shapes == {"W_res": (768, 3072), "L2": (768, 12), "L1": (12, 3072)}
    assert all(p.dtype == torch.float32 for p in layer.parameters())
    assert not layer.aligned and layer.step == 0         # the first forward realigns


def test_argument_checks(metis_lib):
    from spectral_quantized_gemm_b200.lora_svd import LoRASVDLinear
    with pytest.raises(ValueError):
        LoRASVDLinear(700, 3072)
    with pytest.raises(ValueError):
        LoRASVDLinear(768, 3072, beta=0.0)
    with pytest.raises(ValueError):
        LoRASVDLinear(768, 3072, k=65)
    layer = LoRASVDLinear(256, 512, k=8)
    with pytest.raises(ValueError):
        layer(torch.zeros(256, 300))                      # wrong feature size, before any GPU work


def test_checkpoint_state_round_trip(metis_lib):
    from spectral_quantized_gemm_b200.lora_svd import LoRASVDLinear
    a = LoRASVDLinear(256, 512, k=8)
    a.step, a.aligned = 37, True
    b = LoRASVDLinear(256, 512, k=8)
    b.load_state_dict(a.state_dict())
    assert b.step == 37 and b.aligned
    assert torch.equal(b.W_res, a.W_res) and torch.equal(b.L2, a.L2) and torch.equal(b.L1, a.L1)
