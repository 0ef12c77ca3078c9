"""The seeded generator's torch path draws the same bits as its numpy path
(the GPU-side harness relies on it for tensors too large to draw on the
host); checked here with torch on the CPU."""
import numpy as np

import synthetic as S


def test_weights_torch_equal_numpy():
    import torch
    a = S.expert_weights_bf16_np(5, 0, 3, 64, 256)
    b = S.expert_weights_bf16_torch(5, 0, 3, 64, 256, "cpu").view(torch.int16).numpy().view(np.uint16)
    assert (a == b).all()


def test_activations_torch_equal_numpy_across_chunks():
    import torch
    a = S.activations_bf16_np(7, 37, 512)
    b = S.activations_bf16_torch(7, 37, 512, "cpu", chunk_rows=8).view(torch.int16).numpy().view(np.uint16)
    assert (a == b).all()
    assert (S.activations_bf16_np(7, 37, 512, rows=5) == a[:5]).all()
