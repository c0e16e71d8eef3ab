"""Host-side checks of the retention (RetNet) helpers: no GPU needed."""

import numpy as np
import torch

from mlstm_chunkwise_attention_b200 import binding

BF = torch.bfloat16


def test_retention_decays_are_retnets():
    """gamma_h = 1 - 2^(-5 - h); the applied decay stays within bf16 rounding of it; the
    input gate is 1 to fp32 rounding."""
    gamma = binding.retnet_decays(8)
    assert float(gamma[0]) == 1 - 2 ** -5 and float(gamma[7]) == 1 - 2 ** -12
    _, _, g_eff = binding.retention_gates(gamma, 1, 4, BF, "cpu")
    # one bf16 step of the logit moves the decay by at most gamma (1 - gamma) 2^-8 * |logit|
    logit = np.log(gamma.numpy() / (1 - gamma.numpy()))
    bound = gamma.numpy() * (1 - gamma.numpy()) * np.abs(logit) * 2.0 ** -8
    assert np.all(np.abs(g_eff.numpy() - gamma.numpy()) <= bound)
    ig, fg, _ = binding.retention_gates(gamma, 2, 3, BF, "cpu")
    assert ig.shape == fg.shape == (2, 8, 3)
    assert float(torch.nn.functional.logsigmoid(ig.double()).abs().max()) < 1e-12
