"""Host-side checks of the retention (RetNet) input construction: no GPU needed."""

import numpy as np
import torch

import oracle
from mlstm_chunkwise_attention_b200.synthetic import retention_gates, retnet_decays

BF = torch.bfloat16


def test_retention_decays_are_retnets():
    """gamma_h = 1 - 2^(-5 - h); the decay the gates give stays within bf16 rounding of
    it; the input gate is 1 to fp32 rounding."""
    gamma = retnet_decays(8)
    assert float(gamma[0]) == 1 - 2 ** -5 and float(gamma[7]) == 1 - 2 ** -12
    ig, fg = retention_gates(gamma, 1, 4, BF, "cpu")
    g_eff = oracle.sigmoid(fg[0, :, 0].double().numpy())
    # one bf16 step of the logit moves the decay by at most gamma (1 - gamma) 2^-8 * |logit|
    logit = np.log(gamma.numpy() / (1 - gamma.numpy()))
    bound = gamma.numpy() * (1 - gamma.numpy()) * np.abs(logit) * 2.0 ** -8
    assert np.all(np.abs(g_eff - gamma.numpy()) <= bound)
    ig, fg = retention_gates(gamma, 2, 3, BF, "cpu")
    assert ig.shape == fg.shape == (2, 8, 3)
    assert float(np.abs(oracle.logsigmoid(ig.double().numpy())).max()) < 1e-12
