"""Retention (RetNet, a constant per-head decay) through the mLSTMsig kernels.

With log i = 0 and log f = log gamma, the SIG cell is retention:
h_t = sum_{s <= t} gamma^(t - s) (q_t . k_s / sqrt(d)) v_s (flash-linear-attention
README, RetNet row of the model table and the retention timing table; the
mLSTM with constant gates).  The reference here is that closed form and its
gradients in fp64, with the decay the kernels actually apply (the gate
preactivations are stored in the I/O dtype).
"""

import numpy as np
import pytest
import torch

import oracle
from mlstm_chunkwise_attention_b200 import binding
from mlstm_chunkwise_attention_b200.synthetic import retention_gates, retnet_decays
from _parity import TOL, inputs, np64, relerr

pytestmark = pytest.mark.gpu

BF, F32 = torch.bfloat16, torch.float32

# name, dtype, chunk, T  (chunk 64: CUDA cores; 128: chunk-128 kernel; 256: large-chunk kernel)
CASES = [
    ("fp32_chunk64", F32, 64, 200),
    ("bf16_chunk128", BF, 128, 300),
    ("bf16_chunk256_ragged", BF, 256, 700),
]


def retention_closed_form(q, k, v, dh, gamma):
    """h and the gradients of sum(dh * h) for one head, fp64, O(T^2)."""
    T, d = q.shape
    lag = np.arange(T)[:, None] - np.arange(T)[None, :]
    D = np.where(lag >= 0, gamma ** np.clip(lag, 0, None), 0.0)
    A = (q @ k.T) / np.sqrt(d) * D
    h = A @ v
    dA = (dh @ v.T) * D
    return {"h": h, "dq": dA @ k / np.sqrt(d), "dk": dA.T @ q / np.sqrt(d), "dv": A.T @ dh}


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_retention_matches_closed_form(case):
    name, dt, L, T = case
    B, NH, d = 1, 4, 128 if dt == BF else 64
    cpu = inputs(B, NH, T, d, d, seed=41, dtype=dt)
    dev = {k: v.cuda() for k, v in cpu.items()}
    gamma = retnet_decays(NH)
    ig, fg = retention_gates(gamma, B, T, dt, "cuda")
    # the decay the kernels apply: the sigmoid of the stored forget preactivation
    gamma_eff = oracle.sigmoid(fg[0, :, 0].double().cpu().numpy())
    h, saved = binding.forward(dev["q"], dev["k"], dev["v"], ig, fg, L, binding.SIG,
                               keep_saved=True)
    g = binding.backward(dev["q"], dev["k"], dev["v"], ig, fg, h, dev["dh"], saved, L, binding.SIG)
    binding.check_device()
    tol = TOL[dt]
    for hh in range(NH):
        ref = retention_closed_form(np64(cpu["q"][0, hh]), np64(cpu["k"][0, hh]),
                                    np64(cpu["v"][0, hh]), np64(cpu["dh"][0, hh]),
                                    float(gamma_eff[hh]))
        assert relerr(np64(h[0, hh]), ref["h"]) <= tol, f"h head {hh}"
        for key in ("dq", "dk", "dv"):
            err = relerr(np64(g[key][0, hh]), ref[key])
            assert err <= tol, f"{key} head {hh}: {err:.3e}"
