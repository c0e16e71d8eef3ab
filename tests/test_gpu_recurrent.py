"""Recurrent form on the GPU (through the C ABI) against the fp64 oracle.

* one-token steps from the zero state against the oracle's recurrent step;
* the final state of a chunkwise forward against the oracle's chunkwise form,
  then steps that continue the sequence from it against the oracle's recurrent
  forms over the whole sequence (prefill, then generation).
Same tolerances as the chunkwise parity tests (max|err| / max|ref|).
"""

import numpy as np
import pytest
import torch

import oracle
from mlstm_chunkwise_attention_b200 import binding
from _parity import TOL, inputs, np64, relerr

pytestmark = pytest.mark.gpu

SIG, EXP = binding.SIG, binding.EXP
BF, F32 = torch.bfloat16, torch.float32


def _step_all(x, variant, state, T0, T1):
    """Steps for tokens T0..T1-1 of x (device tensors [B, NH, T, d]); returns h [B, NH, T1-T0, d_hv]."""
    B, NH, _, d_qk = x["q"].shape
    d_hv = x["v"].shape[-1]
    other = torch.empty_like(state)
    hs = []
    for t in range(T0, T1):
        sl = lambda a: a[:, :, t].contiguous()
        hs.append(binding.step(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["igate"]), sl(x["fgate"]),
                               state, other, variant))
        state, other = other, state
    binding.check_device()
    return torch.stack(hs, dim=2), state


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("dt,d", [(F32, 64), (BF, 128)], ids=["fp32_d64", "bf16_d128"])
def test_steps_from_zero_state(variant, dt, d):
    B, NH, T = 1, 2, 40
    cpu = inputs(B, NH, T, d, d, seed=61, dtype=dt, ig_mean=-1.0)
    dev = {k: v.cuda() for k, v in cpu.items()}
    state = binding.new_state(B, NH, d, d, variant, "cuda")
    h, state = _step_all(dev, variant, state, 0, T)
    views = binding.state_views(state, B, NH, d, d, variant)
    tol = TOL[dt]
    for hh in range(NH):
        x = {k: np64(v[0, hh]) for k, v in cpu.items()}
        C, n, m = np.zeros((d, d)), np.zeros(d), -np.inf
        ref = []
        for t in range(T):
            ht, C, n, m = oracle.recurrent_step(C, n, m, x["q"][t], x["k"][t], x["v"][t],
                                                x["igate"][t], x["fgate"][t], variant)
            ref.append(ht)
        assert relerr(np64(h[0, hh]), np.array(ref)) <= tol, f"h head {hh}"
        assert relerr(np64(views["C"][0, hh]), C) <= tol, f"C head {hh}"
        if variant == EXP:
            assert relerr(np64(views["n"][0, hh]), n) <= tol, f"n head {hh}"
            assert abs(float(views["m"][0, hh]) - m) <= 1e-4 * max(1.0, abs(m)), f"m head {hh}"


# name, dtype, d, chunk, T prefill, T continued
PREFILL = [
    ("fp32_chunk64", F32, 64, 64, 150, 12),
    ("bf16_chunk128", BF, 128, 128, 300, 12),
    ("bf16_chunk256_ragged", BF, 128, 256, 700, 12),
]


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_prefill_then_steps(variant, case):
    name, dt, d, L, T, Tn = case
    B, NH = 1, 2
    cpu = inputs(B, NH, T + Tn, d, d, seed=62, dtype=dt, ig_mean=-2.0)
    dev = {k: v.cuda() for k, v in cpu.items()}
    pre = {k: v[:, :, :T].contiguous() for k, v in dev.items()}
    h_pre, saved = binding.forward(pre["q"], pre["k"], pre["v"], pre["igate"], pre["fgate"], L, variant)
    state = binding.final_state(pre["k"], pre["v"], saved, L, variant)
    binding.check_device()
    views = binding.state_views(state, B, NH, d, d, variant)
    views = {k: (v.clone() if v is not None else None) for k, v in views.items()}
    h_new, _ = _step_all(dev, variant, state, T, T + Tn)
    tol = TOL[dt]
    for hh in range(NH):
        x = {k: np64(v[0, hh]) for k, v in cpu.items()}
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
        cw = oracle.chunkwise_forward(x["q"][:T], x["k"][:T], x["v"][:T], li[:T], lf[:T], variant, L)
        assert relerr(np64(views["C"][0, hh]), cw["C_final"]) <= tol, f"C head {hh}"
        if variant == EXP:
            assert relerr(np64(views["n"][0, hh]), cw["n_final"]) <= tol, f"n head {hh}"
            assert abs(float(views["m"][0, hh]) - cw["m_final"]) <= 1e-4 * max(1.0, abs(cw["m_final"]))
        full = (oracle.recurrent_forward(x["q"], x["k"], x["v"], li, lf, SIG)["h"] if variant == SIG
                else oracle.recurrent_forward_stabilised(x["q"], x["k"], x["v"], li, lf)["h"])
        assert relerr(np64(h_new[0, hh]), full[T:]) <= tol, f"continued h head {hh}"
        assert relerr(np64(h_pre[0, hh]), full[:T]) <= tol, f"prefill h head {hh}"
