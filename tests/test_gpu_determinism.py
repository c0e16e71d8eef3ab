"""Run-to-run determinism of the CUDA path, through the C ABI.

The same inputs through the same entry points must give the same bits every time:
every kernel writes each output element from one thread, in a fixed order of
operations, and waits for every hand-over it depends on.  A missing wait or a race
between warps shows up here as results that differ between repeated calls, often
in one 32-row block (one TMEM lane quarter) of one chunk.  The shapes hold enough
heads and chunks that the kernels run several waves of CTAs; each is repeated, and
the forward output, every saved region and every gradient are compared with the
first call.  The gate gradients of problems whose dq or dk kernel accumulates the
per-token dot products of several column slices with float atomics (d_qk > 128) may
differ in the last bits between calls; they are compared to 1e-6 there.
"""

import pytest
import torch

from mlstm_chunkwise_attention_b200 import binding
from _parity import inputs

pytestmark = pytest.mark.gpu

SIG, EXP = binding.SIG, binding.EXP
BF = torch.bfloat16

# name, B, NH, T, d_qk, d_hv, chunk, variant, igate mean, repeats
CASES = [
    ("walkers_exp_chunk128_d128", 2, 96, 1024, 128, 128, 128, EXP, -2.0, 6),
    ("walkers_sig_chunk128_d128", 2, 96, 1024, 128, 128, 128, SIG, 0.0, 4),
    ("xl_exp_chunk1024_d128", 2, 16, 2048, 128, 128, 1024, EXP, 0.0, 4),
    ("xl_sig_chunk256_d128", 2, 32, 1024, 128, 128, 256, SIG, 0.0, 4),
    ("tc_exp_chunk128_dqk256_dhv512", 1, 16, 1024, 256, 512, 128, EXP, 0.0, 3),
    ("exp_chunk64_d128", 2, 32, 1024, 128, 128, 64, EXP, -2.0, 3),
]


def _run(dev, L, var):
    h, saved = binding.forward(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], L, var)
    g = binding.backward(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], h, dev["dh"],
                         saved, L, var)
    binding.check_device()
    out = {"h": h}
    sv = binding.saved_views(saved, dev["q"], dev["v"], L, var)
    out.update({"saved_" + k: v for k, v in sv.items() if v is not None})
    out.update(g)
    return out


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_repeated_calls_give_identical_bits(case):
    name, B, NH, T, dqk, dhv, L, var, igm, reps = case
    cpu = inputs(B, NH, T, dqk, dhv, seed=len(name) * 131 + T, dtype=BF, ig_mean=igm)
    dev = {k: v.cuda() for k, v in cpu.items()}
    first = _run(dev, L, var)
    atomics = dqk > 128
    for rep in range(1, reps):
        o = _run(dev, L, var)
        for key, ref in first.items():
            if atomics and key in ("digate_pre", "dfgate_pre"):
                d = (o[key].float() - ref.float()).abs().max().item()
                assert d <= 1e-6 * ref.float().abs().max().item(), f"{key} call {rep}"
            else:
                assert torch.equal(o[key], ref), f"{key} differs on call {rep}"
