"""The allocation-free forward entry point, through the C ABI.

Callers that cannot allocate device memory when they run the op use
mlstm_fwd_noalloc, whose scratch is a fixed array inside the library.  This
file is collected last so that a failure here leaves every other test run.
"""

import numpy as np
import pytest
import torch

from mlstm_chunkwise_attention_b200 import binding
from mlstm_chunkwise_attention_b200.synthetic import make_inputs

pytestmark = pytest.mark.gpu

# name, B, NH, T, d_qk, d_hv, chunk, variant, dtype, tolerance used by the parity tests
CASES = [
    ("exp_bf16_tensor_core_path", 1, 2, 700, 128, 128, 256, binding.EXP, torch.bfloat16, 1e-2),
    ("sig_fp32_cuda_core_path", 1, 2, 256, 64, 64, 64, binding.SIG, torch.float32, 1e-4),
]


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(float(np.max(np.abs(b))), 1e-30))


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_forward_matches_mlstm_fwd_on_two_calls(case):
    assert torch.cuda.is_available(), "needs a CUDA device"
    name, B, NH, T, dqk, dhv, L, var, dt, tol = case
    cpu = make_inputs(B, NH, T, dqk, dhv, seed=123, igate_mean=-1.0, fgate_mean=3.0, dtype=dt)
    x = {k: v.cuda() for k, v in cpu.items()}
    h_ref, _ = binding.forward(x["q"], x["k"], x["v"], x["igate"], x["fgate"], L, var,
                               keep_saved=False)
    binding.check_device()
    sizes = binding.problem_sizes(x["q"], x["v"], L, var)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        h = torch.full_like(x["v"], float("nan"))
        st = binding.mlstm_fwd_noalloc(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                                       x["igate"].data_ptr(), x["fgate"].data_ptr(), h.data_ptr(),
                                       *sizes, stream)
        assert st == 0, binding.mlstm_status_string(st)
        binding.check_device()
        assert _rel(h, h_ref) <= tol


def test_noalloc_rejects_problems_beyond_its_scratch():
    assert torch.cuda.is_available(), "needs a CUDA device"
    # B8 H32 T4096 d128 needs hundreds of MB of scratch, far beyond 32 MiB
    st = binding.mlstm_fwd_noalloc(16, 16, 16, 16, 16, 16, 8, 32, 4096, 128, 128, 128,
                                   binding.EXP, binding.BF16, None)
    assert st == 3
