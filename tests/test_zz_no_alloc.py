"""The allocation-free forward entry point, through the C ABI.

Callers that cannot allocate device memory when they run the op (a framework that
owns every device allocation, a plugin behind a custom allocator, a launch path where
an allocation would synchronise) use mlstm_fwd_noalloc, whose scratch is a fixed
array inside the library.  It runs the same kernels as mlstm_fwd on the same inputs,
so its output must be bit-identical to mlstm_fwd's; it is also checked against the
oracle.  This file is collected last so that a failure here leaves every other test
run.
"""

import pytest
import torch

from mlstm_chunkwise_attention_b200 import binding
from _parity import head64, inputs, np64, oracle_fwd_head, relerr

pytestmark = pytest.mark.gpu

# name, B, NH, T, d_qk, d_hv, chunk, variant, dtype, tolerance against the oracle
CASES = [
    ("exp_bf16_tensor_core_path", 1, 2, 700, 128, 128, 256, binding.EXP, torch.bfloat16, 1e-2),
    ("sig_fp32_cuda_core_path", 1, 2, 256, 64, 64, 64, binding.SIG, torch.float32, 1e-4),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_forward_matches_mlstm_fwd_on_two_calls(case):
    assert torch.cuda.is_available(), "needs a CUDA device"
    name, B, NH, T, dqk, dhv, L, var, dt, tol = case
    cpu = inputs(B, NH, T, dqk, dhv, seed=123, ig_mean=-1.0, fg_mean=3.0, dtype=dt,
                 with_dh=False)
    x = {k: v.cuda() for k, v in cpu.items()}
    h_ref, _ = binding.forward(x["q"], x["k"], x["v"], x["igate"], x["fgate"], L, var,
                               keep_saved=False)
    binding.check_device()
    sizes = binding.problem_sizes(x["q"], x["v"], L, var)
    stream = torch.cuda.current_stream().cuda_stream
    ptrs = [x[n].data_ptr() for n in ("q", "k", "v", "igate", "fgate")]
    outs = [torch.full_like(x["v"], float("nan")) for _ in range(2)]
    torch.cuda.synchronize()
    free_before = None
    for i, h in enumerate(outs):
        if i == 1:
            free_before = torch.cuda.mem_get_info()[0]
        st = binding.mlstm_fwd_noalloc(*ptrs, h.data_ptr(), *sizes, stream)
        assert st == 0, binding.mlstm_status_string(st)
        binding.check_device()
        # the first call on the device may load code and place the array; the
        # second allocates nothing
        if i == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
        assert torch.equal(h, h_ref), f"call {i}"
    for b in range(B):
        for hh in range(NH):
            ref = oracle_fwd_head(head64(cpu, b, hh), L, var)
            assert relerr(np64(outs[1][b, hh]), ref["h"]) <= tol


def test_noalloc_rejects_problems_beyond_its_scratch():
    assert torch.cuda.is_available(), "needs a CUDA device"
    # B8 H32 T4096 d128 needs hundreds of MB of scratch, far beyond 32 MiB
    st = binding.mlstm_fwd_noalloc(16, 16, 16, 16, 16, 16, 8, 32, 4096, 128, 128, 128,
                                   binding.EXP, binding.BF16, None)
    assert st == 3
