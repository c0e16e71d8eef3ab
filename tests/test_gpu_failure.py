"""The failure report of the tensor-core kernels, on the GPU, without a fault.

Every wait in a tensor-core kernel is bounded; a CTA whose wait runs out raises its
launch's failure flag and winds down.  mlstm_selftest_timeout enqueues one kernel
whose wait (on a barrier nothing completes) runs out after 2 s, in the flag family of
the chunk-128 output kernel.  The failure must be reported once by
mlstm_device_status, and must not silence the launches that follow it, whether or not
the status is read in between.
"""

import pytest
import torch

from mlstm_chunkwise_attention_b200 import binding
from _parity import gpu_fwd, head64, inputs, np64, oracle_fwd_head, relerr

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # MLSTM_ERR_TIMEOUT


def test_timeout_reported_once_and_later_launches_run():
    assert torch.cuda.is_available(), "needs a CUDA device"
    # chunk 128 at d 64 runs the state kernel and the chunk-128 output kernel, whose
    # flag family the self-test uses
    assert binding.load().mlstm_launch_name(0, 2, 1, 2, 300, 64, 64, 128, binding.EXP,
                                            binding.BF16) == b"output_fwd_tc"
    binding.check_device()  # nothing pending before the test
    stream = torch.cuda.current_stream().cuda_stream
    assert binding.mlstm_selftest_timeout(stream) == 0
    # a forward enqueued behind the failed launch, with no status read in between
    cpu = inputs(1, 2, 300, 64, 64, seed=515, dtype=torch.bfloat16, ig_mean=-1.0,
                 with_dh=False)
    dev = {k: v.cuda() for k, v in cpu.items()}
    h, _ = binding.forward(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], 128,
                           binding.EXP, keep_saved=False)
    assert binding.mlstm_device_status(stream) == TIMEOUT
    assert binding.mlstm_device_status(stream) == 0  # reported once
    for hh in range(2):
        ref = oracle_fwd_head(head64(cpu, 0, hh), 128, binding.EXP)
        assert relerr(np64(h[0, hh]), ref["h"]) <= 1e-2
    # and a call after the report runs too
    _, h2, _ = gpu_fwd(cpu, 128, binding.EXP)
    assert torch.equal(h, h2)
