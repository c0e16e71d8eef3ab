"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the fp64 oracle on the same (I/O-dtype-rounded) inputs, compare."""

import numpy as np
import torch

import oracle
from mlstm_chunkwise_attention_b200 import binding
from mlstm_chunkwise_attention_b200.synthetic import make_inputs

# max|err| / max|ref| bounds for bf16 and fp32 I/O
TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def relerr(got, ref, floor=1e-30):
    """max|got - ref| / max(max|ref|, floor)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the CUDA result"
    return float(np.max(np.abs(got - ref)) / max(float(np.max(np.abs(ref))), floor))


def np64(t):
    return t.detach().double().cpu().numpy()


def inputs(B, NH, T, d_qk, d_hv, seed, dtype, ig_mean=0.0, fg_mean=3.0, with_dh=True, **kw):
    return make_inputs(B, NH, T, d_qk, d_hv, seed=seed, igate_mean=ig_mean, fgate_mean=fg_mean,
                       dtype=dtype, with_dh=with_dh, **kw)


def gpu_fwd(cpu, chunk, variant):
    dev = {k: v.cuda() for k, v in cpu.items()}
    h, saved = binding.forward(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], chunk, variant)
    binding.check_device()  # synchronises; raises if a kernel reported a timeout
    return dev, h, saved


def gpu_bwd(dev, h, saved, chunk, variant):
    g = binding.backward(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], h, dev["dh"],
                         saved, chunk, variant)
    binding.check_device()
    return g


def head64(cpu, b, hh):
    return {k: np64(v[b, hh]) for k, v in cpu.items()}


def oracle_fwd_head(x, chunk, variant):
    li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
    return oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, variant, chunk)


def io_round(a, dtype):
    """a rounded to the I/O dtype, as a tensor of that dtype would hold it."""
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(dtype).double().numpy()


def oracle_bwd_head(x, variant, dtype=None):
    """Parallel-form backward of one head.  With dtype (the I/O dtype), the backward's h
    input is the oracle's own forward output rounded to it, as the boundary passes h."""
    li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
    h_in = None
    if dtype is not None:
        h_in = io_round(oracle.parallel_forward(x["q"], x["k"], x["v"], li, lf, variant)["h"], dtype)
    g = oracle.parallel_backward(x["q"], x["k"], x["v"], li, lf, variant, x["dh"], h_in=h_in)
    di, df = oracle.preact_grads(g["dlog_i"], g["dlog_f"], x["igate"], x["fgate"], variant)
    return {"dq": g["dq"], "dk": g["dk"], "dv": g["dv"], "digate_pre": di, "dfgate_pre": df}
