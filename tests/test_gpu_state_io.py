"""Chunkwise calls that start from a state, and chained calls, on the GPU (C ABI).

Expected values come from the fp64 oracle run over the state written as prefix
tokens (tests/_state_prefix.py, pinned in test_state_prefix.py):
* mlstm_fwd_state: h and the final state, from a random initial state;
* two chained calls (the second starts from the first one's final state)
  against the oracle over the whole sequence from the zero state;
* mlstm_bwd_state: dq, dk, dv, both gate gradients and the initial state's
  gradient, with the initial state held constant.
Final states are compared as unstabilised states exp(m) (C, n).  Same
tolerances as the chunkwise parity tests (max|err| / max|ref|).
"""

import numpy as np
import pytest
import torch

import oracle
from mlstm_chunkwise_attention_b200 import binding
from _parity import TOL, inputs, np64, relerr
from _state_prefix import extend, prefix, random_state, state_grads, true_state

pytestmark = pytest.mark.gpu

SIG, EXP = binding.SIG, binding.EXP
BF, F32 = torch.bfloat16, torch.float32

# name, dtype, d, chunk, T  (chunk 64: CUDA cores; 128: chunk-128 kernel; 256+: large-chunk kernel)
CASES = [
    ("fp32_chunk64", F32, 64, 64, 150),
    ("bf16_chunk128", BF, 128, 128, 300),
    ("bf16_chunk256_ragged", BF, 128, 256, 700),
    ("bf16_d64_chunk512", BF, 64, 512, 600),
    # few heads, many chunks: the state walks run in segments (4 of 4 chunks; 2 of 6 and 5),
    # completed from the initial state, the final state's gradient and into dstate_in
    ("bf16_chunk64_split4", BF, 64, 64, 1000),
    ("bf16_chunk256_split2_ragged", BF, 128, 256, 2600),
]


def _device_state(states, B, NH, d_qk, d_hv, variant):
    """A state buffer holding the per-head (C, n, m) of ``states`` (row-major over B, NH)."""
    buf = binding.new_state(B, NH, d_qk, d_hv, variant, "cuda")
    views = binding.state_views(buf, B, NH, d_qk, d_hv, variant)
    for idx, (C, n, m) in enumerate(states):
        bb, hh = divmod(idx, NH)
        views["C"][bb, hh].copy_(torch.from_numpy(C).float())
        if variant == EXP:
            views["n"][bb, hh].copy_(torch.from_numpy(n).float())
            views["m"][bb, hh] = float(m)
    torch.cuda.synchronize()
    return buf


def _true(views, bb, hh, variant):
    n = np64(views["n"][bb, hh]) if variant == EXP else None
    m = float(views["m"][bb, hh]) if variant == EXP else 0.0
    return true_state(np64(views["C"][bb, hh]), n, m, variant)


def _head(cpu, hh, variant):
    """One head's inputs in fp64, with the log gates."""
    x = {k: np64(v[0, hh]) for k, v in cpu.items()}
    li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
    return x["q"], x["k"], x["v"], li, lf, x["igate"], x["fgate"], x["dh"]


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_forward_backward_from_a_state(variant, case):
    name, dt, d, L, T = case
    B, NH = 1, 2
    cpu = inputs(B, NH, T, d, d, seed=71, dtype=dt, ig_mean=-2.0)
    dev = {k: v.cuda() for k, v in cpu.items()}
    rng = np.random.default_rng(72)
    states = [random_state(rng, d, d, variant) for _ in range(B * NH)]
    s_in = _device_state(states, B, NH, d, d, variant)
    h, saved, s_out = binding.forward_state(dev["q"], dev["k"], dev["v"], dev["igate"],
                                            dev["fgate"], L, variant, s_in)
    g = binding.backward_state(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], h,
                               dev["dh"], saved, L, variant, s_in)
    binding.check_device()
    out_views = binding.state_views(s_out, B, NH, d, d, variant)
    d_views = binding.state_views(g["dstate_in"], B, NH, d, d, variant)
    tol = TOL[dt]
    for hh in range(NH):
        C0, n0, m0 = states[hh]
        q, k, v, li, lf, ig, fg, dh = _head(cpu, hh, variant)
        pre = prefix(C0, n0, m0, variant)
        ext = extend(pre, q, k, v, li, lf)
        fwd = oracle.chunkwise_forward(*ext, variant, L)
        assert relerr(np64(h[0, hh]), fwd["h"][d:]) <= tol, f"h head {hh}"
        ref_C, ref_n = true_state(fwd["C_final"], fwd["n_final"], fwd["m_final"], variant)
        got_C, got_n = _true(out_views, 0, hh, variant)
        assert relerr(got_C, ref_C) <= tol, f"final C head {hh}"
        if variant == EXP:
            assert relerr(got_n, ref_n) <= tol, f"final n head {hh}"
        bw = oracle.parallel_backward(*ext, variant, np.concatenate([np.zeros((d, d)), dh]))
        di, df = oracle.preact_grads(bw["dlog_i"][d:], bw["dlog_f"][d:], ig, fg, variant)
        ref = {"dq": bw["dq"][d:], "dk": bw["dk"][d:], "dv": bw["dv"][d:], "digate_pre": di,
               "dfgate_pre": df}
        for key, r in ref.items():
            err = relerr(np64(g[key][0, hh]), r)
            assert err <= tol, f"{key} head {hh}: {err:.3e}"
        dC, dn = state_grads(pre, bw["dk"][:d], bw["dv"][:d], m0, variant)
        assert relerr(np64(d_views["C"][0, hh]), dC) <= tol, f"dstate C head {hh}"
        if variant == EXP:
            assert relerr(np64(d_views["n"][0, hh]), dn) <= tol, f"dstate n head {hh}"


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_chained_calls_equal_one_call(variant, case):
    name, dt, d, L, T = case
    B, NH = 1, 2
    T1 = T // 3 + 5  # the first call ends inside a chunk
    cpu = inputs(B, NH, T, d, d, seed=73, dtype=dt, ig_mean=-2.0, with_dh=False)
    dev = {k: v.cuda() for k, v in cpu.items()}
    part = lambda a, b: {k: x[:, :, a:b].contiguous() for k, x in dev.items()}
    x1, x2 = part(0, T1), part(T1, T)
    h1, _, s1 = binding.forward_state(x1["q"], x1["k"], x1["v"], x1["igate"], x1["fgate"], L,
                                      variant, None, keep_saved=False)
    h2, _, s2 = binding.forward_state(x2["q"], x2["k"], x2["v"], x2["igate"], x2["fgate"], L,
                                      variant, s1, keep_saved=False)
    binding.check_device()
    views = binding.state_views(s2, B, NH, d, d, variant)
    tol = TOL[dt]
    for hh in range(NH):
        x = {k: np64(v[0, hh]) for k, v in cpu.items()}
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
        fwd = oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, variant, L)
        assert relerr(np64(h1[0, hh]), fwd["h"][:T1]) <= tol, f"first call h head {hh}"
        assert relerr(np64(h2[0, hh]), fwd["h"][T1:]) <= tol, f"second call h head {hh}"
        ref_C, ref_n = true_state(fwd["C_final"], fwd["n_final"], fwd["m_final"], variant)
        got_C, got_n = _true(views, 0, hh, variant)
        assert relerr(got_C, ref_C) <= tol, f"final C head {hh}"
        if variant == EXP:
            assert relerr(got_n, ref_n) <= tol, f"final n head {hh}"


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gradient_through_the_final_state(variant, case):
    """Backward of a loss on the final state alone (dh = 0): the gradients of
    <dC~_T, C~_T> + <dn~_T, n~_T> with m_T held constant, i.e. of <W, C_T> + <w, n_T> for
    the unstabilised state with W = exp(-m_T) dC~_T, against their closed form
    (tests/_state_prefix.py, pinned by finite differences in test_state_prefix.py)."""
    from _state_prefix import final_state_term_grads
    name, dt, d, L, T = case
    B, NH = 1, 2
    cpu = inputs(B, NH, T, d, d, seed=74, dtype=dt, ig_mean=-2.0)
    dev = {k: v.cuda() for k, v in cpu.items()}
    rng = np.random.default_rng(75)
    douts = [random_state(rng, d, d, variant, scale=1.0) for _ in range(B * NH)]
    d_out = _device_state(douts, B, NH, d, d, variant)
    h, saved, _ = binding.forward_state(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"],
                                        L, variant)
    zero_dh = torch.zeros_like(dev["dh"])
    g = binding.backward_state(dev["q"], dev["k"], dev["v"], dev["igate"], dev["fgate"], h, zero_dh,
                               saved, L, variant, dstate_out=d_out)
    binding.check_device()
    tol = TOL[dt]
    assert float(g["dq"].abs().max()) == 0.0
    for hh in range(NH):
        q, k, v, li, lf, ig, fg, _ = _head(cpu, hh, variant)
        m_T = oracle.chunkwise_forward(q, k, v, li, lf, variant, L)["m_final"]
        dC, dn, _ = douts[hh]
        s = float(np.exp(-m_T)) if variant == EXP else 1.0
        ref = final_state_term_grads(q, k, v, li, lf, s * dC, s * dn if variant == EXP else None)
        di, df = oracle.preact_grads(ref["dlog_i"], ref["dlog_f"], ig, fg, variant)
        want = {"dk": ref["dk"], "dv": ref["dv"], "digate_pre": di, "dfgate_pre": df}
        for key, r in want.items():
            err = relerr(np64(g[key][0, hh]), r)
            assert err <= tol, f"{key} head {hh}: {err:.3e}"
