"""Sequence segments on the GPU (C ABI) against the fp64 oracle.

* mlstm_log_decay against the sum of log sigmoid over the segment;
* mlstm_state_chain: the state after a then b, chained from a's state and b's
  state from zero, against the oracle's chunkwise final state over a + b
  (compared as unstabilised states);
* the sequence-parallel protocol of seqpar.py with its segments run one after
  the other in this process (no cross-process exchange: the gathered lists are
  the local ones): the outputs of every segment, and the gradients of every
  segment's tokens, against the oracle over the whole sequence.
"""

import numpy as np
import pytest
import torch

import oracle
from mlstm_chunkwise_attention_b200 import binding, seqpar
from _parity import TOL, inputs, np64, relerr
from _state_prefix import true_state

pytestmark = pytest.mark.gpu

SIG, EXP = binding.SIG, binding.EXP
BF, F32 = torch.bfloat16, torch.float32

# name, dtype, d, chunk, T, segments
CASES = [
    ("fp32_chunk64_3seg", F32, 64, 64, 300, 3),
    ("bf16_chunk128_4seg", BF, 128, 128, 1024, 4),
    ("bf16_chunk256_2seg_ragged", BF, 128, 256, 1100, 2),
]


def _true(state, B, NH, d_qk, d_hv, variant, bb, hh):
    v = binding.state_views(state, B, NH, d_qk, d_hv, variant)
    n = np64(v["n"][bb, hh]) if variant == EXP else None
    m = float(v["m"][bb, hh]) if variant == EXP else 0.0
    return true_state(np64(v["C"][bb, hh]), n, m, variant)


@pytest.mark.parametrize("dt", [F32, BF], ids=["fp32", "bf16"])
def test_log_decay(dt):
    cpu = inputs(2, 3, 777, 64, 64, seed=81, dtype=dt, with_dh=False)
    G = binding.log_decay(cpu["fgate"].cuda())
    binding.check_device()
    ref = oracle.logsigmoid(np64(cpu["fgate"])).sum(axis=-1)
    assert relerr(np64(G), ref) <= 1e-5


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
def test_state_chain(variant):
    B, NH, d, L, Ta, Tb = 1, 2, 64, 64, 130, 200
    cpu = inputs(B, NH, Ta + Tb, d, d, seed=82, dtype=F32, ig_mean=-2.0, with_dh=False)
    dev = {k: v.cuda() for k, v in cpu.items()}
    a = {k: x[:, :, :Ta].contiguous() for k, x in dev.items()}
    b = {k: x[:, :, Ta:].contiguous() for k, x in dev.items()}
    _, _, Sa = binding.forward_state(a["q"], a["k"], a["v"], a["igate"], a["fgate"], L, variant,
                                     None, keep_saved=False, want_h=False)
    _, _, Sb = binding.forward_state(b["q"], b["k"], b["v"], b["igate"], b["fgate"], L, variant,
                                     None, keep_saved=False, want_h=False)
    out = binding.state_chain(Sa, Sb, binding.log_decay(b["fgate"]), B, NH, d, d, variant)
    binding.check_device()
    for hh in range(NH):
        x = {k: np64(v[0, hh]) for k, v in cpu.items()}
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
        fwd = oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, variant, L)
        ref_C, ref_n = true_state(fwd["C_final"], fwd["n_final"], fwd["m_final"], variant)
        got_C, got_n = _true(out, B, NH, d, d, variant, 0, hh)
        assert relerr(got_C, ref_C) <= TOL[F32], f"C head {hh}"
        if variant == EXP:
            assert relerr(got_n, ref_n) <= TOL[F32], f"n head {hh}"


def _run_segments(cpu, L, variant, P, with_backward):
    """The protocol of seqpar.py with its P segments run one after the other here."""
    dev = {k: v.cuda() for k, v in cpu.items()}
    T = dev["q"].shape[2]
    bounds = [round(T * r / P) for r in range(P + 1)]
    segs = [{k: x[:, :, bounds[r]:bounds[r + 1]].contiguous() for k, x in dev.items()}
            for r in range(P)]
    ops = seqpar.DeviceOps()
    B, NH, _, d = dev["q"].shape
    sizes = (B, NH, d, dev["v"].shape[-1])
    local = [ops.local_state(s, L, variant) for s in segs]
    decays = [g for _, g in local]
    chained = seqpar.chain_states([s for s, _ in local], decays, sizes, variant, ops)
    parts = []
    for r in range(P):
        h, saved = ops.forward_from(segs[r], L, variant, chained[r], keep_saved=with_backward)
        parts.append(seqpar.Segment(h=h, state_in=chained[r], states=chained, decays=decays,
                                    saved=saved, index=r))
    grads = None
    if with_backward:
        dls = [ops.local_dstate(segs[r], segs[r]["dh"], parts[r], L, variant) for r in range(P)]
        grads = []
        for r in range(P):
            dout = seqpar.final_state_gradient(r, dls, chained, decays, sizes, variant, ops)
            grads.append(ops.backward_from(segs[r], segs[r]["dh"], parts[r], L, variant, dout))
    binding.check_device()
    return bounds, parts, grads


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_segments_in_sequence_equal_one_call(variant, case):
    name, dt, d, L, T, P = case
    B, NH = 1, 2
    cpu = inputs(B, NH, T, d, d, seed=83, dtype=dt, ig_mean=-2.0, with_dh=False)
    bounds, parts, _ = _run_segments(cpu, L, variant, P, with_backward=False)
    h_all = torch.cat([p.h for p in parts], dim=2)
    for hh in range(NH):
        x = {k: np64(v[0, hh]) for k, v in cpu.items()}
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], variant)
        ref = oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, variant, L)["h"]
        for r in range(P):
            sl = slice(bounds[r], bounds[r + 1])
            assert relerr(np64(h_all[0, hh, sl]), ref[sl]) <= TOL[dt], f"segment {r} head {hh}"


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_segment_backward_equals_one_call(variant, case):
    """The sequence-parallel backward (each segment's own initial-state share, carried
    back to the earlier segments as their final-state gradients) against the oracle's
    backward over the whole sequence."""
    name, dt, d, L, T, P = case
    B, NH = 1, 2
    cpu = inputs(B, NH, T, d, d, seed=84, dtype=dt, ig_mean=-2.0)
    bounds, _, grads = _run_segments(cpu, L, variant, P, with_backward=True)
    got = {k: torch.cat([g[k] for g in grads], dim=2) for k in grads[0]}
    ref = oracle.backward_heads(np64(cpu["q"]), np64(cpu["k"]), np64(cpu["v"]), np64(cpu["igate"]),
                                np64(cpu["fgate"]), variant, np64(cpu["dh"]))
    names = {"dq": "dq", "dk": "dk", "dv": "dv", "digate_pre": "digate", "dfgate_pre": "dfgate"}
    for key, rk in names.items():
        for hh in range(NH):
            err = relerr(np64(got[key][0, hh]), ref[rk][0, hh])
            assert err <= TOL[dt], f"{key} head {hh}: {err:.3e}"
