"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerance: max|err| / max|ref| <= 1e-2 for bf16 I/O and <= 1e-4 for fp32 I/O,
per output tensor, on the same seeded inputs (the oracle reads the
dtype-rounded values).  Small cases compare every element of every head;
full-size workloads compare whole sampled heads (heads are independent) or
sampled rows, plus properties that hold at any size.
"""

import zlib

import numpy as np
import pytest
import torch

import oracle
from mlstm_chunkwise_attention_b200 import binding
from mlstm_chunkwise_attention_b200.synthetic import WORKLOADS, sample_heads, sample_rows
from _parity import (TOL, gpu_bwd, gpu_fwd, head64, inputs, io_round, np64, oracle_bwd_head,
                     oracle_fwd_head, relerr)

pytestmark = pytest.mark.gpu

SIG, EXP = binding.SIG, binding.EXP
F32, BF = torch.float32, torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    binding.load()  # fails loudly if the library is not built


# name, B, NH, T, d_qk, d_hv, chunk, variant, dtype, ig_mean, fg_mean
SMALL = [
    ("sig_fp32_b1h2_t256_d64", 1, 2, 256, 64, 64, 64, SIG, F32, 0.0, 3.0),
    ("exp_fp32_ragged_t200", 1, 2, 200, 64, 128, 64, EXP, F32, -2.0, 3.0),
    ("exp_bf16_multitile_ragged", 2, 2, 700, 128, 128, 256, EXP, BF, -2.0, 3.0),
    ("sig_bf16_multitile_ragged", 2, 2, 700, 128, 128, 256, SIG, BF, 0.0, 3.0),
    ("exp_bf16_dqk256_dhv512", 1, 2, 300, 256, 512, 128, EXP, BF, 0.0, 3.0),
    ("sig_bf16_dqk256_dhv512", 1, 1, 300, 256, 512, 128, SIG, BF, -10.0, 4.0),
    ("sig_bf16_igate_bias_m10", 1, 2, 512, 64, 64, 64, SIG, BF, -10.0, 4.0),
    ("exp_bf16_igate_bias_m10", 1, 2, 512, 64, 64, 64, EXP, BF, -10.0, 3.0),
    ("exp_bf16_one_partial_chunk", 1, 1, 37, 64, 64, 64, EXP, BF, 0.0, 3.0),
    ("exp_fp32_t1", 1, 1, 1, 64, 64, 64, EXP, F32, -4.0, 3.0),
    ("sig_bf16_chunk4096_ragged", 1, 1, 4500, 64, 64, 4096, SIG, BF, 0.0, 3.0),
    ("exp_bf16_chunk1024", 1, 1, 2048, 128, 128, 1024, EXP, BF, 0.0, 3.0),
    ("exp_bf16_dqk256_dhv64_chunk512_ragged", 1, 2, 1000, 256, 64, 512, EXP, BF, 0.0, 3.0),
    ("sig_bf16_dqk64_dhv128_chunk256_ragged", 1, 2, 600, 64, 128, 256, SIG, BF, -2.0, 3.0),
    ("exp_fp32_dqk256", 1, 1, 384, 256, 64, 128, EXP, F32, 1.0, 2.0),
    ("exp_bf16_chunk128_d128_ragged", 2, 2, 700, 128, 128, 128, EXP, BF, -2.0, 3.0),
    ("sig_bf16_chunk128_d128_ragged", 1, 3, 1000, 128, 128, 128, SIG, BF, 0.0, 3.0),
    ("exp_bf16_chunk128_d128_one_partial", 1, 2, 77, 128, 128, 128, EXP, BF, 0.0, 3.0),
    ("exp_bf16_chunk128_d128_t1", 1, 2, 1, 128, 128, 128, EXP, BF, -1.0, 3.0),
    ("sig_bf16_chunk128_d128_t128_one_full", 1, 2, 128, 128, 128, 128, SIG, BF, 0.0, 3.0),
    ("exp_bf16_chunk128_d128_t129_one_token_tail", 2, 1, 129, 128, 128, 128, EXP, BF, -2.0, 3.0),
    # chunk 64 on the tensor cores: a 64-token chunk in a half-filled 128-row tile
    ("exp_bf16_chunk64_d128_ragged", 2, 2, 700, 128, 128, 64, EXP, BF, -2.0, 3.0),
    ("sig_bf16_chunk64_d128_ragged", 1, 3, 333, 128, 128, 64, SIG, BF, 0.0, 3.0),
    ("exp_bf16_chunk64_t1", 1, 2, 1, 128, 128, 64, EXP, BF, -1.0, 3.0),
    ("sig_bf16_chunk64_dqk256_dhv512", 1, 1, 200, 256, 512, 64, SIG, BF, 0.0, 3.0),
    ("exp_bf16_chunk64_dqk64_dhv128_t65", 1, 2, 65, 64, 128, 64, EXP, BF, 0.0, 3.0),
    # one head, 32 chunks: the state walks run as 8 segments of 4 chunks plus a completion
    ("exp_bf16_chunk64_d128_split8", 1, 1, 2048, 128, 128, 64, EXP, BF, -2.0, 3.0),
    ("sig_bf16_chunk128_d64_split4_ragged", 1, 2, 2000, 64, 64, 128, SIG, BF, 0.0, 3.0),
]


def _compare_all_heads(cpu, h, g, L, var, tol, grad_tol=None):
    """Every element of every head against the oracle; the bar applies per output tensor
    (max|err| over all heads / max|ref| over all heads), tol for h and grad_tol (default
    tol; a dict maps a gradient's name, else "default", to its bar) for the gradients.  The oracle backward reads h in the I/O dtype, as mlstm_bwd
    receives it."""
    Bn, NH = cpu["q"].shape[:2]
    worst = {}
    for b in range(Bn):
        for hh in range(NH):
            x = head64(cpu, b, hh)
            pairs = [("h", np64(h[b, hh]), oracle_fwd_head(x, L, var)["h"])]
            ref_g = oracle_bwd_head(x, var, cpu["q"].dtype)
            pairs += [(key, np64(g[key][b, hh]), val) for key, val in ref_g.items()]
            for key, got, ref in pairs:
                assert np.all(np.isfinite(got)), f"non-finite {key} ({b},{hh})"
                e, r = float(np.max(np.abs(got - ref))), float(np.max(np.abs(ref)))
                ce, cr, _ = worst.get(key, (0.0, 0.0, None))
                worst[key] = (max(ce, e), max(cr, r), (b, hh) if e > ce else worst.get(key, (0, 0, None))[2])
    # a gradient that is exactly zero in the mathematics (a closed forget gate, one token)
    # is compared on the scale of the other gradients
    gscale = max(worst[k][1] for k in worst if k != "h")
    for key, (e, r, at) in worst.items():
        floor = 1e-3 * gscale if key != "h" else 1e-30
        err = e / max(r, floor)
        bar = tol if key == "h" or grad_tol is None else grad_tol
        if isinstance(bar, dict):
            bar = bar.get(key, bar["default"])
        assert err <= bar, f"{key}: {err:.3e} (largest error in head {at})"


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_forward_backward_all_heads(case):
    name, Bn, NH, T, dqk, dhv, L, var, dt, igm, fgm = case
    cpu = inputs(Bn, NH, T, dqk, dhv, seed=zlib.crc32(name.encode()) % 10000, dtype=dt, ig_mean=igm, fg_mean=fgm)
    dev, h, saved = gpu_fwd(cpu, L, var)
    g = gpu_bwd(dev, h, saved, L, var)
    _compare_all_heads(cpu, h, g, L, var, TOL[dt])


# mLSTMexp with large positive input-gate preactivations, on every tensor-core path:
# exp(i~) far above 1 stresses the max state, the separable decay factors and the
# hi/lo state planes in fp32.  q and k are N(0.7, 1), so q.k > 0 mostly and the
# normaliser sum_s A_ts does not cancel: with random signs and a large i~ the
# normaliser's floor exp(-m_t) is negligible and |a_t| can fall orders of magnitude
# below sum_s |A_ts|, where h = num / a amplifies any bf16 rounding by that ratio (an
# input-conditioning limit of bf16 operands, not of the stabiliser).
# name, B, NH, T, d_qk, d_hv, chunk, igate mean, igate std, spike value (every 53rd
# token from token 11 on), forget mean
BIG_IGATE = [
    ("exp_walkers_chunk128_d128", 2, 2, 700, 128, 128, 128, 8.0, 2.0, None, 3.0),
    ("exp_walkers_chunk128_d128_spikes40", 1, 2, 640, 128, 128, 128, 0.0, 1.0, 40.0, 3.0),
    ("exp_chunk128_dqk256_dhv512", 1, 2, 300, 256, 512, 128, 8.0, 2.0, None, 3.0),
    ("exp_chunk128_dqk64_dhv64_spikes40", 1, 2, 400, 64, 64, 128, 0.0, 1.0, 40.0, 3.0),
    ("exp_xl_chunk256_ragged", 1, 2, 700, 128, 128, 256, 8.0, 2.0, None, 3.0),
    ("exp_xl_chunk256_spikes40", 1, 2, 600, 64, 128, 256, 0.0, 1.0, 40.0, 3.0),
    ("exp_xl_chunk1024", 1, 2, 2048, 128, 128, 1024, 8.0, 2.0, None, 3.0),
    ("exp_xl_chunk1024_spikes40", 1, 1, 1500, 128, 128, 1024, 0.0, 1.0, 40.0, 3.0),
    ("exp_chunk64_d128", 1, 2, 500, 128, 128, 64, 8.0, 2.0, None, 3.0),
    ("exp_chunk64_d64_spikes40", 1, 2, 333, 64, 64, 64, 0.0, 1.0, 40.0, 3.0),
]


@pytest.mark.parametrize("case", BIG_IGATE, ids=[c[0] for c in BIG_IGATE])
def test_exp_large_input_gates_all_heads(case):
    name, Bn, NH, T, dqk, dhv, L, igm, igs, spike, fgm = case
    cpu = inputs(Bn, NH, T, dqk, dhv, seed=zlib.crc32(name.encode()) % 10000, dtype=BF,
                 ig_mean=igm, fg_mean=fgm, igate_std=igs, qk_mean=0.7)
    if spike is not None:
        cpu["igate"][..., 11::53] = spike
    dev, h, saved = gpu_fwd(cpu, L, EXP)
    g = gpu_bwd(dev, h, saved, L, EXP)
    # With +40 spikes one token dominates each row, h_t is nearly v_s, and the gradient
    # term dA_ts = dh_t.(v_s - h_t) / den_t cancels down to the last bits of the bf16
    # output h: an fp64 emulation with only h rounded puts the gradients 1e-2 to 5e-2 off
    # the exact ones, and a forward that differs in the last bit of h moves them as much.
    # The gate gradients sum such terms over the sequence: moving a random half of the
    # bf16 h by one ulp moves the oracle's dfgate_pre by up to 0.23 and digate_pre by up
    # to 0.13 of their largest element in the chunk-128 d64 case.  h itself is held to
    # 1e-2; dq, dk, dv to a sanity bound of 1e-1, the gate gradients to 0.25.
    spike_tol = {"default": 1e-1, "digate_pre": 0.25, "dfgate_pre": 0.25}
    _compare_all_heads(cpu, h, g, L, EXP, 1e-2, grad_tol=spike_tol if spike is not None else None)


@pytest.mark.parametrize("var", [SIG, EXP])
def test_saved_gate_prep_and_states_match_oracle(var):
    """K-a (cumsums, max states) and K-b (states entering each chunk)."""
    Bn, NH, T, dqk, dhv, L = 1, 2, 320, 64, 128, 64
    cpu = inputs(Bn, NH, T, dqk, dhv, seed=77, dtype=F32, ig_mean=-1.0, fg_mean=2.0, with_dh=False)
    dev, h, saved = gpu_fwd(cpu, L, var)
    sv = binding.saved_views(saved, dev["q"], dev["v"], L, var)
    for hh in range(NH):
        x = head64(cpu, 0, hh)
        ref = oracle_fwd_head(x, L, var)
        assert relerr(np64(sv["b"][hh]), ref["b"]) < 1e-5
        assert relerr(np64(sv["log_i"][hh]), ref["log_i"]) < 1e-5
        assert relerr(np64(sv["C"][hh]), ref["C_enter"]) < 1e-5
        if var == EXP:
            np.testing.assert_allclose(np64(sv["m"][hh]), ref["m_row"], rtol=1e-5, atol=1e-4)
            assert relerr(np64(sv["abar"][hh]), ref["abar"]) < 1e-5
            assert relerr(np64(sv["n"][hh]), ref["n_enter"]) < 1e-5


def test_saturated_normaliser_has_zero_gradient():
    """T = 1 with |i q'.k| > 1: h = sign(a) v, so dq, dk and d igate are exactly 0."""
    cpu = inputs(1, 1, 1, 64, 64, seed=3, dtype=F32)
    q, k = cpu["q"][0, 0, 0], cpu["k"][0, 0, 0]
    s = float(q @ k) / 8.0
    cpu["igate"] = torch.full((1, 1, 1), float(np.log(4.0 / max(abs(s), 1e-3))), dtype=F32)
    dev, h, saved = gpu_fwd(cpu, 64, EXP)
    g = gpu_bwd(dev, h, saved, 64, EXP)
    want_h = np.sign(s) * np64(cpu["v"][0, 0])
    assert relerr(np64(h[0, 0]), want_h) <= 1e-4
    scale = float(np.abs(np64(cpu["dh"])).max() * np.abs(np64(cpu["v"])).max())
    for key in ("dq", "dk", "digate_pre"):
        assert np.abs(np64(g[key])).max() <= 1e-5 * scale, key
    assert relerr(np64(g["dv"][0, 0]), np.sign(s) * np64(cpu["dh"][0, 0])) <= 1e-4


def _preact(v, T):
    return torch.full((1, 1, T), float(v), dtype=F32)


def test_open_gates_sig_is_causal_linear_attention():
    T, d = 200, 64
    cpu = inputs(1, 1, T, d, d, seed=5, dtype=F32, with_dh=False)
    cpu["igate"] = _preact(200.0, T)
    cpu["fgate"] = _preact(200.0, T)
    _, h, _ = gpu_fwd(cpu, 64, SIG)
    q, k, v = (np64(cpu[n][0, 0]) for n in ("q", "k", "v"))
    want = np.tril(q @ k.T / np.sqrt(d)) @ v
    assert relerr(np64(h[0, 0]), want) <= 1e-4


@pytest.mark.parametrize("var", [SIG, EXP])
def test_closed_forget_gate_is_one_step_readout(var):
    T, d = 130, 64
    cpu = inputs(1, 1, T, d, d, seed=6, dtype=F32, with_dh=False)
    cpu["fgate"] = _preact(-200.0, T)
    _, h, _ = gpu_fwd(cpu, 64, var)
    q, k, v, ig = (np64(cpu[n][0, 0]) for n in ("q", "k", "v", "igate"))
    s = np.einsum("td,td->t", q, k) / np.sqrt(d)
    if var == SIG:
        want = (s / (1.0 + np.exp(-ig)))[:, None] * v
    else:
        want = (s / np.maximum(np.abs(s), np.exp(-ig)))[:, None] * v
    assert relerr(np64(h[0, 0]), want) <= 1e-4


def test_constant_decay_is_retention():
    T, d, gamma = 256, 64, 0.95
    cpu = inputs(1, 1, T, d, d, seed=7, dtype=F32, with_dh=False)
    cpu["igate"] = _preact(200.0, T)
    cpu["fgate"] = _preact(np.log(gamma / (1 - gamma)), T)
    _, h, _ = gpu_fwd(cpu, 64, SIG)
    q, k, v = (np64(cpu[n][0, 0]) for n in ("q", "k", "v"))
    gam = 1.0 / (1.0 + np.exp(-float(cpu["fgate"][0, 0, 0])))
    idx = np.arange(T)
    lag = idx[:, None] - idx[None, :]
    want = ((q @ k.T / np.sqrt(d)) * np.where(lag >= 0, gam ** np.clip(lag, 0, None), 0.0)) @ v
    assert relerr(np64(h[0, 0]), want) <= 1e-4


def test_chunk_size_invariance_on_gpu():
    """The same inputs through chunk 64, 128, 256 and 512 give the same h."""
    cpu = inputs(1, 2, 1024, 64, 64, seed=8, dtype=F32, with_dh=False)
    outs = [np64(gpu_fwd(cpu, L, EXP)[1]) for L in (64, 128, 256, 512)]
    for o in outs[1:]:
        assert relerr(o, outs[0]) <= 1e-4


def test_repeat_calls_are_deterministic_forward():
    cpu = inputs(1, 2, 300, 64, 64, seed=9, dtype=BF, with_dh=False)
    a = np64(gpu_fwd(cpu, 64, EXP)[1])
    b = np64(gpu_fwd(cpu, 64, EXP)[1])
    assert np.array_equal(a, b)


def test_host_errors_on_device_buffers():
    cpu = inputs(1, 1, 128, 64, 64, seed=10, dtype=BF, with_dh=False)
    dev = {k: v.cuda() for k, v in cpu.items()}
    sizes = binding.problem_sizes(dev["q"], dev["v"], 64, EXP)
    h = torch.empty_like(dev["v"])
    need = binding.mlstm_fwd_workspace_size(*sizes)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ptr = [dev[n].data_ptr() for n in ("q", "k", "v", "igate", "fgate")]
    st = binding.mlstm_fwd(*ptr, h.data_ptr(), None, ws.data_ptr(), need - 1, *sizes, None)
    assert st == 3
    st = binding.mlstm_fwd(ptr[0] + 2, *ptr[1:], h.data_ptr(), None, ws.data_ptr(), need, *sizes, None)
    assert st == 1
    st = binding.mlstm_fwd(*ptr, h.data_ptr(), None, ws.data_ptr(), need, *sizes, None)
    assert st == 0
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times
# ---------------------------------------------------------------------------

def _full(name, variant=None, heads_fwd=2, heads_bwd=1):
    """Whole sampled heads of a full-size workload; the backward oracle is the
    fp64 chunkwise form (no [T, T] matrices), pinned to BPTT on small inputs."""
    spec = dict(WORKLOADS[name])
    if variant is not None:
        spec["variant"] = variant
    dt = BF if spec["dtype"] == "bf16" else F32
    cpu = inputs(spec["B"], spec["NH"], spec["T"], spec["d_qk"], spec["d_hv"], seed=spec["seed"],
                 dtype=dt, ig_mean=spec["igate_mean"], fg_mean=spec["fgate_mean"])
    L, var = spec["chunk"], spec["variant"]
    dev, h, saved = gpu_fwd(cpu, L, var)
    g = gpu_bwd(dev, h, saved, L, var)
    tol = TOL[dt]
    for (b, hh) in sample_heads(spec["B"], spec["NH"], heads_fwd, spec["seed"]):
        x = head64(cpu, b, hh)
        ref = oracle_fwd_head(x, L, var)
        assert relerr(np64(h[b, hh]), ref["h"]) <= tol, f"h ({b},{hh})"
    for (b, hh) in sample_heads(spec["B"], spec["NH"], heads_bwd, spec["seed"] + 1):
        x = head64(cpu, b, hh)
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], var)
        cb = oracle.chunkwise_backward(x["q"], x["k"], x["v"], li, lf, var, L, x["dh"],
                                       h_in=io_round(oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, var, L)["h"], dt))
        di, df = oracle.preact_grads(cb["dlog_i"], cb["dlog_f"], x["igate"], x["fgate"], var)
        ref_g = {"dq": cb["dq"], "dk": cb["dk"], "dv": cb["dv"], "digate_pre": di, "dfgate_pre": df}
        floor = 1e-3 * max(np.max(np.abs(v)) for v in ref_g.values())
        for key, val in ref_g.items():
            err = relerr(np64(g[key][b, hh]), val, floor=floor)
            assert err <= tol, f"{key} ({b},{hh}): {err:.3e}"


@pytest.mark.parametrize("var", [SIG, EXP], ids=["sig", "exp"])
def test_few_heads_long_sequence_split_walks(var):
    """Two heads, 64 chunks of 256: the state walks run as 16 segments and a completion pass,
    gate_prep (mLSTMsig) spreads a head's chunks over CTAs, and the gate gradients run over 4
    segments of the sequence after their totals; both heads against the fp64 chunkwise forms."""
    Bn, NH, T, d, L = 1, 2, 16384, 64, 256
    cpu = inputs(Bn, NH, T, d, d, seed=91 + var, dtype=BF, ig_mean=-2.0 if var == EXP else 0.0,
                 fg_mean=3.0)
    dev, h, saved = gpu_fwd(cpu, L, var)
    g = gpu_bwd(dev, h, saved, L, var)
    for hh in range(NH):
        x = head64(cpu, 0, hh)
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], var)
        fwd = oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, var, L)
        assert relerr(np64(h[0, hh]), fwd["h"]) <= 1e-2, f"h head {hh}"
        cb = oracle.chunkwise_backward(x["q"], x["k"], x["v"], li, lf, var, L, x["dh"],
                                       h_in=io_round(fwd["h"], BF))
        di, df = oracle.preact_grads(cb["dlog_i"], cb["dlog_f"], x["igate"], x["fgate"], var)
        ref_g = {"dq": cb["dq"], "dk": cb["dk"], "dv": cb["dv"], "digate_pre": di, "dfgate_pre": df}
        floor = 1e-3 * max(np.max(np.abs(v)) for v in ref_g.values())
        for key, val in ref_g.items():
            err = relerr(np64(g[key][0, hh]), val, floor=floor)
            assert err <= 1e-2, f"{key} head {hh}: {err:.3e}"


def test_full_headline_exp_b8h32_t4096_fwd_bwd():
    _full("exp_b8h32_t4096_d128_c128", heads_fwd=3, heads_bwd=2)


def test_full_headline_every_head_sampled_rows():
    """Every one of the 256 heads of the headline workload (the walkers run one CTA per
    head in more than one wave) on sampled rows: h and dq on rows spread over the
    sequence, dk, dv and d igate on columns of the last chunk, each from its own row or
    column of the oracle's parallel form."""
    spec = WORKLOADS["exp_b8h32_t4096_d128_c128"]
    T, L, var = spec["T"], spec["chunk"], spec["variant"]
    cpu = inputs(spec["B"], spec["NH"], T, spec["d_qk"], spec["d_hv"], seed=spec["seed"], dtype=BF,
                 ig_mean=spec["igate_mean"], fg_mean=spec["fgate_mean"])
    dev, h, saved = gpu_fwd(cpu, L, var)
    g = gpu_bwd(dev, h, saved, L, var)
    rows = sample_rows(T, 6, spec["seed"], chunk=L)
    tail = list(range(T - L, T))
    cols = tail  # every column of the last chunk
    need = sorted(set(rows) | set(tail))
    # the bar applies per output tensor: max|err| and max|ref| over every sampled element
    # of every head
    worst = {}

    def acc(key, got, ref, at):
        e, r = float(np.max(np.abs(got - ref))), float(np.max(np.abs(ref)))
        ce, cr, ca = worst.get(key, (0.0, 0.0, None))
        worst[key] = (max(ce, e), max(cr, r), at if e > ce else ca)

    for b in range(spec["B"]):
        for hh in range(spec["NH"]):
            x = head64(cpu, b, hh)
            li, lf = oracle.gate_logs(x["igate"], x["fgate"], var)
            fr = oracle.parallel_forward_rows(x["q"], x["k"], x["v"], li, lf, var, need)
            hf = np.zeros((T, spec["d_hv"]))
            af, df = np.zeros(T), np.ones(T)
            hf[need], af[need], df[need] = fr["h"], fr["a"], fr["den"]
            acc("h", np64(h[b, hh])[rows], hf[rows], (b, hh))
            hf = io_round(hf, BF)  # the backward's h input, in the I/O dtype
            # dq of row r reads only row r of the forward
            br = oracle.parallel_backward_rows(x["q"], x["k"], x["v"], li, lf, var, x["dh"], hf, af,
                                               df, rows)
            acc("dq", np64(g["dq"][b, hh])[rows], br["dq"], (b, hh))
            # dk, dv, d log i of column s read the forward rows t >= s (all in `tail`)
            bc = oracle.parallel_backward_rows(x["q"], x["k"], x["v"], li, lf, var, x["dh"], hf, af,
                                               df, cols)
            di, _ = oracle.preact_grads(bc["dlog_i"], np.zeros(len(cols)), x["igate"][cols],
                                        x["fgate"][cols], var)
            for key, val in (("dk", bc["dk"]), ("dv", bc["dv"]), ("digate_pre", di)):
                acc(key, np64(g[key][b, hh])[cols], val, (b, hh))
    for key, (e, r, at) in worst.items():
        assert e / r <= 1e-2, f"{key}: {e / r:.3e} (largest error in head {at})"


@pytest.mark.parametrize("var", [SIG, EXP])
def test_full_training_b4h16_t8192_d256(var):
    _full("train_b4h16_t8192_d256_c256", variant=var, heads_fwd=2, heads_bwd=1)


def test_full_long_context_sig_b1h8_t65536():
    """T = 65536, d_qk 256, d_hv 512, chunk 1024: second-level tiling inside the chunk."""
    _full("sig_long_b1h8_t65536_c1024", heads_fwd=1, heads_bwd=1)


@pytest.mark.parametrize("var", [SIG, EXP])
@pytest.mark.parametrize("L", [64, 128, 256, 512, 1024])
def test_sweep_t16384_d128(var, L):
    """Chunk-size sweep at T = 16384, d 128 (the sweep's per-head shape), whole heads."""
    cpu = inputs(1, 4, 16384, 128, 128, seed=3000 + L + var, dtype=BF, ig_mean=0.0, fg_mean=3.0)
    dev, h, saved = gpu_fwd(cpu, L, var)
    g = gpu_bwd(dev, h, saved, L, var)
    for hh in (0, 3):
        x = head64(cpu, 0, hh)
        assert relerr(np64(h[0, hh]), oracle_fwd_head(x, L, var)["h"]) <= 1e-2
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], var)
        cb = oracle.chunkwise_backward(x["q"], x["k"], x["v"], li, lf, var, L, x["dh"],
                                       h_in=io_round(oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, var, L)["h"], BF))
        di, df = oracle.preact_grads(cb["dlog_i"], cb["dlog_f"], x["igate"], x["fgate"], var)
        ref_g = {"dq": cb["dq"], "dk": cb["dk"], "dv": cb["dv"], "digate_pre": di, "dfgate_pre": df}
        floor = 1e-3 * max(np.max(np.abs(v)) for v in ref_g.values())
        for key, val in ref_g.items():
            err = relerr(np64(g[key][0, hh]), val, floor=floor)
            assert err <= 1e-2, f"{key} L={L} head {hh}: {err:.3e}"


def test_sweep_igate_bias_minus10():
    """The -10 input-gate bias distribution at chunk 512."""
    for var in (SIG, EXP):
        cpu = inputs(1, 2, 8192, 128, 128, seed=3100 + var, dtype=BF, ig_mean=-10.0, fg_mean=3.0)
        dev, h, saved = gpu_fwd(cpu, 512, var)
        g = gpu_bwd(dev, h, saved, 512, var)
        x = head64(cpu, 0, 1)
        assert relerr(np64(h[0, 1]), oracle_fwd_head(x, 512, var)["h"]) <= 1e-2
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], var)
        cb = oracle.chunkwise_backward(x["q"], x["k"], x["v"], li, lf, var, 512, x["dh"],
                                       h_in=io_round(oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, var, 512)["h"], BF))
        di, df = oracle.preact_grads(cb["dlog_i"], cb["dlog_f"], x["igate"], x["fgate"], var)
        floor = 1e-3 * max(np.max(np.abs(v)) for v in (cb["dq"], cb["dk"], cb["dv"], di, df))
        for key, val in (("dq", cb["dq"]), ("dk", cb["dk"]), ("dv", cb["dv"]),
                         ("digate_pre", di), ("dfgate_pre", df)):
            assert relerr(np64(g[key][0, 1]), val, floor=floor) <= 1e-2, key


@pytest.mark.parametrize("var", [SIG, EXP], ids=["sig", "exp"])
def test_backward_same_bits_with_serial_launches(var):
    """The backward walker overlaps dq on a side stream; with every kernel on the caller's
    stream (mlstm_set_serial_launches) the gradients are bit-identical."""
    cpu = inputs(2, 3, 777, 128, 128, seed=4242 + var, dtype=BF, ig_mean=-2.0, fg_mean=3.0)
    dev, h, saved = gpu_fwd(cpu, 128, var)
    g1 = gpu_bwd(dev, h, saved, 128, var)
    binding.mlstm_set_serial_launches(True)
    try:
        g2 = gpu_bwd(dev, h, saved, 128, var)
    finally:
        binding.mlstm_set_serial_launches(False)
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key
