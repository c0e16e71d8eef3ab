"""Pins of the fp64 oracle to facts outside itself.

Each check ties one oracle function to a hand-worked value, a closed form, a
different evaluation order of the same definition, finite differences, or an
identity the mathematics fixes.  Every check takes the oracle module as an
argument so that ``test_planted_mistake_is_caught`` can run all of them against
copies of the oracle with one plausible bug planted each, and show that at
least one check fails for every such bug.  None of this needs a GPU.
"""

import inspect
import json
import os
import types

import numpy as np
import pytest

import oracle
from oracle import mlstm_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SIG, EXP = 0, 1


def rnd(seed, T, d_qk, d_hv, ig_mean=0.0, fg_mean=3.0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, d_qk))
    k = r.standard_normal((T, d_qk))
    v = r.standard_normal((T, d_hv))
    ig = r.standard_normal(T) + ig_mean
    fg = r.standard_normal(T) + fg_mean
    return q, k, v, ig, fg


def rel(a, b):
    return np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------------------
# checks (each raises AssertionError on disagreement)
# ---------------------------------------------------------------------------

def check_hand_cases(M):
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 5
    for case in cases:
        q, k, v = (np.array(case[n], float) for n in ("q", "k", "v"))
        li, lf = np.array(case["log_i"], float), np.array(case["log_f"], float)
        var = SIG if case["variant"] == "sig" else EXP
        want = np.array(case["h"], float)
        got = [M.recurrent_forward(q, k, v, li, lf, var)["h"],
               M.parallel_forward(q, k, v, li, lf, var)["h"],
               M.chunkwise_forward(q, k, v, li, lf, var, 1)["h"]]
        if var == EXP:
            got.append(M.recurrent_forward_stabilised(q, k, v, li, lf)["h"])
        for g in got:
            np.testing.assert_allclose(g, want, rtol=1e-12, atol=1e-12, err_msg=case["name"])


def check_logsigmoid(M):
    assert abs(M.logsigmoid(0.0) + np.log(2.0)) < 1e-15
    assert abs(M.logsigmoid(-800.0) + 800.0) < 1e-12
    assert M.logsigmoid(800.0) == 0.0
    assert abs(M.logsigmoid(np.log(3.0)) - np.log(0.75)) < 1e-14
    assert abs(M.sigmoid(np.log(3.0)) - 0.75) < 1e-14
    li, lf = M.gate_logs(np.array([np.log(3.0)]), np.array([np.log(3.0)]), EXP)
    assert abs(li[0] - np.log(3.0)) < 1e-15 and abs(lf[0] - np.log(0.75)) < 1e-14
    li, _ = M.gate_logs(np.array([np.log(3.0)]), np.array([0.0]), SIG)
    assert abs(li[0] - np.log(0.75)) < 1e-14


def check_open_gates(M, T=9, d_qk=4, d_hv=5):
    """i = f = 1 under SIG: h_t = sum_{s<=t} (q'_t . k_s) v_s = tril(Q'K^T) V."""
    q, k, v, _, _ = rnd(1, T, d_qk, d_hv)
    zeros = np.zeros(T)
    want = np.tril(q @ k.T / np.sqrt(d_qk)) @ v
    assert rel(M.recurrent_forward(q, k, v, zeros, zeros, SIG)["h"], want) < 1e-13
    assert rel(M.parallel_forward(q, k, v, zeros, zeros, SIG)["h"], want) < 1e-13
    for L in (1, T):
        assert rel(M.chunkwise_forward(q, k, v, zeros, zeros, SIG, L)["h"], want) < 1e-13
    li, lf = M.gate_logs(np.full(T, 800.0), np.full(T, 800.0), SIG)
    assert rel(M.recurrent_forward(q, k, v, li, lf, SIG)["h"], want) < 1e-13


def check_closed_forget(M, variant):
    """f = 0: C_t = i_t k_t v_t^T only, so h_t is a single outer-product readout."""
    T, d_qk, d_hv = 12, 4, 3
    q, k, v, ig, _ = rnd(2, T, d_qk, d_hv)
    li, _ = M.gate_logs(ig, np.zeros(T), variant)
    s = np.einsum("td,td->t", q, k) / np.sqrt(d_qk)
    if variant == SIG:
        want = (1.0 / (1.0 + np.exp(-ig)) * s)[:, None] * v
    else:
        want = (s / np.maximum(np.abs(s), np.exp(-ig)))[:, None] * v
    closed = np.full(T, -np.inf)
    assert rel(M.recurrent_forward(q, k, v, li, closed, variant)["h"], want) < 1e-13
    assert rel(M.parallel_forward(q, k, v, li, closed, variant)["h"], want) < 1e-13
    nearly = np.full(T, -1000.0)  # exp(-1000) == 0 in fp64 and the cumsums stay finite
    for L in (1, 3, 4, 12):
        assert rel(M.chunkwise_forward(q, k, v, li, nearly, variant, L)["h"], want) < 1e-13
    if variant == EXP:
        assert rel(M.recurrent_forward_stabilised(q, k, v, li, nearly)["h"], want) < 1e-13


def check_retention(M):
    """Constant f = gamma, i = 1 under SIG: h_t = sum_s gamma^(t-s) (q'_t.k_s) v_s."""
    T, d = 20, 6
    q, k, v, _, _ = rnd(3, T, d, d)
    gamma = 0.9
    idx = np.arange(T)
    lag = idx[:, None] - idx[None, :]
    decay = np.where(lag >= 0, gamma ** np.clip(lag, 0, None), 0.0)
    want = ((q @ k.T / np.sqrt(d)) * decay) @ v
    li, lf = np.zeros(T), np.full(T, np.log(gamma))
    assert rel(M.recurrent_forward(q, k, v, li, lf, SIG)["h"], want) < 1e-12
    assert rel(M.parallel_forward(q, k, v, li, lf, SIG)["h"], want) < 1e-12
    for L in (1, 4, 5, 20):
        assert rel(M.chunkwise_forward(q, k, v, li, lf, SIG, L)["h"], want) < 1e-12


def check_single_token(M):
    """T = 1: h_1 = i_1 (q'_1 . k_1) v_1 (SIG); EXP divides by max(|i_1 q'.k|, 1)."""
    q, k, v, ig, fg = rnd(4, 1, 5, 3, 1.0)
    s = float(q[0] @ k[0]) / np.sqrt(5)
    li, lf = M.gate_logs(ig, fg, SIG)
    np.testing.assert_allclose(M.recurrent_forward(q, k, v, li, lf, SIG)["h"][0],
                               s * v[0] / (1.0 + np.exp(-ig[0])), rtol=1e-14)
    li, lf = M.gate_logs(ig, fg, EXP)
    i1 = np.exp(ig[0])
    np.testing.assert_allclose(M.recurrent_forward(q, k, v, li, lf, EXP)["h"][0],
                               i1 * s * v[0] / max(abs(i1 * s), 1.0), rtol=1e-14)


def check_steps(M, variant, seed=51):
    """Stepping token by token from the zero state reproduces the recurrent forms (which
    the closed forms above pin), and the chunkwise form's final state is the state after
    the last step, with a ragged last chunk."""
    q, k, v, ig, fg = rnd(seed, 23, 4, 5, 3.0)
    C, n, m = np.zeros((4, 5)), np.zeros(4), -np.inf
    hs = []
    for t in range(23):
        h, C, n, m = M.recurrent_step(C, n, m, q[t], k[t], v[t], ig[t], fg[t], variant)
        hs.append(h)
    li, lf = M.gate_logs(ig, fg, variant)
    ref = (M.recurrent_forward(q, k, v, li, lf, SIG)["h"] if variant == SIG
           else M.recurrent_forward_stabilised(q, k, v, li, lf)["h"])
    np.testing.assert_allclose(np.array(hs), ref, rtol=1e-11, atol=1e-13)
    cw = M.chunkwise_forward(q, k, v, li, lf, variant, 7)
    np.testing.assert_allclose(cw["C_final"], C, rtol=1e-11, atol=1e-13)
    if variant == EXP:
        np.testing.assert_allclose(cw["n_final"], n, rtol=1e-11, atol=1e-13)
        assert abs(cw["m_final"] - m) < 1e-12


def check_parallel_vs_recurrent(M, variant, seed=5, ig_mean=0.0, fg_mean=3.0):
    q, k, v, ig, fg = rnd(seed, 40, 8, 6, ig_mean, fg_mean)
    li, lf = M.gate_logs(ig, fg, variant)
    r = M.recurrent_forward(q, k, v, li, lf, variant)
    p = M.parallel_forward(q, k, v, li, lf, variant)
    assert rel(p["h"], r["h"]) < 1e-12
    if variant == EXP:
        assert rel(p["a"], r["a"]) < 1e-12


def check_stabilised(M, seed=9, ig_mean=0.0):
    q, k, v, ig, fg = rnd(seed, 50, 6, 4, ig_mean, 3.0)
    li, lf = M.gate_logs(ig, fg, EXP)
    r = M.recurrent_forward(q, k, v, li, lf, EXP)
    s = M.recurrent_forward_stabilised(q, k, v, li, lf)
    assert rel(s["h"], r["h"]) < 1e-12
    assert rel(s["abar"] * np.exp(s["m"]), r["a"]) < 1e-12
    # the max state is the recurrence m_t = max(log f_t + m_{t-1}, log i_t)
    m = -np.inf
    for t in range(len(ig)):
        m = max(lf[t] + m, li[t])
        assert abs(s["m"][t] - m) < 1e-12


def check_huge_input_gates(M):
    """Preactivations near 700 overflow exp() unless the max state is used."""
    q, k, v, ig, fg = rnd(13, 16, 4, 4, 700.0, 3.0)
    li, lf = M.gate_logs(ig, fg, EXP)
    s = M.recurrent_forward_stabilised(q, k, v, li, lf)
    assert np.all(np.isfinite(s["h"]))
    # a constant shift of log i scales C and n alike, so h is unchanged wherever
    # the shifted normaliser is still above the floor
    shifted = M.recurrent_forward(q, k, v, li - 700.0, lf, EXP)
    mask = np.abs(shifted["a"]) > 1.0
    assert mask.sum() >= 3
    assert rel(s["h"][mask], shifted["h"][mask]) < 1e-12
    assert rel(M.chunkwise_forward(q, k, v, li, lf, EXP, 4)["h"], s["h"]) < 1e-12


def check_chunk_invariance(M, variant, T=50, L=16):
    q, k, v, ig, fg = rnd(100 + T + L, T, 8, 5, -1.0, 2.0)
    li, lf = M.gate_logs(ig, fg, variant)
    r = M.recurrent_forward(q, k, v, li, lf, variant)["h"]
    c = M.chunkwise_forward(q, k, v, li, lf, variant, L)
    assert rel(c["h"], r) < 1e-12
    if variant == EXP:
        s = M.recurrent_forward_stabilised(q, k, v, li, lf)
        np.testing.assert_allclose(c["m_row"], s["m"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(c["abar"], s["abar"], rtol=1e-11, atol=1e-12)


def check_chunk_states(M, variant):
    """C entering chunk c is the recurrence's C after c*L steps (times exp(-m))."""
    T, L = 48, 8
    q, k, v, ig, fg = rnd(14, T, 6, 5, -2.0, 3.0)
    li, lf = M.gate_logs(ig, fg, variant)
    steps = list(range(0, T, L))
    r = M.recurrent_forward(q, k, v, li, lf, variant, state_steps=steps)
    c = M.chunkwise_forward(q, k, v, li, lf, variant, L)
    m = M.recurrent_forward_stabilised(q, k, v, li, lf)["m"] if variant == EXP else None
    for j, st in enumerate(steps):
        C, n = r["states"][st]
        scale = 1.0 if variant == SIG or st == 0 else np.exp(-m[st - 1])
        np.testing.assert_allclose(c["C_enter"][j], C * scale, rtol=1e-11, atol=1e-13)
        if variant == EXP:
            np.testing.assert_allclose(c["n_enter"][j], n * scale, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(c["m_enter"][j], -np.inf if st == 0 else m[st - 1])
    np.testing.assert_allclose(c["g"], lf.reshape(-1, L).sum(axis=1), rtol=1e-13)


def _loss(M, q, k, v, ig, fg, dh, variant):
    li, lf = M.gate_logs(ig, fg, variant)
    return float(np.sum(dh * M.recurrent_forward(q, k, v, li, lf, variant)["h"]))


def check_finite_differences(M, variant, seed=20):
    T, d_qk, d_hv = 6, 3, 3
    for attempt in range(50):
        q, k, v, ig, fg = rnd(seed * 100 + attempt, T, d_qk, d_hv, 0.5, 1.0)
        if variant == SIG:
            break
        li, lf = oracle.gate_logs(ig, fg, variant)
        a = oracle.recurrent_forward(q, k, v, li, lf, variant)["a"]
        if np.all(np.abs(np.abs(a) - 1.0) > 1e-3):  # stay off the normaliser kink
            break
    dh = np.random.default_rng(seed).standard_normal((T, d_hv))
    li, lf = M.gate_logs(ig, fg, variant)
    g = M.parallel_backward(q, k, v, li, lf, variant, dh)
    dig, dfg = M.preact_grads(g["dlog_i"], g["dlog_f"], ig, fg, variant)
    analytic = {"q": g["dq"], "k": g["dk"], "v": g["dv"], "ig": dig, "fg": dfg}
    args = {"q": q, "k": k, "v": v, "ig": ig, "fg": fg}
    eps = 1e-6
    for name, x in args.items():
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            num[idx] = (_loss(M, **{**args, name: xp}, dh=dh, variant=variant)
                        - _loss(M, **{**args, name: xm}, dh=dh, variant=variant)) / (2 * eps)
        np.testing.assert_allclose(analytic[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def check_bptt(M, variant, seed=30, ig_mean=0.0):
    q, k, v, ig, fg = rnd(seed, 24, 5, 4, ig_mean, 2.0)
    dh = np.random.default_rng(seed + 1).standard_normal((24, 4))
    li, lf = M.gate_logs(ig, fg, variant)
    p = M.parallel_backward(q, k, v, li, lf, variant, dh)
    r = M.recurrent_backward(q, k, v, li, lf, variant, dh)
    for name in ("dq", "dk", "dv", "dlog_i", "dlog_f"):
        assert rel(p[name], r[name]) < 1e-11, name


def check_chunkwise_backward(M, variant, T=50, L=16, seed=33):
    """The chunkwise backward agrees with BPTT, including a ragged last chunk."""
    q, k, v, ig, fg = rnd(seed, T, 6, 5, -1.0, 2.0)
    dh = np.random.default_rng(seed + 1).standard_normal((T, 5))
    li, lf = M.gate_logs(ig, fg, variant)
    r = M.recurrent_backward(q, k, v, li, lf, variant, dh)
    cb = M.chunkwise_backward(q, k, v, li, lf, variant, L, dh)
    for name in ("dq", "dk", "dv", "dlog_i", "dlog_f"):
        assert rel(cb[name], r[name]) < 1e-10, name


def check_identities(M, variant):
    """d log i_s = k_s.dk_s and d log f_r = sum_{t>=r} (q'_t.dq'_t - k_t.dk_t)."""
    T = 32
    q, k, v, ig, fg = rnd(40, T, 6, 5, -0.5, 2.0)
    dh = np.random.default_rng(41).standard_normal((T, 5))
    li, lf = M.gate_logs(ig, fg, variant)
    for g in (M.recurrent_backward(q, k, v, li, lf, variant, dh),
              M.parallel_backward(q, k, v, li, lf, variant, dh)):
        pk = np.einsum("td,td->t", k, g["dk"])
        pq = np.einsum("td,td->t", q, g["dq"])  # q . dq == q' . dq'
        assert rel(pk, g["dlog_i"]) < 1e-11
        assert rel(np.cumsum((pq - pk)[::-1])[::-1], g["dlog_f"]) < 1e-11
        assert abs(g["dlog_f"][0]) < 1e-12 * np.max(np.abs(g["dlog_f"]))  # f_1 scales C_0 = 0


def check_rows(M, variant):
    T = 40
    q, k, v, ig, fg = rnd(50, T, 6, 5, -1.0, 2.0)
    dh = np.random.default_rng(51).standard_normal((T, 5))
    li, lf = M.gate_logs(ig, fg, variant)
    rows = [0, 1, 17, 39]
    full = M.parallel_forward(q, k, v, li, lf, variant)
    part = M.parallel_forward_rows(q, k, v, li, lf, variant, rows)
    assert rel(part["h"], full["h"][rows]) < 1e-13
    rec = M.recurrent_forward(q, k, v, li, lf, variant)
    g = M.recurrent_backward(q, k, v, li, lf, variant, dh)
    gr = M.parallel_backward_rows(q, k, v, li, lf, variant, dh, rec["h"], rec["a"], rec["den"], rows)
    for name in ("dq", "dk", "dv", "dlog_i"):
        assert rel(gr[name], g[name][rows]) < 1e-11, name


def check_normaliser_tie(M):
    """Reading 4, by hand: one mLSTMexp token with |a| exactly 1 takes the constant branch.

    d_qk = 4, q = k = (1, 1, 0, 0), log i = 0: C = k v^T, n = k, q' = q / 2, so
    a = n . q' = 1 = the floor (exp(-m) with m = log i = 0 in the stabilised forms) and
    h = C^T q' / 1 = v.  With den held at the floor, L = dh . h = (dh . v)(k . q') gives
    dq = (dh . v) k / 2, dk = (dh . v) q / 2, dv = dh, d log i = dh . v, d log f = 0.
    Taking the |a| branch instead would make h = v (k . q') / (k . q') and dq = dk = 0.
    """
    q = np.array([[1.0, 1.0, 0.0, 0.0]])
    k = q.copy()
    v = np.array([[0.5, -1.0, 2.0]])
    dh = np.array([[1.0, 2.0, -0.5]])
    li, lf = np.array([0.0]), np.array([M.logsigmoid(3.0)])
    dhv = float(dh[0] @ v[0])  # -2.5
    want = {"dq": dhv * k / 2, "dk": dhv * q / 2, "dv": dh, "dlog_i": np.array([dhv]),
            "dlog_f": np.array([0.0])}
    got = [M.parallel_backward(q, k, v, li, lf, EXP, dh), M.recurrent_backward(q, k, v, li, lf, EXP, dh),
           M.chunkwise_backward(q, k, v, li, lf, EXP, 1, dh), M.chunkwise_backward(q, k, v, li, lf, EXP, 4, dh)]
    for g in got:
        np.testing.assert_allclose(g["h"], v, rtol=0, atol=1e-15)
        for name, w in want.items():
            np.testing.assert_allclose(g[name], w, rtol=0, atol=1e-14, err_msg=name)


ALL_CHECKS = [
    check_normaliser_tie,
    check_hand_cases, check_logsigmoid, check_open_gates,
    lambda M: check_closed_forget(M, SIG), lambda M: check_closed_forget(M, EXP),
    check_retention, check_single_token,
    lambda M: check_parallel_vs_recurrent(M, SIG), lambda M: check_parallel_vs_recurrent(M, EXP),
    check_stabilised, check_huge_input_gates,
    lambda M: check_chunk_invariance(M, SIG), lambda M: check_chunk_invariance(M, EXP),
    lambda M: check_chunk_states(M, SIG), lambda M: check_chunk_states(M, EXP),
    lambda M: check_bptt(M, SIG), lambda M: check_bptt(M, EXP),
    lambda M: check_identities(M, SIG), lambda M: check_identities(M, EXP),
    lambda M: check_chunkwise_backward(M, SIG), lambda M: check_chunkwise_backward(M, EXP),
    lambda M: check_rows(M, SIG), lambda M: check_rows(M, EXP),
    lambda M: check_finite_differences(M, SIG), lambda M: check_finite_differences(M, EXP),
    lambda M: check_steps(M, SIG), lambda M: check_steps(M, EXP),
]


# ---------------------------------------------------------------------------
# the pins, on the real oracle
# ---------------------------------------------------------------------------

def test_normaliser_tie_takes_the_constant_branch():
    check_normaliser_tie(oracle)


@pytest.mark.parametrize("variant", [SIG, EXP])
def test_steps_and_final_state(variant):
    check_steps(oracle, variant)


def test_hand_worked_cases():
    check_hand_cases(oracle)


def test_logsigmoid_known_values():
    check_logsigmoid(oracle)


@pytest.mark.parametrize("T,d_qk,d_hv", [(1, 3, 2), (9, 4, 5), (33, 8, 8)])
def test_sig_open_gates_is_causal_linear_attention(T, d_qk, d_hv):
    check_open_gates(oracle, T, d_qk, d_hv)


@pytest.mark.parametrize("variant", [SIG, EXP])
def test_closed_forget_gate_is_one_step_readout(variant):
    check_closed_forget(oracle, variant)


def test_constant_decay_is_retention():
    check_retention(oracle)


def test_single_token():
    check_single_token(oracle)


@pytest.mark.parametrize("variant", [SIG, EXP])
@pytest.mark.parametrize("seed,ig_mean,fg_mean", [(5, 0.0, 3.0), (6, -2.0, 3.0), (7, 2.0, 0.0), (8, -10.0, 4.0)])
def test_parallel_equals_recurrent(variant, seed, ig_mean, fg_mean):
    check_parallel_vs_recurrent(oracle, variant, seed, ig_mean, fg_mean)


@pytest.mark.parametrize("seed,ig_mean", [(9, 0.0), (10, -2.0), (11, 5.0), (12, -10.0)])
def test_stabilised_equals_unstabilised(seed, ig_mean):
    check_stabilised(oracle, seed, ig_mean)


def test_stabilised_survives_huge_input_gates():
    check_huge_input_gates(oracle)


@pytest.mark.parametrize("variant", [SIG, EXP])
@pytest.mark.parametrize("T,L", [(8, 1), (8, 2), (8, 4), (8, 8), (48, 16), (64, 64), (60, 12),
                                 (50, 16), (7, 4), (5, 8), (33, 32)])
def test_chunkwise_invariant_to_chunk_size(variant, T, L):
    check_chunk_invariance(oracle, variant, T, L)


@pytest.mark.parametrize("variant", [SIG, EXP])
def test_chunk_states_are_recurrent_states(variant):
    check_chunk_states(oracle, variant)


@pytest.mark.parametrize("variant", [SIG, EXP])
@pytest.mark.parametrize("seed", [20, 21, 22])
def test_backward_matches_finite_differences(variant, seed):
    check_finite_differences(oracle, variant, seed)


@pytest.mark.parametrize("variant", [SIG, EXP])
@pytest.mark.parametrize("seed,ig_mean", [(30, 0.0), (31, -2.0), (32, 1.5)])
def test_parallel_backward_equals_bptt(variant, seed, ig_mean):
    check_bptt(oracle, variant, seed, ig_mean)


@pytest.mark.parametrize("variant", [SIG, EXP])
@pytest.mark.parametrize("T,L,seed", [(50, 16, 33), (48, 8, 34), (7, 4, 35), (40, 40, 36), (33, 1, 37)])
def test_chunkwise_backward_equals_bptt(variant, T, L, seed):
    check_chunkwise_backward(oracle, variant, T, L, seed)


@pytest.mark.parametrize("variant", [SIG, EXP])
def test_gate_gradient_identities(variant):
    check_identities(oracle, variant)


@pytest.mark.parametrize("variant", [SIG, EXP])
def test_row_evaluators_match_full(variant):
    check_rows(oracle, variant)


# ---------------------------------------------------------------------------
# planted mistakes: a copy of the oracle with one bug must fail some check
# ---------------------------------------------------------------------------

MUTATIONS = [
    ("logsigmoid sign", "return -np.logaddexp(0.0, -x)", "return -np.logaddexp(0.0, x)"),
    ("exp input gate squashed", "log_i = np.array(igate_pre, dtype=np.float64)", "log_i = logsigmoid(igate_pre)"),
    ("normaliser floor dropped", "den[t] = max(abs(a[t]), 1.0)\n            h[t] = num / den[t]",
     "den[t] = abs(a[t])\n            h[t] = num / den[t]"),
    ("input gate dropped", "C = f_t * C + i_t * np.outer(k[t], v[t])", "C = f_t * C + np.outer(k[t], v[t])"),
    ("decay row off by one", "row[:t] = np.cumsum(log_f[t:0:-1])[::-1]", "row[:t] = np.cumsum(log_f[t - 1::-1])[::-1]"),
    ("state decay term dropped", "beta = np.exp(g[c] + m_enter[c] - m_state[c])\n            w =",
     "beta = np.exp(m_enter[c] - m_state[c])\n            w ="),
    ("state weight sign", "w = np.exp(g[c] - b[sl] + log_i[sl] - m_state[c])", "w = np.exp(g[c] + b[sl] + log_i[sl] - m_state[c])"),
    ("max state missing b", "m_row[sl] = b[sl] + np.maximum(m_prev, u)", "m_row[sl] = np.maximum(m_prev, u)"),
    ("inter-chunk factor missing b", "alpha = np.exp(bt + m_enter[c] - mt) if exp_variant", "alpha = np.exp(m_enter[c] - mt) if exp_variant"),
    ("stabilised floor 1", "max(abs(abar[t]), np.exp(-m_new))", "max(abs(abar[t]), 1.0)"),
    ("step decay dropped", "C = decay * C + inp * np.outer(k, v)\n    n = decay * n + inp * k\n    h = (C.T",
     "C = C + inp * np.outer(k, v)\n    n = decay * n + inp * k\n    h = (C.T"),
    ("step floor 1", "h = (C.T @ qs) / max(abs(n @ qs), np.exp(-m_new))", "h = (C.T @ qs) / max(abs(n @ qs), 1.0)"),
    ("final state one chunk early", '"C_final": C, "n_final"', '"C_final": C_enter[-1], "n_final"'),
    ("dk transposed", "dk = dS.T @ qs", "dk = dS @ qs"),
    ("dlog_f summed on the wrong axis", "dlog_f = np.tril(excl).sum(axis=0)", "dlog_f = np.tril(excl).sum(axis=1)"),
    ("da sign", "da = np.where(active, -np.sum(dh * h, axis=1)", "da = np.where(active, np.sum(dh * h, axis=1)"),
    ("normaliser tie takes the |a| branch", "active = np.abs(a) > floor", "active = np.abs(a) >= floor"),
    ("stabilised tie takes the |a| branch", 'active = np.abs(f["abar"]) > np.exp(-m_row)',
     'active = np.abs(f["abar"]) >= np.exp(-m_row)'),
    ("forget chain rule sign", "dfgate = np.asarray(dlog_f) * sigmoid(-np.asarray(fgate_pre", "dfgate = np.asarray(dlog_f) * sigmoid(np.asarray(fgate_pre"),
    ("bptt forget grad uses C_t", "df[t] = np.sum(dC * Cs[t]) + dn @ ns[t]", "df[t] = np.sum(dC * Cs[t + 1]) + dn @ ns[t]"),
    ("column dA misses da", "dA_col = dnum[r:] @ v[r] + da[r:]", "dA_col = dnum[r:] @ v[r]"),
    ("state gradient misses the decay", "G = beta * G + (alpha[:, None] * qs[lo:hi]).T @ dnum[lo:hi]",
     "G = G + (alpha[:, None] * qs[lo:hi]).T @ dnum[lo:hi]"),
    ("dk misses the state gradient", "dk[sl] = dS.T @ qs[sl] + w[:, None] * (v[sl] @ dC[c].T + dn[c][None, :])",
     "dk[sl] = dS.T @ qs[sl] + w[:, None] * dn[c][None, :]"),
    ("dv uses the state entering the chunk", "dv[sl] = A.T @ dnum[sl] + w[:, None] * (k[sl] @ dC[c])",
     "dv[sl] = A.T @ dnum[sl] + w[:, None] * (k[sl] @ dC[c - 1])"),
    ("chunk mask misses diagonal", "tril = np.tril(np.ones((hi - lo, hi - lo), dtype=bool))",
     "tril = np.tril(np.ones((hi - lo, hi - lo), dtype=bool), -1)"),
    ("chunk decay taken at the wrong row", "g = np.array([b[hi - 1] for (_, hi) in bounds])",
     "g = np.array([b[lo] for (lo, _) in bounds])"),
]


def _mutant(old, new):
    src = inspect.getsource(mlstm_oracle)
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new):
    M = _mutant(old, new)
    caught = False
    for check in ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(M)
        except Exception:  # an AssertionError, or the mutant crashing outright
            caught = True
            break
    assert caught, f"no pin catches the planted mistake: {name}"


def test_unmutated_copy_passes_every_check():
    M = _mutant("SIG = 0", "SIG = 0")
    for check in ALL_CHECKS:
        check(M)


@pytest.mark.parametrize("variant", [SIG, EXP])
def test_backward_forms_agree_for_a_given_h_input(variant):
    """Reading 6: the backward takes the output h as an input.  For any h_in (here the
    exact h perturbed by a relative 1e-3), the parallel and chunkwise backward forms use
    it in the normaliser gradient alike and agree; h_in = the exact h reproduces the
    default; and for mLSTMsig (no normaliser) h_in changes nothing."""
    rng = np.random.default_rng(61)
    T, d, L = 45, 8, 8
    q, k, v, dh = (rng.standard_normal((T, d)) for _ in range(4))
    li, lf = oracle.gate_logs(rng.standard_normal(T) - 1.0, rng.standard_normal(T) + 2.0, variant)
    h = oracle.parallel_forward(q, k, v, li, lf, variant)["h"]
    h_in = h * (1.0 + 1e-3 * rng.standard_normal(h.shape))
    p = oracle.parallel_backward(q, k, v, li, lf, variant, dh, h_in=h_in)
    c = oracle.chunkwise_backward(q, k, v, li, lf, variant, L, dh, h_in=h_in)
    for key in ("dq", "dk", "dv", "dlog_i", "dlog_f"):
        np.testing.assert_allclose(c[key], p[key], rtol=1e-9, atol=1e-11)
    same = oracle.parallel_backward(q, k, v, li, lf, variant, dh, h_in=h)
    dflt = oracle.parallel_backward(q, k, v, li, lf, variant, dh)
    for key in ("dq", "dk", "dv", "dlog_i", "dlog_f"):
        np.testing.assert_array_equal(same[key], dflt[key])
        if variant == SIG:
            np.testing.assert_allclose(p[key], dflt[key], rtol=1e-12, atol=1e-14)
    if variant == EXP:  # the perturbation reaches the gradients through da only
        assert np.max(np.abs(p["dq"] - dflt["dq"])) > 0
