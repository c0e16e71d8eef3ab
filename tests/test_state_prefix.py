"""Pins of the state-as-prefix construction (tests/_state_prefix.py), fp64, CPU.

The construction is checked against things other than itself:
* the oracle's one-token step started from the state (C, n, m) gives the same
  outputs as the oracle's parallel form over prefix + tokens, and the same final
  state as its chunkwise form (compared as unstabilised states, which do not
  depend on where the max state happens to sit);
* the state gradient read off the prefix tokens' dk, dv matches central finite
  differences of the stepped loss with respect to the state's entries.
"""

import numpy as np
import pytest

import oracle
from _state_prefix import extend, prefix, random_state, state_grads, true_state

SIG, EXP = oracle.SIG, oracle.EXP


def _tokens(rng, T, d_qk, d_hv, variant):
    q = rng.standard_normal((T, d_qk))
    k = rng.standard_normal((T, d_qk))
    v = rng.standard_normal((T, d_hv))
    ig = rng.standard_normal(T) + (-2.0 if variant == EXP else 0.0)
    fg = rng.standard_normal(T) + 2.0
    return q, k, v, ig, fg


def _steps(C, n, m, q, k, v, ig, fg, variant):
    d_qk = C.shape[0]
    n = np.zeros(d_qk) if n is None else n
    hs = []
    for t in range(q.shape[0]):
        h, C, n, m = oracle.recurrent_step(C, n, m, q[t], k[t], v[t], ig[t], fg[t], variant)
        hs.append(h)
    return np.array(hs), C, n, m


def _rel(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(1.0, float(np.max(np.abs(b)))))


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
def test_prefix_reproduces_steps_from_state(variant):
    rng = np.random.default_rng(11)
    d_qk, d_hv, T = 8, 6, 13
    C, n, m = random_state(rng, d_qk, d_hv, variant)
    if variant == EXP:
        n = n * np.array([1, -1, -1, 1, 1, -1, 1, -1])
    q, k, v, ig, fg = _tokens(rng, T, d_qk, d_hv, variant)
    h_ref, C_T, n_T, m_T = _steps(C.copy(), None if n is None else n.copy(), m, q, k, v, ig, fg,
                                  variant)
    li, lf = oracle.gate_logs(ig, fg, variant)
    ext = extend(prefix(C, n, m, variant), q, k, v, li, lf)
    h_par = oracle.parallel_forward(*ext, variant)["h"]
    assert _rel(h_par[:d_qk], np.zeros((d_qk, d_hv))) == 0.0  # the prefix rows read nothing
    assert _rel(h_par[d_qk:], h_ref) < 1e-10
    cw = oracle.chunkwise_forward(*ext, variant, 4)
    got_C, got_n = true_state(cw["C_final"], cw["n_final"], cw["m_final"], variant)
    ref_C, ref_n = true_state(C_T, n_T, m_T, variant)
    assert _rel(got_C, ref_C) < 1e-10
    if variant == EXP:
        assert _rel(got_n, ref_n) < 1e-10


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
def test_prefix_state_gradient_matches_finite_differences(variant):
    rng = np.random.default_rng(12)
    d_qk, d_hv, T = 6, 5, 9
    C, n, m = random_state(rng, d_qk, d_hv, variant)
    if variant == EXP:
        n = n * np.array([1, -1, 1, -1, -1, 1])  # the construction takes either sign
    q, k, v, ig, fg = _tokens(rng, T, d_qk, d_hv, variant)
    dh = rng.standard_normal((T, d_hv))
    li, lf = oracle.gate_logs(ig, fg, variant)
    pre = prefix(C, n, m, variant)
    ext = extend(pre, q, k, v, li, lf)
    dh_ext = np.concatenate([np.zeros((d_qk, d_hv)), dh])
    g = oracle.parallel_backward(*ext, variant, dh_ext)
    dC, dn = state_grads(pre, g["dk"][:d_qk], g["dv"][:d_qk], m, variant)

    def loss(Cx, nx):
        h, _, _, _ = _steps(Cx, nx, m, q, k, v, ig, fg, variant)
        return float(np.sum(dh * h))

    eps = 1e-6
    for (j, c) in [(0, 0), (2, 3), (5, 1)]:
        Cp, Cm = C.copy(), C.copy()
        Cp[j, c] += eps
        Cm[j, c] -= eps
        fd = (loss(Cp, n) - loss(Cm, n)) / (2 * eps)
        assert abs(fd - dC[j, c]) <= 1e-6 * max(1.0, abs(fd)), (j, c, fd, dC[j, c])
    if variant == EXP:
        for j in (0, 3):
            npl, nmi = n.copy(), n.copy()
            npl[j] += eps
            nmi[j] -= eps
            fd = (loss(C, npl) - loss(C, nmi)) / (2 * eps)
            assert abs(fd - dn[j]) <= 1e-6 * max(1.0, abs(fd)), (j, fd, dn[j])


@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
def test_final_state_term_gradients_match_finite_differences(variant):
    """The closed form in _state_prefix.final_state_term_grads against central finite
    differences of <W, C_T> + <w, n_T> over the oracle's unstabilised recurrence."""
    from _state_prefix import final_state_term_grads
    rng = np.random.default_rng(13)
    d_qk, d_hv, T = 5, 4, 11
    q, k, v, ig, fg = _tokens(rng, T, d_qk, d_hv, variant)
    W = rng.standard_normal((d_qk, d_hv))
    w = rng.standard_normal(d_qk) if variant == EXP else None

    def loss(k_, v_, ig_, fg_):
        li, lf = oracle.gate_logs(ig_, fg_, variant)
        C, n = oracle.recurrent_forward(q, k_, v_, li, lf, variant, state_steps=(T,))["states"][T]
        return float(np.sum(W * C) + (w @ n if w is not None else 0.0))

    li, lf = oracle.gate_logs(ig, fg, variant)
    g = final_state_term_grads(q, k, v, li, lf, W, w)
    di, df = oracle.preact_grads(g["dlog_i"], g["dlog_f"], ig, fg, variant)
    eps = 1e-6

    def fd(arr, idx, which):
        a, b = arr.copy(), arr.copy()
        a[idx] += eps
        b[idx] -= eps
        args_a = {"k": k, "v": v, "ig": ig, "fg": fg, which: a}
        args_b = {"k": k, "v": v, "ig": ig, "fg": fg, which: b}
        return (loss(args_a["k"], args_a["v"], args_a["ig"], args_a["fg"])
                - loss(args_b["k"], args_b["v"], args_b["ig"], args_b["fg"])) / (2 * eps)

    for idx in [(0, 1), (6, 3), (10, 0)]:
        assert abs(fd(k, idx, "k") - g["dk"][idx]) <= 1e-6 * max(1.0, abs(g["dk"][idx]))
    for idx in [(2, 2), (9, 1)]:
        assert abs(fd(v, idx, "v") - g["dv"][idx]) <= 1e-6 * max(1.0, abs(g["dv"][idx]))
    for t in (0, 5, 10):
        assert abs(fd(ig, t, "ig") - di[t]) <= 1e-6 * max(1.0, abs(di[t]))
        assert abs(fd(fg, t, "fg") - df[t]) <= 1e-6 * max(1.0, abs(df[t]))
