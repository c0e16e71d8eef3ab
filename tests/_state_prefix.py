"""A recurrent state written as a prefix of tokens (test construction, fp64).

Starting the mLSTM recurrence from a state (C, n, m) is the same as running it
from the zero state over d_qk extra tokens placed first, whose only effect on
every later token is to leave exactly that state behind:
  token j = 0 .. d_qk - 1:  k_j = s_j e_j (s_j = +-1, e_j a unit vector), q_j = 0,
  log f_j = 0, so after them the unstabilised state is C = sum_j i_j k_j v_j^T
  (row j is s_j i_j v_j) and n = sum_j i_j k_j (entry j is s_j i_j).
  SIG (no normaliser): s_j = 1, i_j = 1/2, v_j = 2 C[j].
  EXP: the stabilised state (C~, n~, m) stands for exp(m) (C~, n~); with
  s_j = sign(n~_j), i_j = exp(m) |n~_j| (n~_j != 0 is needed) and v_j = C~[j] / n~_j.
Their own outputs are zero (q = 0) and dropped.  Later tokens then see the
state decayed by their own forget gates, as in the recurrence started from it,
so the oracle's forward and backward over the longer sequence give the
expected values of a call that starts from a state, with no new oracle code;
test_state_prefix.py pins the construction against the oracle's own
one-token step.
"""

import numpy as np

import oracle


def prefix(C, n, m, variant):
    """q, k, v, log_i, log_f of the d_qk prefix tokens for the state (C, n, m) of one head."""
    C = np.asarray(C, dtype=np.float64)
    d_qk, _ = C.shape
    k = np.eye(d_qk)
    q = np.zeros((d_qk, d_qk))
    log_f = np.zeros(d_qk)
    if variant == oracle.SIG:
        log_i = np.full(d_qk, np.log(0.5))
        v = 2.0 * C
    else:
        n = np.asarray(n, dtype=np.float64)
        assert np.all(n != 0), "the construction needs a normaliser state without zeros"
        k = np.diag(np.sign(n))
        log_i = float(m) + np.log(np.abs(n))
        v = C / n[:, None]
    return q, k, v, log_i, log_f


def extend(pre, q, k, v, log_i, log_f):
    """The prefix followed by the real tokens."""
    return tuple(np.concatenate([np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)])
                 for a, b in zip(pre, (q, k, v, log_i, log_f)))


def state_grads(pre, dk_pre, dv_pre, m, variant):
    """Gradient of the loss with respect to the stabilised state (C~, n~), from the
    prefix tokens' dk, dv (m held constant).

    Row j of the true C is s_j i_j v_j, so dL/dC_true[j] = dv_j / (s_j i_j); entry j of
    the true n is s_j i_j (k_j = s_j e_j enters C and n through its entry j), so
    dk_j[j] = i_j (dC_true[j] . v_j + dn_true[j]).  The stabilised state is exp(-m) times the true one, so its
    gradient is exp(m) times the true gradient (exp(m) = 1 for SIG).
    """
    _, k, v, log_i, _ = pre
    i = np.exp(log_i)
    sgn = np.diagonal(k)
    dC_true = dv_pre / (sgn * i)[:, None]
    scale = 1.0 if variant == oracle.SIG else float(np.exp(m))
    dC = scale * dC_true
    dn = None
    if variant == oracle.EXP:
        diag = np.diagonal(dk_pre)
        dn_true = diag / i - np.sum(dC_true * v, axis=1)
        dn = scale * dn_true
    return dC, dn


def true_state(C, n, m, variant):
    """exp(m) (C, n): the unstabilised state (SIG: C itself)."""
    if variant == oracle.SIG:
        return np.asarray(C, dtype=np.float64), None
    s = float(np.exp(m))
    return s * np.asarray(C, dtype=np.float64), s * np.asarray(n, dtype=np.float64)


def random_state(rng, d_qk, d_hv, variant, scale=0.3):
    """A state of one head: C ~ N(0, scale^2), n~ in [0.5, 2) (EXP), m ~ N(0, 1) (EXP)."""
    C = rng.standard_normal((d_qk, d_hv)) * scale
    if variant == oracle.SIG:
        return C, None, 0.0
    n = rng.uniform(0.5, 2.0, d_qk)
    m = float(rng.standard_normal())
    return C, n, m


def final_state_term_grads(q, k, v, log_i, log_f, W, w):
    """Gradients of <W, C_T> + <w, n_T> (unstabilised final state after the last token)
    with respect to k, v, log i and log f, in closed form (fp64); q does not enter.

    With D_s = exp(sum_{r > s} log f_r + log i_s) the decay from token s to the end,
    C_T = sum_s D_s k_s v_s^T and n_T = sum_s D_s k_s, so with l_s = D_s (k_s^T W v_s + k_s.w):
    dk_s = D_s (W v_s + w), dv_s = D_s W^T k_s, d log i_s = l_s, d log f_r = sum_{s < r} l_s.
    """
    k, v, log_i, log_f = (np.asarray(a, dtype=np.float64) for a in (k, v, log_i, log_f))
    T = k.shape[0]
    after = np.concatenate([np.cumsum(log_f[::-1])[::-1][1:], [0.0]])  # sum_{r > s} log f_r
    D = np.exp(after + log_i)
    Wv = v @ W.T                                   # row s: W v_s
    lam = D * (np.sum(k * Wv, axis=1) + (k @ w if w is not None else 0.0))
    dk = D[:, None] * (Wv + (w[None, :] if w is not None else 0.0))
    dv = D[:, None] * (k @ W)
    dlog_f = np.concatenate([[0.0], np.cumsum(lam)[:-1]])
    return {"dq": np.zeros_like(np.asarray(q, dtype=np.float64)), "dk": dk, "dv": dv,
            "dlog_i": lam, "dlog_f": dlog_f}
