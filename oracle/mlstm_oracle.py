"""Plain fp64 CPU oracle for the mLSTM cell that chunkwise (TFLA) kernels compute.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may call it.  It shares no code with the CUDA
library, and it never consumes a value produced by the CUDA library.

Sources (web pages; none of them prints an equation, so the formulas below are
the plainest reading of what they state):

* "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
  (atlas.scime.ai summary), section *Approach*: the mLSTM has an exponential
  input gate with a normaliser state and a max state (mLSTMexp); the mLSTMsig
  variant swaps the exponential input gate for a sigmoid and drops the
  normaliser and max states.  Section *Problem*: chunkwise-parallel kernels
  materialise per-chunk states.
* Same title, arXiv abstract page (mlsanity.com), *Abstract*: the mLSTM is the
  xLSTM with matrix memory, a gated linear RNN computed in its
  chunkwise-parallel form, with a second level of tiling inside each chunk.
* "Gated Linear Attention Transformers with Hardware-Efficient Training",
  *Abstract*: linear attention is an RNN with a matrix-valued hidden state and
  has data-dependent gates.
* "flash-linear-attention" README (giters.com), list of computation forms:
  Parallel (quadratic, attention-like), FusedRecurrent (step by step),
  ParallelChunk (chunkwise with materialised states).

Readings taken where the pages are silent (one per item):

1. Per head, t = 1..T, with C_0 = 0 and n_0 = 0:
   q'_t = q_t / sqrt(d_qk); log f_t = logsigmoid(f~_t) for both variants;
   log i_t = logsigmoid(i~_t) (SIG) or i~_t (EXP);
   C_t = f_t C_{t-1} + i_t k_t v_t^T,   n_t = f_t n_{t-1} + i_t k_t;
   SIG: h_t = C_t^T q'_t;   EXP: h_t = C_t^T q'_t / max(|n_t . q'_t|, 1).
2. The max state m_t = max(log f_t + m_{t-1}, log i_t) with m_0 = -inf
   stabilises EXP; the stabilised output equals the plain one for any m_0.
3. No epsilon is added to the normaliser.
4. On a normaliser tie |a_t| == 1 the constant branch is taken (zero gradient).
5. The stabiliser carries no gradient (the output does not depend on it).
6. The backward receives the forward's output h as one of its inputs, in the
   I/O dtype like q, k, v and the gates.  The normaliser's gradient,
   da_t = -(dh_t . h_t) sign(a_t) / den_t, is evaluated with that h: the
   backward functions take it as ``h_in`` (None: the exact fp64 h).
"""

import numpy as np

SIG = 0
EXP = 1


# ---------------------------------------------------------------------------
# gates
# ---------------------------------------------------------------------------

def logsigmoid(x):
    """log(1 / (1 + exp(-x))) in fp64, without overflow for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    return -np.logaddexp(0.0, -x)


def sigmoid(x):
    return np.exp(logsigmoid(x))


def gate_logs(igate_pre, fgate_pre, variant):
    """Log input and forget gates from their preactivations (reading 1).

    Forget gate: sigmoid for both variants.  Input gate: exponential for
    mLSTMexp, sigmoid for mLSTMsig (TFLA summary page, *Approach*).
    """
    log_f = logsigmoid(fgate_pre)
    if variant == SIG:
        log_i = logsigmoid(igate_pre)
    elif variant == EXP:
        log_i = np.array(igate_pre, dtype=np.float64)
    else:
        raise ValueError("variant must be SIG (0) or EXP (1)")
    return log_i, log_f


def preact_grads(dlog_i, dlog_f, igate_pre, fgate_pre, variant):
    """Chain rule from d log-gate to d preactivation.

    d/dx logsigmoid(x) = sigmoid(-x); the exponential input gate of mLSTMexp
    has log i = i~, so its derivative is 1.
    """
    dfgate = np.asarray(dlog_f) * sigmoid(-np.asarray(fgate_pre, dtype=np.float64))
    if variant == SIG:
        digate = np.asarray(dlog_i) * sigmoid(-np.asarray(igate_pre, dtype=np.float64))
    else:
        digate = np.array(dlog_i, dtype=np.float64)
    return digate, dfgate


def _as64(*arrays):
    return [np.asarray(a, dtype=np.float64) for a in arrays]


# ---------------------------------------------------------------------------
# recurrent form (FusedRecurrent semantics, step by step)
# ---------------------------------------------------------------------------

def recurrent_forward(q, k, v, log_i, log_f, variant, state_steps=()):
    """Step-by-step matrix-memory recurrence, unstabilised (reading 1).

    One head: q, k [T, d_qk]; v [T, d_hv]; log_i, log_f [T].
    Returns h [T, d_hv] and, for EXP, the normaliser a_t = n_t . q'_t and the
    denominator max(|a_t|, 1).  For every j in ``state_steps`` it also returns
    C and n after j steps (j = 0 is the zero initial state).
    """
    q, k, v, log_i, log_f = _as64(q, k, v, log_i, log_f)
    T, d_qk = q.shape
    d_hv = v.shape[1]
    qs = q / np.sqrt(d_qk)
    C = np.zeros((d_qk, d_hv))
    n = np.zeros(d_qk)
    h = np.zeros((T, d_hv))
    a = np.zeros(T)
    den = np.ones(T)
    want = set(state_steps)
    states = {}
    if 0 in want:
        states[0] = (C.copy(), n.copy())
    for t in range(T):
        f_t = np.exp(log_f[t])
        i_t = np.exp(log_i[t])
        C = f_t * C + i_t * np.outer(k[t], v[t])
        n = f_t * n + i_t * k[t]
        if t + 1 in want:
            states[t + 1] = (C.copy(), n.copy())
        num = C.T @ qs[t]
        if variant == SIG:
            h[t] = num
        else:
            a[t] = n @ qs[t]
            den[t] = max(abs(a[t]), 1.0)
            h[t] = num / den[t]
    return {"h": h, "a": a, "den": den, "states": states}


def recurrent_forward_stabilised(q, k, v, log_i, log_f):
    """mLSTMexp with the max state m_t (reading 2), step by step.

    C~_t = exp(log f_t + m_{t-1} - m_t) C~_{t-1} + exp(log i_t - m_t) k_t v_t^T,
    n~ likewise, h_t = C~_t^T q'_t / max(|n~_t . q'_t|, exp(-m_t)), m_0 = -inf.
    """
    q, k, v, log_i, log_f = _as64(q, k, v, log_i, log_f)
    T, d_qk = q.shape
    d_hv = v.shape[1]
    qs = q / np.sqrt(d_qk)
    C = np.zeros((d_qk, d_hv))
    n = np.zeros(d_qk)
    m = -np.inf
    h = np.zeros((T, d_hv))
    m_all = np.zeros(T)
    abar = np.zeros(T)
    for t in range(T):
        m_new = max(log_f[t] + m, log_i[t])
        decay = np.exp(log_f[t] + m - m_new)
        inp = np.exp(log_i[t] - m_new)
        C = decay * C + inp * np.outer(k[t], v[t])
        n = decay * n + inp * k[t]
        abar[t] = n @ qs[t]
        h[t] = (C.T @ qs[t]) / max(abs(abar[t]), np.exp(-m_new))
        m = m_new
        m_all[t] = m
    return {"h": h, "m": m_all, "abar": abar}


def recurrent_step(C, n, m, q, k, v, igate_pre, fgate_pre, variant):
    """One token of the recurrence from the state of the previous token (FusedRecurrent
    form of the flash-linear-attention README; readings 1 and 2).

    SIG: C' = f C + i k v^T, h = C'^T q' (n and m are carried unchanged).
    EXP: m' = max(log f + m, log i), C' = exp(log f + m - m') C + exp(log i - m') k v^T,
    n' likewise, h = C'^T q' / max(|n' . q'|, exp(-m')).
    The zero state is C = 0, n = 0, m = -inf.  Returns (h, C', n', m').
    """
    C, n, q, k, v = _as64(C, n, q, k, v)
    log_i, log_f = gate_logs(np.float64(igate_pre), np.float64(fgate_pre), variant)
    qs = q / np.sqrt(q.shape[0])
    if variant == SIG:
        C = np.exp(log_f) * C + np.exp(log_i) * np.outer(k, v)
        return C.T @ qs, C, n, m
    m_new = max(log_f + m, log_i)
    decay = np.exp(log_f + m - m_new)
    inp = np.exp(log_i - m_new)
    C = decay * C + inp * np.outer(k, v)
    n = decay * n + inp * k
    h = (C.T @ qs) / max(abs(n @ qs), np.exp(-m_new))
    return h, C, n, m_new


# ---------------------------------------------------------------------------
# parallel (quadratic) form
# ---------------------------------------------------------------------------

def _log_decay_row(log_i, log_f, t):
    """log D_ts for s = 0..t: sum_{r=s+1}^{t} log f_r + log i_s, summed directly.

    The sums are accumulated from r = t downwards, never as a difference of two
    prefix sums, so log f = -inf (a closed forget gate) stays NaN-free.
    """
    row = np.empty(t + 1)
    row[t] = 0.0
    if t > 0:
        row[:t] = np.cumsum(log_f[t:0:-1])[::-1]
    return row + log_i[: t + 1]


def parallel_log_decay(log_i, log_f):
    """[T, T] matrix of log D_ts (-inf for s > t)."""
    log_i, log_f = _as64(log_i, log_f)
    T = log_i.shape[0]
    logD = np.full((T, T), -np.inf)
    for t in range(T):
        logD[t, : t + 1] = _log_decay_row(log_i, log_f, t)
    return logD


def parallel_forward(q, k, v, log_i, log_f, variant):
    """Quadratic attention-like form (Parallel semantics).

    A_ts = (q'_t . k_s) D_ts;  SIG: h = A V;  EXP: h_t = (A V)_t / max(|sum_s A_ts|, 1).
    """
    q, k, v, log_i, log_f = _as64(q, k, v, log_i, log_f)
    d_qk = q.shape[1]
    qs = q / np.sqrt(d_qk)
    D = np.exp(parallel_log_decay(log_i, log_f))
    A = (qs @ k.T) * D
    num = A @ v
    if variant == SIG:
        T = q.shape[0]
        return {"h": num, "a": np.zeros(T), "den": np.ones(T), "A": A}
    a = A.sum(axis=1)
    den = np.maximum(np.abs(a), 1.0)
    return {"h": num / den[:, None], "a": a, "den": den, "A": A}


# ---------------------------------------------------------------------------
# chunkwise form (ParallelChunk semantics: materialised per-chunk states)
# ---------------------------------------------------------------------------

def chunkwise_forward(q, k, v, log_i, log_f, variant, L):
    """Chunkwise-parallel form with states materialised at chunk boundaries.

    Steps in the order the kernels take them (TFLA summary page, *Problem* and
    *Approach*; arXiv abstract):

    a1. per chunk: b_t = inclusive cumsum of log f inside the chunk,
        g = b at the chunk's last row; EXP: the max state m_t of the recurrence,
        evaluated as b_t + max(m_{k-1}, max_{s<=t in chunk}(log i_s - b_s)).
    a2. state entering each chunk, C_k = exp(g_k + m_{k-1} - m_k) C_{k-1}
        + K^T diag(exp(g_k - b_s + log i_s - m_k)) V (m == 0 for SIG), n likewise.
    a3. outputs: h_t = [alpha_t q'_t C_{k-1} + sum_{s<=t} D_ts (q'_t.k_s) v_s] / den_t
        with alpha_t = exp(b_t + m_{k-1} - m_t), D_ts = exp(b_t - b_s + log i_s - m_t),
        den_t = max(|alpha_t q'_t.n_{k-1} + sum_s D_ts q'_t.k_s|, exp(-m_t)) (EXP), 1 (SIG).

    When L does not divide T the last chunk holds the remaining T mod L rows.
    """
    q, k, v, log_i, log_f = _as64(q, k, v, log_i, log_f)
    T, d_qk = q.shape
    d_hv = v.shape[1]
    if L < 1:
        raise ValueError("chunk size must be positive")
    NC = -(-T // L)
    bounds = [(c * L, min((c + 1) * L, T)) for c in range(NC)]
    qs = q / np.sqrt(d_qk)
    exp_variant = variant == EXP

    # a1: gate preprocessing
    b = np.empty(T)
    for (lo, hi) in bounds:
        b[lo:hi] = np.cumsum(log_f[lo:hi])
    g = np.array([b[hi - 1] for (_, hi) in bounds])
    m_row = np.zeros(T)
    m_state = np.zeros(NC)
    m_enter = np.zeros(NC)
    if exp_variant:
        m_prev = -np.inf
        for c, (lo, hi) in enumerate(bounds):
            sl = slice(lo, hi)
            u = np.maximum.accumulate(log_i[sl] - b[sl])
            m_row[sl] = b[sl] + np.maximum(m_prev, u)
            m_enter[c] = m_prev
            m_state[c] = m_row[hi - 1]
            m_prev = m_state[c]

    # a2: inter-chunk states (state entering chunk c)
    C_enter = np.zeros((NC, d_qk, d_hv))
    n_enter = np.zeros((NC, d_qk))
    C = np.zeros((d_qk, d_hv))
    n = np.zeros(d_qk)
    for c, (lo, hi) in enumerate(bounds):
        C_enter[c] = C
        n_enter[c] = n
        sl = slice(lo, hi)
        if exp_variant:
            beta = np.exp(g[c] + m_enter[c] - m_state[c])
            w = np.exp(g[c] - b[sl] + log_i[sl] - m_state[c])
        else:
            beta = np.exp(g[c])
            w = np.exp(g[c] - b[sl] + log_i[sl])
        C = beta * C + k[sl].T @ (w[:, None] * v[sl])
        n = beta * n + k[sl].T @ w

    # a3: outputs
    h = np.empty((T, d_hv))
    abar = np.zeros(T)
    den = np.ones(T)
    for c, (lo, hi) in enumerate(bounds):
        sl = slice(lo, hi)
        tril = np.tril(np.ones((hi - lo, hi - lo), dtype=bool))
        bt = b[sl]
        mt = m_row[sl]
        alpha = np.exp(bt + m_enter[c] - mt) if exp_variant else np.exp(bt)
        logD = bt[:, None] - bt[None, :] + log_i[sl][None, :] - mt[:, None]
        D = np.where(tril, np.exp(np.where(tril, logD, 0.0)), 0.0)
        A = (qs[sl] @ k[sl].T) * D
        num = alpha[:, None] * (qs[sl] @ C_enter[c]) + A @ v[sl]
        if exp_variant:
            abar[sl] = alpha * (qs[sl] @ n_enter[c]) + A.sum(axis=1)
            den[sl] = np.maximum(np.abs(abar[sl]), np.exp(-mt))
        h[sl] = num / den[sl][:, None]
    return {
        "h": h, "b": b, "g": g, "log_i": log_i.copy(), "m_row": m_row,
        "m_state": m_state, "m_enter": m_enter, "C_enter": C_enter,
        "n_enter": n_enter, "abar": abar, "den": den,
        # state after the last row (EXP: scaled by exp(-m_T)), what a step-by-step
        # continuation of the sequence starts from
        "C_final": C, "n_final": n, "m_final": m_state[-1] if exp_variant else 0.0,
    }


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _output_grads(dh, h, a, den, variant, floor=1.0):
    """dnum_t = dh_t / den_t and da_t for h_t = num_t / max(|a_t|, floor)."""
    dnum = dh / den[:, None]
    if variant == SIG:
        return dnum, np.zeros(dh.shape[0])
    active = np.abs(a) > floor
    da = np.where(active, -np.sum(dh * h, axis=1) * np.sign(a) / den, 0.0)
    return dnum, da


def parallel_backward(q, k, v, log_i, log_f, variant, dh, h_in=None):
    """Gradients of sum(dh * h) through the parallel form (readings 4, 5, 6).

    dA_ts = dnum_t . v_s + da_t;  dq'_t = sum_s dA_ts D_ts k_s;
    dk_s = sum_t dA_ts D_ts q'_t;  dv_s = sum_t A_ts dnum_t;
    with G_ts = dA_ts A_ts: d log i_s = sum_{t>=s} G_ts and
    d log f_r = sum_{t>=r} sum_{s<r} G_ts.
    """
    q, k, v, log_i, log_f, dh = _as64(q, k, v, log_i, log_f, dh)
    d_qk = q.shape[1]
    qs = q / np.sqrt(d_qk)
    fwd = parallel_forward(q, k, v, log_i, log_f, variant)
    A = fwd["A"]
    D = np.exp(parallel_log_decay(log_i, log_f))
    h_used = fwd["h"] if h_in is None else np.asarray(h_in, dtype=np.float64)
    dnum, da = _output_grads(dh, h_used, fwd["a"], fwd["den"], variant)
    dA = dnum @ v.T + da[:, None]
    dA = np.tril(dA)
    dS = dA * D
    dqs = dS @ k
    dk = dS.T @ qs
    dv = A.T @ dnum
    G = dA * A
    dlog_i = G.sum(axis=0)
    # sum_{s<r} G_ts for every (t, r): exclusive prefix sums along s
    excl = np.zeros_like(G)
    excl[:, 1:] = np.cumsum(G, axis=1)[:, :-1]
    dlog_f = np.tril(excl).sum(axis=0)
    return {"dq": dqs / np.sqrt(d_qk), "dk": dk, "dv": dv,
            "dlog_i": dlog_i, "dlog_f": dlog_f, "h": fwd["h"]}


def recurrent_backward(q, k, v, log_i, log_f, variant, dh):
    """Backpropagation through time of the unstabilised recurrence.

    Keeps every C_t, so it is meant for small T.  Independent of the parallel
    backward: it differentiates the step-by-step definition directly.
    """
    q, k, v, log_i, log_f, dh = _as64(q, k, v, log_i, log_f, dh)
    T, d_qk = q.shape
    d_hv = v.shape[1]
    qs = q / np.sqrt(d_qk)
    f = np.exp(log_f)
    i = np.exp(log_i)
    Cs = np.zeros((T + 1, d_qk, d_hv))
    ns = np.zeros((T + 1, d_qk))
    h = np.zeros((T, d_hv))
    a = np.zeros(T)
    den = np.ones(T)
    for t in range(T):
        Cs[t + 1] = f[t] * Cs[t] + i[t] * np.outer(k[t], v[t])
        ns[t + 1] = f[t] * ns[t] + i[t] * k[t]
        num = Cs[t + 1].T @ qs[t]
        if variant == EXP:
            a[t] = ns[t + 1] @ qs[t]
            den[t] = max(abs(a[t]), 1.0)
        h[t] = num / den[t]
    dnum, da = _output_grads(dh, h, a, den, variant)
    dC = np.zeros((d_qk, d_hv))
    dn = np.zeros(d_qk)
    dqs = np.zeros((T, d_qk))
    dk = np.zeros((T, d_qk))
    dv = np.zeros((T, d_hv))
    df = np.zeros(T)
    di = np.zeros(T)
    for t in range(T - 1, -1, -1):
        dC = dC + np.outer(qs[t], dnum[t])
        dn = dn + da[t] * qs[t]
        dqs[t] = Cs[t + 1] @ dnum[t] + da[t] * ns[t + 1]
        dk[t] = i[t] * (dC @ v[t] + dn)
        dv[t] = i[t] * (dC.T @ k[t])
        di[t] = k[t] @ dC @ v[t] + dn @ k[t]
        df[t] = np.sum(dC * Cs[t]) + dn @ ns[t]
        dC = f[t] * dC
        dn = f[t] * dn
    return {"dq": dqs / np.sqrt(d_qk), "dk": dk, "dv": dv,
            "dlog_i": di * i, "dlog_f": df * f, "h": h}


def chunkwise_backward(q, k, v, log_i, log_f, variant, L, dh, h_in=None):
    """Gradients of sum(dh * h) in the chunkwise order, fp64 (no [T, T] matrices).

    Uses the forward's chunk quantities (chunkwise_forward) with the max state
    held constant (reading 5):

    a4. reverse over chunks: dC_c, the gradient of the state leaving chunk c,
        dC_{c-1} = beta_c dC_c + sum_{t in c} alpha_t q'_t dnum_t^T and
        dn_{c-1} = beta_c dn_c + sum_{t in c} alpha_t da_t q'_t;
    a5. per chunk, with dA_ts = dnum_t . v_s + da_t and D the in-chunk decay:
        dq'_t = alpha_t (C_{c-1} dnum_t + da_t n_{c-1}) + sum_s dA_ts D_ts k_s,
        dk_s  = w_s (dC_c v_s + dn_c) + sum_t dA_ts D_ts q'_t,
        dv_s  = w_s dC_c^T k_s + sum_t D_ts (q'_t . k_s) dnum_t;
    a6. d log i_s = k_s . dk_s and d log f_r = sum_{t>=r} (q'_t.dq'_t - k_t.dk_t).
    """
    q, k, v, log_i, log_f, dh = _as64(q, k, v, log_i, log_f, dh)
    T, d_qk = q.shape
    d_hv = v.shape[1]
    qs = q / np.sqrt(d_qk)
    f = chunkwise_forward(q, k, v, log_i, log_f, variant, L)
    exp_variant = variant == EXP
    NC = -(-T // L)
    bounds = [(c * L, min((c + 1) * L, T)) for c in range(NC)]
    b, m_row, g = f["b"], f["m_row"], f["g"]
    m_state, m_enter = f["m_state"], f["m_enter"]
    den = f["den"]
    dnum = dh / den[:, None]
    if exp_variant:
        active = np.abs(f["abar"]) > np.exp(-m_row)
        h_used = f["h"] if h_in is None else np.asarray(h_in, dtype=np.float64)  # reading 6
        da = np.where(active, -np.sum(dh * h_used, axis=1) * np.sign(f["abar"]) / den, 0.0)
    else:
        da = np.zeros(T)

    def alpha_of(c, lo, hi):
        if exp_variant:
            return np.exp(b[lo:hi] + m_enter[c] - m_row[lo:hi])
        return np.exp(b[lo:hi])

    # a4: gradient of the state leaving each chunk
    dC = np.zeros((NC, d_qk, d_hv))
    dn = np.zeros((NC, d_qk))
    G = np.zeros((d_qk, d_hv))
    gn = np.zeros(d_qk)
    for c in range(NC - 1, -1, -1):
        dC[c] = G
        dn[c] = gn
        lo, hi = bounds[c]
        beta = np.exp(g[c] + m_enter[c] - m_state[c]) if exp_variant else np.exp(g[c])
        alpha = alpha_of(c, lo, hi)
        G = beta * G + (alpha[:, None] * qs[lo:hi]).T @ dnum[lo:hi]
        gn = beta * gn + (alpha * da[lo:hi]) @ qs[lo:hi]

    # a5: per-chunk gradients
    dqs = np.zeros((T, d_qk))
    dk = np.zeros((T, d_qk))
    dv = np.zeros((T, d_hv))
    for c, (lo, hi) in enumerate(bounds):
        sl = slice(lo, hi)
        n_rows = hi - lo
        tril = np.tril(np.ones((n_rows, n_rows), dtype=bool))
        bt, mt = b[sl], m_row[sl]
        logD = bt[:, None] - bt[None, :] + log_i[sl][None, :] - mt[:, None]
        D = np.where(tril, np.exp(np.where(tril, logD, 0.0)), 0.0)
        alpha = alpha_of(c, lo, hi)
        mk = m_state[c] if exp_variant else 0.0
        w = np.exp(g[c] - bt + log_i[sl] - mk)
        dA = dnum[sl] @ v[sl].T + da[sl][:, None]
        dS = dA * D
        A = (qs[sl] @ k[sl].T) * D
        dqs[sl] = dS @ k[sl] + alpha[:, None] * (dnum[sl] @ f["C_enter"][c].T
                                                  + da[sl][:, None] * f["n_enter"][c][None, :])
        dk[sl] = dS.T @ qs[sl] + w[:, None] * (v[sl] @ dC[c].T + dn[c][None, :])
        dv[sl] = A.T @ dnum[sl] + w[:, None] * (k[sl] @ dC[c])

    # a6: gate gradients from the per-token dot products
    pq = np.einsum("td,td->t", qs, dqs)
    pk = np.einsum("td,td->t", k, dk)
    dlog_f = np.cumsum((pq - pk)[::-1])[::-1]
    return {"dq": dqs / np.sqrt(d_qk), "dk": dk, "dv": dv, "dlog_i": pk, "dlog_f": dlog_f,
            "h": f["h"], "den": den, "dC_leave": dC}


# ---------------------------------------------------------------------------
# single rows / columns, for sequences too long for the [T, T] matrices
# ---------------------------------------------------------------------------

def parallel_forward_rows(q, k, v, log_i, log_f, variant, rows):
    """h_t (and a_t, den_t) for the listed rows t, each from its own row of A."""
    q, k, v, log_i, log_f = _as64(q, k, v, log_i, log_f)
    d_qk = q.shape[1]
    qs = q / np.sqrt(d_qk)
    out_h, out_a, out_den = [], [], []
    for t in rows:
        A_row = (k[: t + 1] @ qs[t]) * np.exp(_log_decay_row(log_i, log_f, t))
        num = A_row @ v[: t + 1]
        if variant == SIG:
            out_h.append(num); out_a.append(0.0); out_den.append(1.0)
        else:
            a_t = A_row.sum()
            d_t = max(abs(a_t), 1.0)
            out_h.append(num / d_t); out_a.append(a_t); out_den.append(d_t)
    return {"h": np.array(out_h), "a": np.array(out_a), "den": np.array(out_den)}


def _log_decay_col(log_i, log_f, s):
    """log D_ts for t = s..T-1: log i_s + sum_{r=s+1}^{t} log f_r, summed forward."""
    T = log_i.shape[0]
    col = np.empty(T - s)
    col[0] = 0.0
    if T - s > 1:
        col[1:] = np.cumsum(log_f[s + 1 :])
    return col + log_i[s]


def parallel_backward_rows(q, k, v, log_i, log_f, variant, dh, h, a, den, rows):
    """dq for rows t, and dk, dv, d log i for columns s, of the parallel form.

    h, a, den are the forward results for all T rows (any oracle forward);
    dq_t needs row t only, dk_s / dv_s / d log i_s need rows t >= s.
    """
    q, k, v, log_i, log_f, dh, h, a, den = _as64(q, k, v, log_i, log_f, dh, h, a, den)
    d_qk = q.shape[1]
    qs = q / np.sqrt(d_qk)
    dnum, da = _output_grads(dh, h, a, den, variant)
    dq, dk, dv, dli = [], [], [], []
    for r in rows:
        D_row = np.exp(_log_decay_row(log_i, log_f, r))
        dA_row = v[: r + 1] @ dnum[r] + da[r]
        dq.append(((dA_row * D_row) @ k[: r + 1]) / np.sqrt(d_qk))
        D_col = np.exp(_log_decay_col(log_i, log_f, r))
        dA_col = dnum[r:] @ v[r] + da[r:]
        S_col = qs[r:] @ k[r]
        dk.append((dA_col * D_col) @ qs[r:])
        dv.append((S_col * D_col) @ dnum[r:])
        dli.append(np.sum(dA_col * S_col * D_col))
    return {"dq": np.array(dq), "dk": np.array(dk), "dv": np.array(dv),
            "dlog_i": np.array(dli)}


# ---------------------------------------------------------------------------
# batched helpers ([B, NH, T, d] arrays, heads independent)
# ---------------------------------------------------------------------------

def backward_heads(q, k, v, igate_pre, fgate_pre, variant, dh):
    """Parallel-form backward on every head, returning preactivation gradients."""
    res = {n: np.empty(x.shape, dtype=np.float64) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("digate", igate_pre), ("dfgate", fgate_pre))}
    B, NH = q.shape[:2]
    for bb in range(B):
        for hh in range(NH):
            li, lf = gate_logs(igate_pre[bb, hh], fgate_pre[bb, hh], variant)
            g = parallel_backward(q[bb, hh], k[bb, hh], v[bb, hh], li, lf, variant, dh[bb, hh])
            di, df = preact_grads(g["dlog_i"], g["dlog_f"], igate_pre[bb, hh], fgate_pre[bb, hh], variant)
            res["dq"][bb, hh] = g["dq"]; res["dk"][bb, hh] = g["dk"]; res["dv"][bb, hh] = g["dv"]
            res["digate"][bb, hh] = di; res["dfgate"][bb, hh] = df
    return res
