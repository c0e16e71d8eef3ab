"""Seeded synthetic inputs for the mLSTM chunkwise kernels.

This module draws random tensors and names the workloads; it holds none of the
method's arithmetic.  Tensors are drawn on the CPU with ``torch.Generator`` in
fp32, in the order q, k, v, input-gate preactivation, forget-gate
preactivation, upstream gradient dh, and then rounded to the I/O dtype, so the
same seed gives the same values whichever consumer (GPU path or CPU oracle)
reads them.

The workloads are the kernel benchmarks of "Tiled Flash Linear Attention: More
Efficient Linear RNN and xLSTM Kernels" (TFLA summary page, *Key results* and
*Measured effects*) with synthetic data: q, k, v ~ N(0, 1), gate
preactivations ~ N(mean, 1).  The -10 input-gate mean stands for the -10
input-gate bias initialisation the same page reports (*Measured effects*).
"""

import torch

SIG = 0
EXP = 1

# name -> shape, chunk, variant, I/O dtype, gate distributions, seed, passes
WORKLOADS = {
    # small fp32 case the oracle finishes in seconds
    "sig_fwd_fp32_b1h2_t256_d64": dict(
        B=1, NH=2, T=256, d_qk=64, d_hv=64, chunk=64, variant=SIG, dtype="fp32",
        igate_mean=0.0, fgate_mean=3.0, seed=0, passes="fwd"),
    # the headline workload: B8 H32 d128 T4096, chunk 128
    "exp_b8h32_t4096_d128_c128": dict(
        B=8, NH=32, T=4096, d_qk=128, d_hv=128, chunk=128, variant=EXP, dtype="bf16",
        igate_mean=-2.0, fgate_mean=3.0, seed=2, passes="fwd"),
    # training pass B4 H16 T8192 d256, chunk 256
    "train_b4h16_t8192_d256_c256": dict(
        B=4, NH=16, T=8192, d_qk=256, d_hv=256, chunk=256, variant=EXP, dtype="bf16",
        igate_mean=0.0, fgate_mean=3.0, seed=4, passes="fwdbwd"),
    # long context B1 H8 T65536 d_qk 256 d_hv 512, chunk 1024
    "sig_long_b1h8_t65536_c1024": dict(
        B=1, NH=8, T=65536, d_qk=256, d_hv=512, chunk=1024, variant=SIG, dtype="bf16",
        igate_mean=-10.0, fgate_mean=4.0, seed=5, passes="fwdbwd"),
}

# chunk-size / sequence-length sweep at B8 H32 d128
SWEEP_T = (1024, 2048, 4096, 8192, 16384)
SWEEP_CHUNK = (64, 128, 256, 512, 1024)
SWEEP_SEED = 3


def torch_dtype(name):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_inputs(B, NH, T, d_qk, d_hv, *, seed, igate_mean=0.0, fgate_mean=3.0,
                igate_std=1.0, fgate_std=1.0, qk_mean=0.0, dtype=torch.bfloat16, with_dh=False):
    """Draw q, k, v [B,NH,T,d], gate preactivations [B,NH,T] (and dh) on the CPU.

    q and k are N(qk_mean, 1); everything else as in the module docstring.
    """
    g = torch.Generator().manual_seed(int(seed))
    out = {}
    out["q"] = (torch.randn(B, NH, T, d_qk, generator=g) + qk_mean).to(dtype)
    out["k"] = (torch.randn(B, NH, T, d_qk, generator=g) + qk_mean).to(dtype)
    out["v"] = torch.randn(B, NH, T, d_hv, generator=g).to(dtype)
    out["igate"] = (torch.randn(B, NH, T, generator=g) * igate_std + igate_mean).to(dtype)
    out["fgate"] = (torch.randn(B, NH, T, generator=g) * fgate_std + fgate_mean).to(dtype)
    if with_dh:
        out["dh"] = torch.randn(B, NH, T, d_hv, generator=g).to(dtype)
    return out


def make_workload(name, with_dh=None, **overrides):
    spec = dict(WORKLOADS[name])
    spec.update(overrides)
    if with_dh is None:
        with_dh = spec["passes"] == "fwdbwd"
    t = make_inputs(spec["B"], spec["NH"], spec["T"], spec["d_qk"], spec["d_hv"],
                    seed=spec["seed"], igate_mean=spec["igate_mean"],
                    fgate_mean=spec["fgate_mean"], dtype=torch_dtype(spec["dtype"]),
                    with_dh=with_dh)
    return spec, t


def sample_heads(B, NH, n, seed):
    """n distinct (b, h) pairs chosen by the seed."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    perm = torch.randperm(B * NH, generator=g)[: min(n, B * NH)].tolist()
    return [(p // NH, p % NH) for p in sorted(perm)]


def sample_rows(T, n, seed, chunk=None):
    """n token indices: the first and last rows, chunk edges, and seeded picks."""
    g = torch.Generator().manual_seed(int(seed) + 104729)
    rows = {0, T - 1}
    if chunk:
        rows.update({min(chunk - 1, T - 1), min(chunk, T - 1)})
    rows.update(torch.randint(0, T, (max(n - len(rows), 0),), generator=g).tolist())
    return sorted(rows)


# ---------------------------------------------------------------------------
# Retention (RetNet) inputs: constant gates that make mLSTMsig a retention
# ---------------------------------------------------------------------------

#: input-gate preactivation whose log-sigmoid is 0 to fp32 rounding (input gate 1)
RETENTION_IGATE = 30.0


def retnet_decays(num_heads):
    """RetNet's per-head decay schedule gamma_h = 1 - 2^(-5 - h), fp64."""
    return 1.0 - torch.pow(2.0, -5.0 - torch.arange(num_heads, dtype=torch.float64))


def retention_gates(gamma, B, T, dtype, device):
    """Gate preactivations [B, NH, T] for a retention with decay gamma[h] per head.

    The input gate is RETENTION_IGATE everywhere and the forget gate of head h is
    logit(gamma_h), both rounded to the I/O dtype; the decay the mLSTMsig cell then
    applies is the sigmoid of that rounded forget preactivation.
    """
    g = torch.as_tensor(gamma, dtype=torch.float64).cpu()
    NH = g.numel()
    fg_h = (torch.log(g) - torch.log1p(-g)).to(dtype)
    fg = fg_h.view(1, NH, 1).expand(B, NH, T).contiguous().to(device)
    ig = torch.full((B, NH, T), RETENTION_IGATE, dtype=dtype, device=device)
    return ig, fg
