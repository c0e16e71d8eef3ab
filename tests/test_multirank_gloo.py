"""Multi-process host logic on CPU: world-size 2 and 3 process groups over gloo.

* seqpar.forward and seqpar.backward, the sequence-parallel protocol (state-only
  pass, all-gather of the segments' states and log decays, chaining, forward from
  the incoming state; each segment's own initial-state gradient, all-gather,
  carried back to the earlier segments, backward with that final-state gradient),
  with their device steps replaced by fp64 stand-ins on the oracle: every rank's
  outputs and gradients must equal the oracle's over the whole sequence for its
  segment, which checks the exchanges, the rank order and the chaining order;
* bench.reduce_max, the max-over-ranks of the timed region.
No GPU: the ranks are CPU processes (spawned, rendezvous on 127.0.0.1).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from _state_prefix import extend, final_state_term_grads, prefix, state_grads

SIG, EXP = oracle.SIG, oracle.EXP


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed, B, NH, T, d, variant):
    rng = np.random.default_rng(seed)
    x = {"q": rng.standard_normal((B, NH, T, d)), "k": rng.standard_normal((B, NH, T, d)),
         "v": rng.standard_normal((B, NH, T, d)),
         "igate": rng.standard_normal((B, NH, T)) + (-2.0 if variant == EXP else 0.0),
         "fgate": rng.standard_normal((B, NH, T)) + 2.0}
    return {k: torch.from_numpy(v) for k, v in x.items()}


class OracleOps:
    """fp64 stand-ins for seqpar's device steps; a state is a float64 tensor
    [B*NH, d*d + d + 1] holding (C, n, m) per head, a decay [B*NH]."""

    def __init__(self, d, variant):
        self.d, self.variant = d, variant

    def _heads(self, x):
        B, NH = x["q"].shape[:2]
        for bb in range(B):
            for hh in range(NH):
                yield bb * NH + hh, {k: v[bb, hh].numpy() for k, v in x.items()}

    def local_state(self, x, chunk, variant):
        B, NH = x["q"].shape[:2]
        d = self.d
        state = torch.zeros(B * NH, d * d + d + 1, dtype=torch.float64)
        decay = torch.zeros(B * NH, dtype=torch.float64)
        for i, h in self._heads(x):
            li, lf = oracle.gate_logs(h["igate"], h["fgate"], variant)
            f = oracle.chunkwise_forward(h["q"], h["k"], h["v"], li, lf, variant, chunk)
            state[i, : d * d] = torch.from_numpy(f["C_final"].reshape(-1))
            if variant == EXP:
                state[i, d * d: d * d + d] = torch.from_numpy(f["n_final"])
                state[i, -1] = f["m_final"]
            decay[i] = float(lf.sum())
        return state, decay

    def chain(self, a, b, g, sizes, variant):
        d = self.d
        out = torch.empty_like(a)
        for i in range(a.shape[0]):
            if variant == SIG:
                fa, fb, m = np.exp(g[i].item()), 1.0, 0.0
            else:
                x, y = g[i].item() + a[i, -1].item(), b[i, -1].item()
                m = max(x, y)
                fa, fb = np.exp(x - m), np.exp(y - m)
            out[i, : d * d + d] = fa * a[i, : d * d + d] + fb * b[i, : d * d + d]
            out[i, -1] = m
        return out

    def _unpack(self, s):
        d = self.d
        return s[: d * d].reshape(d, d).copy(), s[d * d: d * d + d].copy(), float(s[-1])

    def _pack(self, C, n):
        d = self.d
        out = torch.zeros(d * d + d + 1, dtype=torch.float64)
        out[: d * d] = torch.from_numpy(C.reshape(-1))
        if n is not None:
            out[d * d: d * d + d] = torch.from_numpy(n)
        return out

    def _extended(self, h, state_in_i, variant):
        """A head's tokens, behind the prefix that stands for its initial state."""
        li, lf = oracle.gate_logs(h["igate"], h["fgate"], variant)
        args = (h["q"], h["k"], h["v"], li, lf)
        if state_in_i is None:
            return None, args
        C, n, m = self._unpack(state_in_i.numpy())
        pre = prefix(C, n if variant == EXP else None, m, variant)
        return pre, extend(pre, *args)

    def local_dstate(self, x, dh, seg, chunk, variant):
        out = torch.zeros_like(seg.states[-1])
        if seg.state_in is None:
            return out
        for i, h in self._heads(x):
            pre, ext = self._extended(h, seg.state_in[i], variant)
            d = self.d
            dhx = np.concatenate([np.zeros((d, dh.shape[-1])), dh[i // x["q"].shape[1], i % x["q"].shape[1]].numpy()])
            bw = oracle.parallel_backward(*ext, variant, dhx)
            m = self._unpack(seg.state_in[i].numpy())[2]
            dC, dn = state_grads(pre, bw["dk"][:d], bw["dv"][:d], m, variant)
            out[i] = self._pack(dC, dn)
        return out

    def dchain(self, dlocal, dout, state_in, state_out, log_decay, sizes, variant):
        if dout is None:
            return dlocal.clone()
        out = dlocal.clone()
        for i in range(dlocal.shape[0]):
            g = log_decay[i].item()
            f = np.exp(g) if variant == SIG else np.exp(g + state_in[i, -1].item() - state_out[i, -1].item())
            out[i, :-1] = dlocal[i, :-1] + f * dout[i, :-1]
        return out

    def backward_from(self, x, dh, seg, chunk, variant, dstate_out):
        d = self.d
        NH = x["q"].shape[1]
        res = {k: torch.zeros_like(x[n]) for k, n in (("dq", "q"), ("dk", "k"), ("dv", "v"),
                                                      ("digate_pre", "igate"), ("dfgate_pre", "fgate"))}
        for i, h in self._heads(x):
            pre, ext = self._extended(h, None if seg.state_in is None else seg.state_in[i], variant)
            p = 0 if pre is None else d
            dhx = dh[i // NH, i % NH].numpy()
            if p:
                dhx = np.concatenate([np.zeros((d, dhx.shape[-1])), dhx])
            bw = oracle.parallel_backward(*ext, variant, dhx)
            g = {k: bw[k][p:] for k in ("dq", "dk", "dv", "dlog_i", "dlog_f")}
            if dstate_out is not None:
                dC, dn, _ = self._unpack(dstate_out[i].numpy())
                m_T = self._unpack(seg.states[seg.index + 1][i].numpy())[2] if variant == EXP else 0.0
                s = float(np.exp(-m_T))
                fs = final_state_term_grads(*ext, s * dC, s * dn if variant == EXP else None)
                for k in ("dk", "dv", "dlog_i", "dlog_f"):
                    g[k] = g[k] + fs[k][p:]
            di, df = oracle.preact_grads(g["dlog_i"], g["dlog_f"], h["igate"], h["fgate"], variant)
            for k, val in (("dq", g["dq"]), ("dk", g["dk"]), ("dv", g["dv"]), ("digate_pre", di),
                           ("dfgate_pre", df)):
                res[k][i // NH, i % NH] = torch.from_numpy(val)
        return res

    def forward_from(self, x, chunk, variant, state_in, keep_saved):
        """The oracle's one-token step from the incoming state (any state)."""
        d = self.d
        h_out = torch.empty_like(x["v"])
        NH = x["q"].shape[1]
        for i, h in self._heads(x):
            if state_in is None:
                C, n, m = np.zeros((d, d)), np.zeros(d), -np.inf
            else:
                s = state_in[i].numpy()
                C, n, m = s[: d * d].reshape(d, d).copy(), s[d * d: d * d + d].copy(), float(s[-1])
            for t in range(h["q"].shape[0]):
                out, C, n, m = oracle.recurrent_step(C, n, m, h["q"][t], h["k"][t], h["v"][t],
                                                     h["igate"][t], h["fgate"][t], variant)
                h_out[i // NH, i % NH, t] = torch.from_numpy(out)
        return h_out, None


def _seqpar_worker(rank, world, port, variant):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mlstm_chunkwise_attention_b200 import seqpar
        B, NH, T, d, L = 1, 2, 60 * world, 8, 16
        x = _problem(91, B, NH, T, d, variant)
        T_loc = T // world
        mine = {k: v[:, :, rank * T_loc:(rank + 1) * T_loc].contiguous() for k, v in x.items()}
        ops = OracleOps(d, variant)
        seg = seqpar.forward(mine, L, variant, ops=ops)
        for bb in range(B):
            for hh in range(NH):
                h = {k: v[bb, hh].numpy() for k, v in x.items()}
                li, lf = oracle.gate_logs(h["igate"], h["fgate"], variant)
                ref = oracle.parallel_forward(h["q"], h["k"], h["v"], li, lf, variant)["h"]
                got = seg.h[bb, hh].numpy()
                want = ref[rank * T_loc:(rank + 1) * T_loc]
                err = np.max(np.abs(got - want)) / max(1.0, np.max(np.abs(want)))
                assert err < 1e-9, (rank, hh, err)
        assert (seg.state_in is None) == (rank == 0)
        # backward: this rank's gradients against the whole-sequence backward
        rng = np.random.default_rng(92)
        dh_all = torch.from_numpy(rng.standard_normal((B, NH, T, d)))
        dh = dh_all[:, :, rank * T_loc:(rank + 1) * T_loc].contiguous()
        g = seqpar.backward(mine, dh, seg, L, variant, ops=ops)
        ref = oracle.backward_heads(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(),
                                    x["igate"].numpy(), x["fgate"].numpy(), variant, dh_all.numpy())
        sl = slice(rank * T_loc, (rank + 1) * T_loc)
        for key, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("digate_pre", "digate"),
                        ("dfgate_pre", "dfgate")):
            want = ref[rk][:, :, sl]
            err = np.max(np.abs(g[key].numpy() - want)) / max(1.0, np.max(np.abs(want)))
            assert err < 1e-8, (rank, key, err)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _reduce_max_worker(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench.reduce_max(1.5 + rank, world, torch.device("cpu"))
        assert got == 1.5 + world - 1, got
        assert bench.reduce_max(7.0, 1, torch.device("cpu")) == 7.0
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("variant", [SIG, EXP], ids=["sig", "exp"])
def test_seqpar_protocol_gloo(world, variant):
    mp.start_processes(_seqpar_worker, args=(world, _free_port(), variant), nprocs=world,
                       start_method="spawn", join=True)


def test_reduce_max_gloo():
    mp.start_processes(_reduce_max_worker, args=(2, _free_port()), nprocs=2,
                       start_method="spawn", join=True)
