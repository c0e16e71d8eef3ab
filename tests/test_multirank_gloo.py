"""Multi-process host logic on CPU: world-size 2 and 3 process groups over gloo.

* seqpar.forward, the sequence-parallel protocol (state-only pass, all-gather of
  the segments' states and log decays, chaining, forward from the incoming
  state), with its device steps replaced by fp64 stand-ins on the oracle: every
  rank's outputs must equal the oracle's over the whole sequence for its
  segment, which checks the exchange, the rank order and the chaining order;
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
        seg = seqpar.forward(mine, L, variant, ops=OracleOps(d, variant))
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
