"""Sequence-parallel chunkwise forward and backward: one segment of every head's
sequence per rank.

"Tiled Flash Linear Attention" (TFLA summary page, Problem and Approach): the
chunkwise form carries everything a later chunk needs in the state at a chunk
boundary, so a boundary may as well lie between two GPUs.  Rank r holds tokens
[r T_loc, (r + 1) T_loc) of every head.

Forward, exactly:
1. its segment's final state from the zero state (state-only pass, no output
   kernel) and the segment's total log forget gate G_r;
2. an all-gather of the (state, G) pairs over the process group: B * NH *
   (d_qk * d_hv (+ d_qk + 1)) fp32 per rank;
3. the state entering every segment, chaining the segments' states:
   S_in(0) = zero, S_in(r + 1) = chain(S_in(r), S_r, G_r);
4. its segment's outputs from S_in(r) (mlstm_fwd_state).

Backward (the max states held constant, as everywhere):
1. its segment's own share of the gradient with respect to S_in(r) (the
   state-gradient-only pass with dstate_out = 0);
2. an all-gather of those shares;
3. the gradient with respect to its segment's final state: the later
   segments' shares carried back through each segment (mlstm_dstate_chain),
   starting from the gradient with respect to the sequence's final state;
4. its segment's full backward with that final-state gradient.

Every device step runs in the library's kernels; this module only orders the
calls and the exchanges.
"""

from dataclasses import dataclass


@dataclass
class Segment:
    """One rank's share of a forward: h [B, NH, T_loc, d_hv]; the state entering its
    segment (None on rank 0); the states entering every segment and the sequence's
    final state (states[r] for segment r, states[world] the final one); every
    segment's log decay; its saved buffer (None unless kept); and its index (rank)."""
    h: object
    state_in: object
    states: list
    decays: list
    saved: object
    index: int = 0


class DeviceOps:
    """The device operations of the protocol, on the CUDA library."""

    def __init__(self):
        from . import binding
        self.b = binding

    def local_state(self, x, chunk, variant):
        _, _, state = self.b.forward_state(x["q"], x["k"], x["v"], x["igate"], x["fgate"], chunk,
                                           variant, None, keep_saved=False, want_h=False)
        return state, self.b.log_decay(x["fgate"])

    def chain(self, state_a, state_b, log_decay_b, sizes, variant):
        B, NH, d_qk, d_hv = sizes
        return self.b.state_chain(state_a, state_b, log_decay_b, B, NH, d_qk, d_hv, variant)

    def forward_from(self, x, chunk, variant, state_in, keep_saved):
        h, saved, _ = self.b.forward_state(x["q"], x["k"], x["v"], x["igate"], x["fgate"], chunk,
                                           variant, state_in, keep_saved=keep_saved)
        return h, saved

    def local_dstate(self, x, dh, seg, chunk, variant):
        if seg.state_in is None:  # nothing reads the zero state's gradient
            import torch
            return torch.zeros_like(seg.states[-1])
        return self.b.state_gradient(x["q"], x["k"], x["v"], x["igate"], x["fgate"], seg.h, dh,
                                     seg.saved, chunk, variant, seg.state_in)

    def dchain(self, dlocal, dout, state_in, state_out, log_decay, sizes, variant):
        import torch
        B, NH, d_qk, d_hv = sizes
        if dout is None:
            dout = torch.zeros_like(dlocal)
        return self.b.dstate_chain(dlocal, dout, state_in, state_out, log_decay, B, NH, d_qk,
                                   d_hv, variant)

    def backward_from(self, x, dh, seg, chunk, variant, dstate_out):
        return self.b.backward_state(x["q"], x["k"], x["v"], x["igate"], x["fgate"], seg.h, dh,
                                     seg.saved, chunk, variant, seg.state_in,
                                     dstate_out=dstate_out, want_dstate=False)


def chain_states(states_local, decays, sizes, variant, ops):
    """The state entering every segment and the final one: [None, S_in(1), ..., S_in(P)]."""
    out = [None]
    for r, (s, g) in enumerate(zip(states_local, decays)):
        out.append(s if r == 0 else ops.chain(out[-1], s, g, sizes, variant))
    return out


def final_state_gradient(rank, dlocals, states, decays, sizes, variant, ops, dstate_final=None):
    """Gradient with respect to segment ``rank``'s final state: the later segments' own
    shares carried back through each segment, from the sequence's final-state gradient
    (None: zero).  None when it is zero (the last segment, no final-state term)."""
    dout = dstate_final
    for r in range(len(dlocals) - 1, rank, -1):
        dout = ops.dchain(dlocals[r], dout, states[r], states[r + 1], decays[r], sizes, variant)
    return dout


def _sizes(x):
    B, NH, _, d_qk = x["q"].shape
    return (B, NH, d_qk, x["v"].shape[-1])


def forward(x, chunk, variant, *, group=None, ops=None, keep_saved=False):
    """This rank's segment of a sequence-parallel forward.

    x: dict of this rank's q, k [B, NH, T_loc, d_qk], v [B, NH, T_loc, d_hv], igate,
    fgate [B, NH, T_loc] (device tensors); every rank passes the same B, NH, d and
    chunk, and the segments follow rank order.  Collectives: two all-gathers over
    ``group`` (torch.distributed), taken by every rank in the same order.
    keep_saved=True keeps what ``backward`` needs.
    """
    import torch.distributed as dist
    ops = ops or DeviceOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    sizes = _sizes(x)
    state, decay = ops.local_state(x, chunk, variant)
    states = [state.new_empty(state.shape) for _ in range(world)]
    decays = [decay.new_empty(decay.shape) for _ in range(world)]
    dist.all_gather(states, state, group=group)
    dist.all_gather(decays, decay, group=group)
    chained = chain_states(states, decays, sizes, variant, ops)
    h, saved = ops.forward_from(x, chunk, variant, chained[rank], keep_saved)
    return Segment(h=h, state_in=chained[rank], states=chained, decays=decays, saved=saved,
                   index=rank)


def backward(x, dh, seg, chunk, variant, *, group=None, ops=None, dstate_final=None):
    """This rank's gradients of sum(dh * h) over the whole sequence (plus <dstate_final,
    the sequence's final state> when given), for a ``forward(..., keep_saved=True)``.

    Returns the dict of binding.backward (dq, dk, dv, digate_pre, dfgate_pre) for this
    rank's tokens.  Collectives: one all-gather over ``group``.
    """
    import torch.distributed as dist
    ops = ops or DeviceOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    sizes = _sizes(x)
    dlocal = ops.local_dstate(x, dh, seg, chunk, variant)
    dlocals = [dlocal.new_empty(dlocal.shape) for _ in range(world)]
    dist.all_gather(dlocals, dlocal, group=group)
    dout = final_state_gradient(rank, dlocals, seg.states, seg.decays, sizes, variant, ops,
                                dstate_final)
    return ops.backward_from(x, dh, seg, chunk, variant, dout)
