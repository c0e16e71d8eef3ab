"""Sequence-parallel chunkwise forward: one segment of every head's sequence per rank.

"Tiled Flash Linear Attention" (TFLA summary page, Problem and Approach): the
chunkwise form carries everything a later chunk needs in the state at a chunk
boundary, so a boundary may as well lie between two GPUs.  Rank r holds tokens
[r T_loc, (r + 1) T_loc) of every head and computes, exactly:

1. its segment's final state from the zero state (state-only pass, no output
   kernel) and the segment's total log forget gate G_r;
2. an all-gather of the (state, G) pairs over the process group: the one
   exchange step, B * NH * (d_qk * d_hv (+ d_qk + 1)) fp32 per rank;
3. the state entering its segment, chaining the earlier segments' states:
   S_in(0) = zero, S_in(r + 1) = chain(S_in(r), S_r, G_r);
4. its segment's outputs from that state (mlstm_fwd_state).

Every device step runs in the library's kernels; this module only orders the
calls and the exchange.  The backward through segment boundaries (the
gradient with respect to a segment's final state) is not provided.
"""

from dataclasses import dataclass


@dataclass
class Segment:
    """One rank's share: h [B, NH, T_loc, d_hv], the state its segment started from
    (None on rank 0), and its saved buffer (for mlstm_bwd_state with that state)."""
    h: object
    state_in: object
    saved: object


class DeviceOps:
    """The device operations the protocol needs, on the CUDA library."""

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


def incoming_state(rank, states, decays, sizes, variant, ops):
    """The state entering segment ``rank`` (None: the zero state, rank 0), from every
    segment's final state from the zero state and its total log forget gate."""
    state_in = None
    for r in range(rank):
        state_in = states[0] if r == 0 else ops.chain(state_in, states[r], decays[r], sizes, variant)
    return state_in


def forward(x, chunk, variant, *, group=None, ops=None, keep_saved=False):
    """This rank's segment of a sequence-parallel forward.

    x: dict of this rank's q, k [B, NH, T_loc, d_qk], v [B, NH, T_loc, d_hv], igate,
    fgate [B, NH, T_loc] (device tensors); every rank passes the same B, NH, d and
    chunk, and the segments follow rank order.  Collectives: two all-gathers over
    ``group`` (torch.distributed), taken by every rank in the same order.
    """
    import torch.distributed as dist
    ops = ops or DeviceOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, NH, _, d_qk = x["q"].shape
    sizes = (B, NH, d_qk, x["v"].shape[-1])
    state, decay = ops.local_state(x, chunk, variant)
    states = [state.new_empty(state.shape) for _ in range(world)]
    decays = [decay.new_empty(decay.shape) for _ in range(world)]
    dist.all_gather(states, state, group=group)
    dist.all_gather(decays, decay, group=group)
    state_in = incoming_state(rank, states, decays, sizes, variant, ops)
    h, saved = ops.forward_from(x, chunk, variant, state_in, keep_saved)
    return Segment(h=h, state_in=state_in, saved=saved)
