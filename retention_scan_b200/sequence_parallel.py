"""One sequence split along T over the ranks of a process group.

Rank r holds span r of every (b, h) sequence: the tokens that follow rank
r - 1's.  The spans combine with the associative operator of RetNet issue 21
("Proposed improvement/collaboration: removing the O(T^2) training cost", the
paragraph on the associative EMA operator): a span started from zero leaves a
state S_j and multiplies the state entering it by exp(L_j), L_j its total log
decay, so the state entering span r is the left fold over the spans before
it.  Each rank therefore

  1. computes its own span's state from zero and its total log decay
     (la_chunk_state_ws; the last rank skips this: no span follows it),
  2. exchanges those records with every rank in one all-gather (NCCL over
     NVLink between GPUs; B*H*(Dk*Dv + Dk + 1) floats per rank, 2.1 MB for
     32 heads of 128 x 128),
  3. folds the records of the spans before its own onto the sequence's
     initial state (la_state_combine),
  4. runs its span's forward from that state (la_chunk_forward_ws).

The exchange is the only collective; steps 1, 3 and 4 run in the library's
kernels.  On the last rank the returned final state is the whole sequence's.
"""
import torch
import torch.distributed as dist

from . import DECAY_NONE, chunk_forward, chunk_state, state_combine

__all__ = ["span_forward", "record_layout"]


def _pad4(n):
    return (n + 3) // 4 * 4


def record_layout(B, H, Dk, Dv):
    """Offsets (in floats) of a rank's exchanged record: [state | key sum |
    log decay], each part padded to 16 bytes; returns (s, z, l, size)."""
    BH = B * H
    s = 0
    z = s + _pad4(BH * Dk * Dv)
    lg = z + _pad4(BH * Dk)
    return s, z, lg, lg + _pad4(BH)


def _views(buf, B, H, Dk, Dv):
    """[n, size] records -> state [n,B,H,Dk,Dv], z [n,B,H,Dk], log [n,B,H] views."""
    s, z, lg, _ = record_layout(B, H, Dk, Dv)
    n, BH = buf.shape[0], B * H
    return (buf[:, s:s + BH * Dk * Dv].view(n, B, H, Dk, Dv), buf[:, z:z + BH * Dk].view(n, B, H, Dk),
            buf[:, lg:lg + BH].view(n, B, H))


class LibraryOps:
    """The library's kernels for the three compute steps."""

    @staticmethod
    def state(k, v, decay_kind, log_g, normalize, state_out, z_out, log_out):
        chunk_state(k, v, decay_kind, log_g, normalize, state_out=state_out, z_out=z_out, log_g_total=log_out)

    @staticmethod
    def combine(seg_state, seg_log_g, seg_z, init_state, init_z):
        S, z, _ = state_combine(seg_state, seg_log_g, seg_z, init_state, init_z)
        return S, z

    @staticmethod
    def forward(q, k, v, decay_kind, log_g, normalize, init_state, init_z, out):
        return chunk_forward(q, k, v, decay_kind, log_g, normalize, init_state=init_state, init_z=init_z, out=out)


def span_forward_with(rank, world, all_gather, ops, q, k, v, decay_kind=DECAY_NONE, log_g=None, normalize=False,
                      init_state=None, init_z=None, out=None):
    """The host logic of span_forward with the collective and the compute
    steps passed in (all_gather(list_of_outputs, input) and an object with
    state / combine / forward as LibraryOps)."""
    B, H, T, Dk = k.shape
    Dv = v.shape[-1]
    if normalize and init_state is not None and init_z is None:
        raise ValueError("normalize with init_state needs init_z")
    size = record_layout(B, H, Dk, Dv)[3]
    mine = torch.zeros((1, size), dtype=torch.float32, device=k.device)
    if rank < world - 1:
        S, z, lg = _views(mine, B, H, Dk, Dv)
        ops.state(k, v, decay_kind, log_g, normalize, S[0], z[0] if normalize else None, lg[0])
    gathered = torch.empty((world, size), dtype=torch.float32, device=k.device)
    all_gather(list(gathered.unbind(0)), mine[0])
    state_in, z_in = init_state, init_z if normalize else None
    if rank > 0:
        S, z, lg = _views(gathered[:rank], B, H, Dk, Dv)
        state_in, z_in = ops.combine(S, lg, z if normalize else None, init_state, init_z if normalize else None)
    return ops.forward(q, k, v, decay_kind, log_g, normalize, state_in, z_in, out)


def span_forward(q, k, v, decay_kind=DECAY_NONE, log_g=None, normalize=False, init_state=None, init_z=None,
                 out=None, group=None):
    """This rank's span of a sequence split along T over `group` (the default
    process group if None), run as described in the module docstring.

    q, k, v, log_g (per step: this span's [B,H,T_r]; per head: [H]), out: as
    chunk_forward for this rank's span; spans may differ in length.
    init_state / init_z: the whole sequence's initial state, the same on
    every rank (or None).  Returns (out, final_state, final_z) of this span;
    on the last rank, the sequence's final state."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)

    def gather(outs, x):
        dist.all_gather(outs, x, group=group)

    return span_forward_with(rank, world, gather, LibraryOps, q, k, v, decay_kind, log_g, normalize, init_state,
                             init_z, out)
