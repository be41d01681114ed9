"""Sequence-parallel prefill across processes, one per GPU.

Rank r of a group of N holds the r-th of N consecutive runs of every sequence
(the slices may differ in length).  A run of tokens acts on its incoming state
as an affine map, S_out = S_in Lam + H ("Linear Attention, Visualized": "One
chunk as an affine recurrence", "Update the state"), so the prefill needs one
exchange:

1. ``segment_maps`` on the local run (gdn_segment_maps: H and Lam);
2. one all-gather of the maps, stacked in rank order (B*H*(dv*dk + dk*dk) fp32
   values per rank; H alone for the additive write, whose Lam is I);
3. ``compose_segments`` over all N maps (gdn_compose_segments, redundantly on
   every rank, a few microseconds): the state entering every run and the
   final state;
4. ``chunk_fwd`` on the local run from its incoming state: the outputs.

The arithmetic of steps 1, 3 and 4 runs in the library's kernels; this module
moves tensors between ranks with ``torch.distributed`` and nothing else.
"""
from __future__ import annotations

from . import chunk_fwd, compose_segments, segment_maps


def gather_segment_maps(H, Lam=None, group=None):
    """All-gather of every rank's maps in one collective.

    H [B,H,dv,dk] and Lam [B,H,dk,dk] (or None) of this rank's run; returns
    (H_all [N,B,H,dv,dk], Lam_all [N,B,H,dk,dk] or None), entry r from rank r
    of ``group``.
    """
    import torch
    import torch.distributed as dist

    n = dist.get_world_size(group)
    parts = [H.reshape(-1)] + ([] if Lam is None else [Lam.reshape(-1)])
    mine = torch.cat(parts) if len(parts) > 1 else parts[0].contiguous()
    flat = mine.new_empty((n, mine.numel()))
    dist.all_gather(list(flat.unbind(0)), mine, group=group)
    nH = H.numel()
    H_all = flat[:, :nH].reshape((n,) + tuple(H.shape))
    Lam_all = None if Lam is None else flat[:, nH:].reshape((n,) + tuple(Lam.shape))
    return H_all.contiguous(), (None if Lam_all is None else Lam_all.contiguous())


def chunk_fwd_seqpar(q, k, v, g=None, beta=None, S0=None, *, update, gate, group=None, out_dtype=None,
                     algo="auto", prologue=0):
    """Prefill of sequences split along time over the ranks of ``group``.

    q, k, v, g, beta: this rank's run of every sequence, shaped as for
    ``chunk_fwd`` with T = the run's length.  S0 [B,H,dv,dk] or None: the state
    before the first run (the same tensor on every rank).  Returns (o of this
    rank's run, S_T after the last run, identical on every rank).
    """
    import torch.distributed as dist

    r = dist.get_rank(group)
    H, Lam = segment_maps(q, k, v, g, beta, update=update, gate=gate, algo=algo, prologue=prologue)
    H_all, Lam_all = gather_segment_maps(H, None if update == "additive" else Lam, group)
    S_in, S_T = compose_segments(H_all, Lam_all, S0)
    o, _ = chunk_fwd(q, k, v, g, beta, S_in[r], update=update, gate=gate, out_dtype=out_dtype, return_state=False,
                     algo=algo, prologue=prologue)
    return o, S_T
