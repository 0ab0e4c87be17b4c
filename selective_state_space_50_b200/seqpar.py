"""Sequence-sharded forward scan: one segment of the sequence per rank.

The recurrence is sequential in time, but a segment's effect on the state is
summarised by two numbers per (channel, state): the state it ends in when run
from zero, e, and its decay product exp(A Σ_t Δ_t).  The summaries compose with
the associative operator of the two-level scan (booiljung.github.io, "3.2
선택적 스캔(Selective Scan) 알고리즘", §2.2), so the ranks need one exchange:

  pass 1   every rank runs its segment from a zero state           (local)
  exchange all-gather of (Σ Δ, e), [batch, dim] + [batch, dim, N] per rank
  combine  exclusive scan of the summaries -> state entering each segment
  pass 2   ranks 1..S-1 rerun their segment from that state          (local)

Rank 0's pass 1 is already final.  The exchange is one all-gather of
batch*dim*(N+1) floats per rank (NCCL over NVLink in production); each rank
then combines all summaries itself, so there is no second collective.  Ranks
other than 0 do the scan twice; the critical path is two segment scans.

`forward_rank` is the per-rank protocol; its compute and exchange steps are
passed in, so the same protocol runs on the library's CUDA kernels with NCCL,
or, in the tests, on other implementations with gloo.  `forward_segments`
runs all segments of one sequence on one device, in the same order of steps.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple


def forward_rank(rank: int, run_segment: Callable, gather: Callable, combine: Callable):
    """One rank's part of the sequence-sharded forward.

    run_segment(h0) -> (out, last_state, delta_sum): this rank's segment from
        state h0 (None = zeros).
    gather(x) -> x of every rank stacked in rank order (a collective: every
        rank calls it the same number of times, in the same order).
    combine(delta_sums, h_ends) -> h_in, the state entering each segment.

    Returns (out, last_state) of this rank's segment with the true carry-in."""
    out, last, dsum = run_segment(None)
    dsums = gather(dsum)
    ends = gather(last)
    h_in = combine(dsums, ends)
    if rank > 0:
        out, last, _ = run_segment(h_in[rank])
    return out, last


def forward_segments(run_segment: Callable[[int, Optional[object]], Tuple], nseg: int,
                     stack: Callable[[Sequence], object], combine: Callable):
    """All segments of one sequence on one device: pass 1 over every segment,
    one combine, pass 2 over segments 1..nseg-1.  run_segment(s, h0) runs
    segment s.  Returns ([out_s], final state of the last segment)."""
    outs: List = []
    lasts, dsums = [], []
    for s in range(nseg):
        o, l, d = run_segment(s, None)
        outs.append(o)
        lasts.append(l)
        dsums.append(d)
    h_in = combine(stack(dsums), stack(lasts))
    last = lasts[0]
    for s in range(1, nseg):
        outs[s], last, _ = run_segment(s, h_in[s])
    return outs, last


# ---------------------------------------------------------------- CUDA + NCCL

def all_gather_stacked(x, group=None):
    """x of every rank of `group`, stacked in rank order: [world, *x.shape].
    One all_gather_into_tensor into a buffer of the concatenated form (rank
    blocks along the first dimension), which every backend accepts."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    x = x.contiguous()
    flat = x.reshape(-1)
    buf = torch.empty(world * flat.numel(), device=x.device, dtype=x.dtype)
    dist.all_gather_into_tensor(buf, flat, group=group)
    return buf.view((world,) + tuple(x.shape))


def cuda_forward_rank(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                      delta_softplus: bool = True, group=None, stream=None):
    """Sequence-sharded forward on this rank's GPU: u, delta, z [batch, dim,
    L_r] and B, C [batch, dstate, L_r] are this rank's segment (segments in
    rank order make up the sequence).  The exchange is an all-gather on the
    torch.distributed group (NCCL for CUDA tensors).  Returns (out,
    last_state) of this segment."""
    import torch.distributed as dist

    from . import ssm_scan
    rank = dist.get_rank(group)

    def run_segment(h0):
        return ssm_scan.selective_scan_fwd_segment(u, delta, A, B, C, D, z, delta_bias,
                                                   delta_softplus, h0=h0, stream=stream)

    def gather(x):
        return all_gather_stacked(x, group)

    def combine(dsums, ends):
        return ssm_scan.combine_carries(A, dsums, ends, stream=stream)

    return forward_rank(rank, run_segment, gather, combine)


def cuda_forward_segments(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                          delta_softplus: bool = True, nseg: int = 2, stream=None):
    """The whole sequence on one GPU, cut into nseg equal segments (L % nseg
    == 0) and run with the sharded protocol.  Returns (out, last_state)."""
    import torch

    from . import ssm_scan
    L = u.shape[-1]
    if L % nseg:
        raise ValueError("seqlen must be a multiple of nseg")
    Ls = L // nseg
    out = torch.empty_like(u)

    def part(t, s):
        return None if t is None else t[..., s * Ls:(s + 1) * Ls].contiguous()

    pieces = [(part(u, s), part(delta, s), part(B, s), part(C, s), part(z, s)) for s in range(nseg)]

    def run_segment(s, h0):
        us, ds, Bs, Cs, zs = pieces[s]
        return ssm_scan.selective_scan_fwd_segment(us, ds, A, Bs, Cs, D, zs, delta_bias,
                                                   delta_softplus, h0=h0, stream=stream)

    outs, last = forward_segments(run_segment, nseg, torch.stack,
                                  lambda ds, es: ssm_scan.combine_carries(A, ds, es, stream=stream))
    for s in range(nseg):
        out[..., s * Ls:(s + 1) * Ls] = outs[s]
    return out, last
