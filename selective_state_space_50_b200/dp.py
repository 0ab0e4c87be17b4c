"""Data-parallel gradient exchange for the scan's parameters.

When ranks hold different batch rows of the same layer, the scan's parameter
gradients dA [dim, dstate], dD [dim] and ddelta_bias [dim] are sums over batch
rows, so the rank-local sums must be added across ranks: one all-reduce (SUM)
of the three, packed into one flat buffer (about 110 KB at dim 1536,
dstate 16).  The activation gradients (du, ddelta, dz, dB, dC) belong to each
rank's own rows and need no exchange.
"""
from __future__ import annotations

from typing import Dict, Iterable

PARAM_GRADS = ("dA", "dD", "ddelta_bias")


def allreduce_param_grads(grads: Dict[str, object], group=None,
                          names: Iterable[str] = PARAM_GRADS) -> None:
    """Sums the named gradients (present and not None) over the ranks of
    `group`, in place.  Every rank must call it with the same names."""
    import torch
    import torch.distributed as dist
    ts = [grads[k] for k in names if grads.get(k) is not None]
    if not ts:
        return
    flat = torch.cat([t.reshape(-1) for t in ts])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for t in ts:
        n = t.numel()
        t.copy_(flat[off:off + n].view_as(t))
        off += n
