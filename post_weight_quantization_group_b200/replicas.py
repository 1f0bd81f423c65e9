"""Host-side logic of running the decode products as independent replicas,
one process per GPU (``torch.distributed``): the product shards into
independent problems, so ranks exchange nothing in the timed region and meet
only to agree on the time.

* ``replica_layer(layer, rank)``: the distinct layer index (and so the weight
  seeds) of a rank's replica, so no two ranks stream the same weights;
* ``max_over_ranks(seconds, dist, device)``: the job time, the slowest rank;
* ``aggregate_throughput(bytes_per_rank, seconds_max, world)``: whole-job
  bytes per second (every rank moves the same bytes).
"""
from __future__ import annotations

REPLICA_LAYER_STRIDE = 1000


def replica_layer(layer: int, rank: int) -> int:
    """Layer index whose seeds rank ``rank`` uses for its layer ``layer``."""
    if layer < 0 or layer >= REPLICA_LAYER_STRIDE or rank < 0:
        raise ValueError("layer must be in [0, 1000) and rank >= 0")
    return layer + REPLICA_LAYER_STRIDE * rank


def max_over_ranks(seconds: float, dist=None, device=None) -> float:
    """Maximum of ``seconds`` over all ranks of the default process group
    (the value itself without a group).  Every rank must call it."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(seconds)
    import torch
    t = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(bytes_per_rank: int, seconds_max: float, world: int) -> float:
    """Whole-job throughput in bytes per second: all ranks' bytes over the
    slowest rank's time."""
    if seconds_max <= 0 or world < 1:
        raise ValueError("time must be positive and world >= 1")
    return world * bytes_per_rank / seconds_max
