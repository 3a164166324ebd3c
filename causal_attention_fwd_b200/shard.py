"""Head-sharded multi-GPU attention: one problem split over the ranks.

Every (batch b, kv head) unit, with the G = Hq / Hkv query heads that read it,
is independent in the forward and in the backward (dK, dV of a kv head only
sum over its own query heads).  So the units of one problem are dealt round
robin over the ranks (one process per GPU, as the Axis page's data-parallel
paragraph runs one), each rank runs its units as one batch through the same
kernels, and no data crosses between ranks on the path.  Only assembling the
full outputs (for checking, or for a caller that wants them on every rank)
takes a collective, an all-gather.

A rank's units are packed as a batch of independent problems: query-side
tensors [n, S, G, D] and kv-side tensors [n, S, 1, D] (B' = n units, Hq' = G,
Hkv' = 1).  In a tensor-parallel model the QKV projection already leaves each
rank its own heads, so the packing copy is only needed when the full tensors
start on every rank, as in the tests and the benchmark.
"""
from __future__ import annotations


def rank_units(B: int, Hkv: int, world: int, rank: int) -> list[tuple[int, int]]:
    """The (b, kv) units of `rank`: unit u = b * Hkv + kv goes to rank u % world."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of size {world}")
    return [(u // Hkv, u % Hkv) for u in range(rank, B * Hkv, world)]


def pack(x, units, heads_per_unit: int):
    """Gather the heads of `units` from x [B, S, H, D] into a contiguous
    [len(units), S, heads_per_unit, D]: query-side tensors take heads
    kv*G .. kv*G + G - 1 (heads_per_unit = G), kv-side tensors head kv (1)."""
    import torch

    if not units:
        return x.new_empty((0, x.shape[1], heads_per_unit, x.shape[3]))
    parts = [x[b, :, kv * heads_per_unit:(kv + 1) * heads_per_unit] for b, kv in units]
    return torch.stack(parts, 0).contiguous()


def unpack(y, units, out, heads_per_unit: int):
    """Scatter a packed [n, S, heads_per_unit, D] back into the full tensor
    `out` [B, S, H, D] (the inverse of pack)."""
    for n, (b, kv) in enumerate(units):
        out[b, :, kv * heads_per_unit:(kv + 1) * heads_per_unit] = y[n]
    return out


def unpack_lse(y, units, out, G: int):
    """LSE rows: packed [n, G, S] into the full [B, Hq, S]."""
    for n, (b, kv) in enumerate(units):
        out[b, kv * G:(kv + 1) * G] = y[n]
    return out


def all_gather_units(local, B: int, Hkv: int, world: int, group=None):
    """Every rank's packed tensor -> the list of all ranks' packed tensors (in
    rank order), through one all-gather of zero-padded tensors of the largest
    rank's size.  Outside the attention path: for assembling outputs."""
    import torch
    import torch.distributed as dist

    n_max = len(rank_units(B, Hkv, world, 0))  # rank 0 holds the most units
    pad = local.new_zeros((n_max,) + tuple(local.shape[1:]))
    pad[: local.shape[0]] = local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    return [bufs[r][: len(rank_units(B, Hkv, world, r))] for r in range(world)]


def sharded_forward(q, k, v, world: int, rank: int, causal: bool = True, scale: float | None = None,
                    attention_forward=None):
    """This rank's share of the forward: (units, O_local [n,S,G,D], LSE_local
    [n,G,S]).  attention_forward defaults to the CUDA library's helper."""
    if attention_forward is None:
        from .binding import attention_forward
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    units = rank_units(B, Hkv, world, rank)
    if not units:
        import torch

        return units, q.new_empty((0, S, G, D)), q.new_empty((0, G, S), dtype=torch.float32)
    o, lse = attention_forward(pack(q, units, G), pack(k, units, 1), pack(v, units, 1), causal=causal,
                               scale=scale)
    return units, o, lse


def sharded_backward(q, k, v, o_local, lse_local, dout, world: int, rank: int, causal: bool = True,
                     scale: float | None = None, attention_backward=None):
    """This rank's share of the backward: (units, dQ_local, dK_local, dV_local)
    for the units of rank_units(); o_local, lse_local come from sharded_forward."""
    if attention_backward is None:
        from .binding import attention_backward
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    units = rank_units(B, Hkv, world, rank)
    if not units:
        e = q.new_empty((0, S, G, D))
        return units, e, q.new_empty((0, S, 1, D)), q.new_empty((0, S, 1, D))
    dq, dk, dv = attention_backward(pack(q, units, G), pack(k, units, 1), pack(v, units, 1), o_local, lse_local,
                                    pack(dout, units, G), causal=causal, scale=scale)
    return units, dq, dk, dv
