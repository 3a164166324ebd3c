"""Head-sharded multi-GPU path (causal_attention_fwd_b200.shard), host logic
on CPU with gloo ranks.

The kernels cannot run here, so each rank computes its units with the fp64
oracle standing in for the CUDA helpers (the oracle is test infrastructure; the
sharding code only sees a callable with the helpers' signature).  The oracle
computes every (b, kv) unit with the same loops whether the unit sits in the
full problem or in a rank's packed batch, so the reassembled outputs must equal
the unsharded oracle results exactly: this checks the partition (every unit on
exactly one rank), the packing of query and kv heads, the LSE layout and the
all-gather reassembly, for an even and an uneven split.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, shape, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from causal_attention_fwd_b200 import shard
        from causal_attention_fwd_b200.synthetic import make_inputs

        B, Hq, Hkv, S, D = shape
        G = Hq // Hkv
        sc = D ** -0.5
        qb, kb, vb, dob = make_inputs(B, Hq, Hkv, S, D, seed=515)
        qd, kd, vd, dod = (t.double() for t in (qb, kb, vb, dob))

        def fwd(q_, k_, v_, causal, scale):
            o, l = oracle.attn_fwd(q_, k_, v_, scale, causal)
            return torch.from_numpy(o), torch.from_numpy(l)

        def bwd(q_, k_, v_, o_, l_, do_, causal, scale):
            dq, dk, dv, _ = oracle.attn_bwd(q_, k_, v_, do_, scale, causal)
            return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)

        units, o_l, l_l = shard.sharded_forward(qd, kd, vd, world, rank, True, sc, attention_forward=fwd)
        _, dq_l, dk_l, dv_l = shard.sharded_backward(qd, kd, vd, o_l, l_l, dod, world, rank, True, sc,
                                                      attention_backward=bwd)
        full = {}
        for name, loc, heads in (("o", o_l, G), ("dq", dq_l, G), ("dk", dk_l, 1), ("dv", dv_l, 1)):
            parts = shard.all_gather_units(loc, B, Hkv, world)
            out = torch.zeros((B, S, Hq if heads == G else Hkv, D), dtype=torch.float64)
            for r, part in enumerate(parts):
                shard.unpack(part, shard.rank_units(B, Hkv, world, r), out, heads)
            full[name] = out
        parts = shard.all_gather_units(l_l, B, Hkv, world)
        lse = torch.zeros((B, Hq, S), dtype=torch.float64)
        for r, part in enumerate(parts):
            shard.unpack_lse(part, shard.rank_units(B, Hkv, world, r), lse, G)
        if rank == 0:
            ro, rl = oracle.attn_fwd(qd, kd, vd, sc, True)
            rdq, rdk, rdv, _ = oracle.attn_bwd(qd, kd, vd, dod, sc, True)
            same = all(torch.equal(full[n], torch.from_numpy(r))
                       for n, r in (("o", ro), ("dq", rdq), ("dk", rdk), ("dv", rdv)))
            same = same and torch.equal(lse, torch.from_numpy(rl))
            q.put(("result", same, [len(shard.rank_units(B, Hkv, world, r)) for r in range(world)]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, (2, 4, 2, 40, 16)), (3, (1, 10, 5, 33, 8))])
def test_sharded_equals_unsharded(world, shape):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    tag, same, counts = q.get(timeout=10)
    B, Hq, Hkv = shape[:3]
    assert same
    assert sum(counts) == B * Hkv and max(counts) - min(counts) <= 1


def test_rank_units_partition():
    sys.path.insert(0, ROOT)
    from causal_attention_fwd_b200 import shard

    for B, Hkv in ((1, 1), (2, 8), (4, 8), (3, 5)):
        for world in (1, 2, 3, 4, 8):
            got = [u for r in range(world) for u in shard.rank_units(B, Hkv, world, r)]
            assert sorted(got) == [(b, kv) for b in range(B) for kv in range(Hkv)]
    with pytest.raises(ValueError):
        shard.rank_units(1, 1, 2, 2)
