"""World-size-2 gloo run of the multi-rank host logic (CPU only): ranks take
their share of the sublayers, all-gather the sensitivity triples and agree
on the bits."""
import os
import socket

import pytest
import torch.multiprocessing as mp


# one Llama-3-8B-shaped block's sublayers (q, k, v, o, gate, up, down), twice
SIZES = [4096 * 4096, 1024 * 4096, 1024 * 4096, 4096 * 4096, 14336 * 4096, 14336 * 4096,
         4096 * 14336] * 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta

    from post_quantization_kronq_b200.dist import allocate_from_sensitivities, gather_sensitivities, shard_units

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    n_units = 14
    sizes = SIZES
    mine = shard_units(n_units, rank, world)
    # stand-in (tr H_X, tr H_G, s) triples, as kronq_sensitivity returns them
    local = {u: (float(u + 1), float(2 * u + 3), float((u + 1) * (2 * u + 3))) for u in mine}
    traces = gather_sensitivities(local, n_units)
    bits = allocate_from_sensitivities(traces, sizes)
    out[rank] = (mine, traces, bits)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_trace_exchange():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    m0, t0, b0 = out[0]
    m1, t1, b1 = out[1]
    assert sorted(m0 + m1) == list(range(14)) and not set(m0) & set(m1)
    assert t0 == t1 == [(float(u + 1), float(2 * u + 3), float((u + 1) * (2 * u + 3))) for u in range(14)]
    assert b0 == b1
    from oracle.alloc import allocate_budget
    assert b0 == list(allocate_budget([t[2] for t in t0], SIZES, 2.5, 2, 4))
    assert all(2 <= b <= 4 for b in b0)
