"""The multi-rank ring schedule (long_sequence_context_b200/ring.py) on CPU:
N ranks' generators driven in one process (loopback) and as gloo processes
(torch.distributed point-to-point), each block computed by the fp64 oracle
backend.  Every rank's O, LSE, dQ, dK, dV must equal the oracle's attention of
the whole sequence on that rank's chunks (1e-10: the same fp64 arithmetic,
split into blocks and merged)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from long_sequence_context_b200 import ring
from long_sequence_context_b200.inputs import make_qkv
from oracle import oracle as orc


def _inputs(world, causal, S_per_chunk=8, B=1, H=2, D=8, seed=21):
    n_chunks = 2 * world if causal else world
    S = n_chunks * S_per_chunk
    q, k, v, do = (t.double() for t in make_qkv(B, H, S, D, torch.float32, seed=seed))
    return q, k, v, do


def _reference(q, k, v, do, causal, scale):
    o, lse = orc.attn_fwd(q.numpy(), k.numpy(), v.numpy(), causal, scale)
    dq, dk, dv = orc.attn_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, scale)
    return {n: torch.from_numpy(a) for n, a in
            (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}


def _rank_work(rank, world, causal, q, k, v, do, scale, runner):
    from tests.ring_oracle_backend import OracleBlocks
    loc = lambda x: ring.local_chunks(x, rank, world, causal)
    be = OracleBlocks(scale)
    ql, kl, vl, dol = loc(q), loc(k), loc(v), loc(do)
    fwd = runner(ring.fwd_schedule(rank, world, ql, kl, vl, causal, be))
    o, lse = [a for a, _ in fwd], [b for _, b in fwd]
    dq, dk, dv = runner(ring.bwd_schedule(rank, world, ql, kl, vl, o, lse, dol, causal, be))
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


def _check(rank, world, causal, got, ref):
    for name, chunks in got.items():
        want = ring.local_chunks(ref[name], rank, world, causal)
        for g, w in zip(chunks, want):
            np.testing.assert_allclose(g.numpy(), w.numpy(), rtol=0, atol=1e-10,
                                       err_msg=f"rank {rank} {name}")


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_loopback_ring_equals_whole_sequence_oracle(world, causal):
    q, k, v, do = _inputs(world, causal)
    scale = 0.35
    ref = _reference(q, k, v, do, causal, scale)
    from tests.ring_oracle_backend import OracleBlocks
    be = OracleBlocks(scale)
    loc = lambda x, r: ring.local_chunks(x, r, world, causal)
    fwd = ring.run_loopback([ring.fwd_schedule(r, world, loc(q, r), loc(k, r), loc(v, r), causal, be)
                             for r in range(world)])
    bwd = ring.run_loopback([ring.bwd_schedule(r, world, loc(q, r), loc(k, r), loc(v, r),
                                               [a for a, _ in fwd[r]], [b for _, b in fwd[r]],
                                               loc(do, r), causal, be) for r in range(world)])
    for r in range(world):
        got = {"o": [a for a, _ in fwd[r]], "lse": [b for _, b in fwd[r]],
               "dq": bwd[r][0], "dk": bwd[r][1], "dv": bwd[r][2]}
        _check(r, world, causal, got, ref)


def test_zigzag_ownership_and_block_kinds():
    # N = 4: ranks own {0,7}, {1,6}, {2,5}, {3,4} ("Configuring
    # RingAttention+FlashAttention for CP", section 5 item 1)
    assert [ring.rank_chunks(r, 4, True) for r in range(4)] == [[0, 7], [1, 6], [2, 5], [3, 4]]
    assert ring.block_kind(3, 1, True) == ring.FULL
    assert ring.block_kind(2, 2, True) == ring.DIAG
    assert ring.block_kind(1, 3, True) == ring.SKIP
    assert ring.block_kind(1, 3, False) == ring.FULL


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _dist_main(rank, world, port, causal, out_q):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, do = _inputs(world, causal)
        scale = 0.35
        got = _rank_work(rank, world, causal, q, k, v, do, scale, ring.run_dist)
        _check(rank, world, causal, got, _reference(q, k, v, do, causal, scale))
        out_q.put((rank, "ok"))
    except Exception as e:  # reported to the parent
        out_q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (2, False)])
def test_gloo_ranks_ring_equals_whole_sequence_oracle(world, causal):
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dist_main, args=(r, world, port, causal, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        assert p.exitcode == 0
    res = sorted(out_q.get(timeout=5) for _ in range(world))
    assert res == [(r, "ok") for r in range(world)]
