"""The all-gather-K/V context-parallel variant
(long_sequence_context_b200/allgather_cp.py): gloo ranks all-gather K/V,
attend their own zigzag Q chunks, reduce-scatter dK/dV; each block by the
fp64 oracle backend.  Every rank's O, LSE, dQ, dK, dV must equal the oracle's
attention of the whole sequence on its chunks (1e-10).  One more case runs the
library's blocks on the GPU as one rank (no process group)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from long_sequence_context_b200 import allgather_cp, ring
from long_sequence_context_b200.inputs import make_qkv
from oracle import oracle as orc


def _case(world, causal, seed=23):
    n_chunks = 2 * world if causal else world
    q, k, v, do = (t.double() for t in make_qkv(1, 2, n_chunks * 8, 8, torch.float32, seed=seed))
    scale = 0.4
    o, lse = orc.attn_fwd(q.numpy(), k.numpy(), v.numpy(), causal, scale)
    dq, dk, dv = orc.attn_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, scale)
    ref = {n: torch.from_numpy(a) for n, a in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    return q, k, v, do, scale, ref


def _run_and_check(rank, world, causal):
    from tests.ring_oracle_backend import OracleBlocks
    q, k, v, do, scale, ref = _case(world, causal)
    loc = lambda x: ring.local_chunks(x, rank, world, causal)
    be = OracleBlocks(scale)
    o, lse = allgather_cp.allgather_fwd(loc(q), loc(k), loc(v), causal, scale, backend=be)
    dq, dk, dv = allgather_cp.allgather_bwd(loc(q), loc(k), loc(v), o, lse, loc(do), causal, scale,
                                            backend=be)
    for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        for g, w in zip(got, loc(ref[name])):
            np.testing.assert_allclose(g.numpy(), w.numpy(), rtol=0, atol=1e-10, err_msg=f"{rank} {name}")


@pytest.mark.parametrize("causal", [True, False])
def test_one_rank_without_process_group(causal):
    _run_and_check(0, 1, causal)


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
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        _run_and_check(rank, world, causal)
        out_q.put((rank, "ok"))
    except Exception as e:
        out_q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (2, False)])
def test_gloo_ranks_equal_whole_sequence_oracle(world, causal):
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
    assert sorted(out_q.get(timeout=5) for _ in range(world)) == [(r, "ok") for r in range(world)]


@pytest.mark.gpu
def test_library_blocks_one_rank_on_gpu():
    from long_sequence_context_b200 import cpattn as cp
    from tests.util import assert_close, assert_lse_close, np64
    B, H, S, D = 1, 2, 1024, 128
    q, k, v, do = make_qkv(B, H, S, D, torch.bfloat16, seed=41)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    loc = lambda x: ring.local_chunks(x, 0, 1, True)
    o, lse = allgather_cp.allgather_fwd(loc(qd), loc(kd), loc(vd), True)
    dq, dk, dv = allgather_cp.allgather_bwd(loc(qd), loc(kd), loc(vd), o, lse, loc(dod), True)
    cp.check_device_status()
    f = np64
    ro, rl = orc.attn_fwd(f(q), f(k), f(v), True, D ** -0.5)
    rg = orc.attn_bwd(f(q), f(k), f(v), f(do), True, D ** -0.5)
    for g, w in zip(o, loc(torch.from_numpy(ro))):
        assert_close(g, w.numpy(), dtype=torch.bfloat16)
    # block terms are summed in fp32 (cpattn_bwd_accumulate) and rounded once:
    # the bf16 bar, unwidened
    for got, want in zip((dq, dk, dv), rg):
        for g, w in zip(got, loc(torch.from_numpy(want))):
            assert_close(g, w.numpy(), dtype=torch.bfloat16)
    for g, w in zip(lse, loc(torch.from_numpy(rl))):
        assert_lse_close(g, w.numpy())
