"""Context-parallel attention by all-gathering K/V: each rank collects every
rank's K/V chunks, attends its own zigzag Q chunks over them in one pass, and
in the backward reduce-scatters the dK/dV sums back to the chunks' owners.

"Megatron-LM source analysis: Context Parallel" (mieleap.com), section 2: the
forward all-gathers K and V over the context-parallel group before the
attention of the local queries, the backward mirrors it with reduce_scatter.
Chunk ownership and block kinds are those of the ring (ring.py: zigzag 2N
chunks when causal; FULL / DIAG / SKIP per (q chunk, kv chunk)); the block
arithmetic is the library's kernels through ring.CudaBlocks.  Without an
initialised process group the calls run as one rank.
"""
import torch

from . import ring


def _group_info(group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group), True
    return 0, 1, False


def _gather_chunks(chunks, rank, world, causal, use_dist, group):
    """{chunk id: tensor} of every rank's chunks (this rank's own tensors included)."""
    out = {}
    for i, t in enumerate(chunks):
        if use_dist and world > 1:
            import torch.distributed as dist
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t.contiguous(), group=group)
        else:
            parts = [t]
        for r, p in enumerate(parts):
            out[ring.rank_chunks(r, world, causal)[i]] = p
    return out


def allgather_fwd_blocks(rank, world, q, k_all, v_all, causal, be):
    """Forward of this rank's Q chunks over every chunk's K/V (by chunk id)."""
    n_chunks = 2 * world if causal else world
    out = []
    for ai, a in enumerate(ring.rank_chunks(rank, world, causal)):
        o_acc, lse_acc = be.new_acc(q[ai])
        for b in range(n_chunks):
            kind = ring.block_kind(a, b, causal)
            if kind == ring.SKIP:
                continue
            o_p, l_p = be.fwd(q[ai], k_all[b], v_all[b], kind == ring.DIAG)
            be.merge(o_acc, lse_acc, o_p, l_p)
        out.append((be.finalize(o_acc, q[ai].dtype), lse_acc))
    return out


def allgather_bwd_blocks(rank, world, q, k_all, v_all, o, lse, do, causal, be):
    """Block gradients: dQ of this rank's chunks and this rank's dK/dV terms
    for every chunk id (fp32 sums, to be reduce-scattered)."""
    n_chunks = 2 * world if causal else world
    dq = [be.zeros_f32(x) for x in q]
    dk = {b: be.zeros_f32(k_all[b]) for b in range(n_chunks)}
    dv = {b: be.zeros_f32(v_all[b]) for b in range(n_chunks)}
    for ai, a in enumerate(ring.rank_chunks(rank, world, causal)):
        for b in range(n_chunks):
            kind = ring.block_kind(a, b, causal)
            if kind == ring.SKIP:
                continue
            be.bwd_into(q[ai], k_all[b], v_all[b], o[ai], lse[ai], do[ai], kind == ring.DIAG,
                        dq[ai], dk[b], dv[b])
    return dq, dk, dv


def _reduce_scatter_chunks(sums, rank, world, causal, m, use_dist, group):
    """This rank's chunk sums: sum over ranks of every rank's term for them."""
    own = ring.rank_chunks(rank, world, causal)
    if not (use_dist and world > 1):
        return [sums[c] for c in own]
    import torch.distributed as dist
    out = []
    for i in range(m):
        res = torch.empty_like(sums[own[i]])
        dist.reduce_scatter(res, [sums[ring.rank_chunks(r, world, causal)[i]] for r in range(world)],
                            group=group)
        out.append(res)
    return out


def allgather_fwd(q, k, v, causal=True, scale=None, group=None, backend=None):
    """Forward of this rank's chunks (local_chunks order): lists (o, lse)."""
    rank, world, use_dist = _group_info(group)
    scale = float(scale if scale is not None else q[0].shape[-1] ** -0.5)
    be = backend if backend is not None else ring.CudaBlocks(scale)
    k_all = _gather_chunks(k, rank, world, causal, use_dist, group)
    v_all = _gather_chunks(v, rank, world, causal, use_dist, group)
    out = allgather_fwd_blocks(rank, world, q, k_all, v_all, causal, be)
    return [a for a, _ in out], [b for _, b in out]


def allgather_bwd(q, k, v, o, lse, do, causal=True, scale=None, group=None, backend=None):
    """Backward of this rank's chunks: lists (dq, dk, dv) in the inputs' dtype."""
    rank, world, use_dist = _group_info(group)
    scale = float(scale if scale is not None else q[0].shape[-1] ** -0.5)
    be = backend if backend is not None else ring.CudaBlocks(scale)
    k_all = _gather_chunks(k, rank, world, causal, use_dist, group)
    v_all = _gather_chunks(v, rank, world, causal, use_dist, group)
    dq, dk_sum, dv_sum = allgather_bwd_blocks(rank, world, q, k_all, v_all, o, lse, do, causal, be)
    m = len(q)
    dk = _reduce_scatter_chunks(dk_sum, rank, world, causal, m, use_dist, group)
    dv = _reduce_scatter_chunks(dv_sum, rank, world, causal, m, use_dist, group)
    return ([be.cast(x, q[i].dtype) for i, x in enumerate(dq)],
            [be.cast(x, k[i].dtype) for i, x in enumerate(dk)],
            [be.cast(x, v[i].dtype) for i, x in enumerate(dv)])
