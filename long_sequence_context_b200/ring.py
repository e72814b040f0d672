"""Context-parallel ring attention across ranks: one process per GPU, each
rank holding its own chunks of the sequence.

"Configuring RingAttention+FlashAttention for CP" (devpress.csdn.net):
section 3 code -- at ring step t rank r attends to the K/V of rank
(r - t) mod N, receiving it from rank r - 1 while passing what it holds to
rank r + 1; section 5 item 1 -- with a causal mask the sequence is cut into
2N chunks and rank r owns chunks r and 2N - 1 - r (the zigzag); section 3
note 2 -- the mask is exact.  "Megatron-LM source analysis: Context
Parallel": section 5 -- the double-buffered loop, the next step's K/V in
flight while this step's attention runs; section 2 -- the backward mirrors
the exchange: dK and dV travel around the ring with their K and V (here too
the running sums of one step are in flight while the next step computes).

Per (q chunk, kv chunk) block the kind follows the same rule as the one-GPU
path: FULL (kv chunk before the q chunk, or no mask), DIAG (same chunk, masked
j <= i), SKIP (kv chunk after the q chunk).  Every block's arithmetic runs in
the library's kernels through the CudaBlocks backend; this module only
schedules the blocks and moves chunks between ranks:

    forward   per block  cpattn_fwd_step on the (q chunk, kv chunk) pair
              per row    cpattn_merge of the block partials, cpattn_finalize
    backward  per block  cpattn_bwd_accumulate on the pair with the rows' final
                         O and LSE (its exp(s - LSE) and dO.O are those of the
                         whole row), adding the block's terms in fp32 to the
                         running dQ, dK, dV sums (one rounding, at the end)

The schedule is written once, as a generator that yields its exchanges
("start" a send to rank + 1 / receive from rank - 1, "finish" it); run_dist
drives it over torch.distributed point-to-point operations (NCCL on GPUs),
run_loopback drives N ranks' generators in one process, delivering each
rank's message to the next in memory.
"""
import torch

SKIP, FULL, DIAG = 0, 1, 2


def rank_chunks(rank: int, world: int, causal: bool):
    """Chunk indices rank `rank` owns (zigzag when causal)."""
    return [rank, 2 * world - 1 - rank] if causal else [rank]


def block_kind(a: int, b: int, causal: bool) -> int:
    if not causal:
        return FULL
    return FULL if a > b else (DIAG if a == b else SKIP)


def local_chunks(x, rank: int, world: int, causal: bool):
    """This rank's chunks of a full [B, H, S, D] (or [B, H, S]) tensor, each
    contiguous, in rank_chunks order."""
    n_chunks = 2 * world if causal else world
    c = x.shape[2] // n_chunks
    return [x[:, :, i * c:(i + 1) * c].contiguous() for i in rank_chunks(rank, world, causal)]


class CudaBlocks:
    """The library's kernels on one (q chunk, kv chunk) block."""

    def __init__(self, scale: float):
        from . import cpattn as cp
        self.cp = cp
        self.scale = scale
        self._ws = None

    def new_acc(self, q):
        o = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
        lse = torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device)
        return o, lse

    def fwd(self, q, k, v, diag: bool):
        # one block = one-rank attention of the q chunk over the kv chunk
        return self.cp.fwd_step(q, k, v, 1, 0, causal=diag, scale=self.scale)

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        self.cp.merge_(o_acc, lse_acc, o_part, lse_part)

    def finalize(self, o_acc, dtype):
        return self.cp.finalize(o_acc, dtype)

    def zeros_f32(self, like):
        return torch.zeros(like.shape, dtype=torch.float32, device=like.device)

    def bwd_into(self, q, k, v, o, lse, do, diag: bool, dq_acc, dk_acc, dv_acc):
        """Adds the block's dQ, dK, dV terms, in fp32, to the three sums."""
        B, H, S, D = q.shape
        need = self.cp.bwd_workspace_bytes(B, H, S, D)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        self.cp.bwd_accumulate_(q, k, v, o, lse, do, dq_acc, dk_acc, dv_acc, 1, causal=diag,
                                scale=self.scale, workspace=self._ws)

    def add(self, acc, x):
        """acc += x, both fp32."""
        self.cp.accumulate_(acc, x)

    def cast(self, acc, dtype):
        return self.cp.finalize(acc, dtype)


def fwd_schedule(rank, world, q, k, v, causal, be):
    """Generator: the forward of rank `rank`.  q, k, v: its chunk tensors.
    Returns [(o, lse)] per own q chunk (o in q's dtype, lse fp32)."""
    own = rank_chunks(rank, world, causal)
    acc = [be.new_acc(x) for x in q]
    kv = list(k) + list(v)  # K then V of the chunks this rank holds now
    for t in range(world):
        src = (rank - t) % world
        ids = rank_chunks(src, world, causal)
        n = len(ids)
        pending = None
        if t + 1 < world:  # the next step's K/V travels while this step computes
            pending = yield ("start", kv)
        for ai, a in enumerate(own):
            for bi, b in enumerate(ids):
                kind = block_kind(a, b, causal)
                if kind == SKIP:
                    continue
                o_p, l_p = be.fwd(q[ai], kv[bi], kv[n + bi], kind == DIAG)
                be.merge(acc[ai][0], acc[ai][1], o_p, l_p)
        if t + 1 < world:
            kv = yield ("finish", pending)
    return [(be.finalize(o, q[ai].dtype), lse) for ai, (o, lse) in enumerate(acc)]


def bwd_schedule(rank, world, q, k, v, o, lse, do, causal, be):
    """Generator: the backward of rank `rank` from the forward's O and LSE of
    its rows.  Returns (dq, dk, dv) per own chunk in the inputs' dtype.

    The dK/dV sums travel around the ring with their K/V.  Step t adds its
    block terms into fresh sums for the K/V it holds; only then does it take
    in the running sums of that K/V from rank - 1 (sent at the end of that
    rank's step t - 1, so in flight during this step's blocks), add them, and
    send the result on, where it is in flight during step t + 1.  After the
    last step the sums of this rank's own chunks arrive from rank - 1."""
    own = rank_chunks(rank, world, causal)
    dq = [be.zeros_f32(x) for x in q]
    kv = list(k) + list(v)
    pending_dkv = None
    for t in range(world):
        src = (rank - t) % world
        ids = rank_chunks(src, world, causal)
        n = len(ids)
        pending_kv = None
        if t + 1 < world:  # the next step's K/V travels while this step computes
            pending_kv = yield ("start", kv)
        dkv = [be.zeros_f32(x) for x in kv]  # this step's dK, dV terms of the K/V held now
        for ai, a in enumerate(own):
            for bi, b in enumerate(ids):
                kind = block_kind(a, b, causal)
                if kind == SKIP:
                    continue
                be.bwd_into(q[ai], kv[bi], kv[n + bi], o[ai], lse[ai], do[ai], kind == DIAG,
                            dq[ai], dkv[bi], dkv[n + bi])
        if world > 1:
            if t > 0:  # the running sums of the same K/V, from rank - 1
                incoming = yield ("finish", pending_dkv)
                for acc, x in zip(dkv, incoming):
                    be.add(acc, x)
            pending_dkv = yield ("start", dkv)
        if t + 1 < world:
            kv = yield ("finish", pending_kv)
    if world > 1:
        dkv = yield ("finish", pending_dkv)
    m = len(own)
    dk = [be.cast(dkv[i], k[i].dtype) for i in range(m)]
    dv = [be.cast(dkv[m + i], v[i].dtype) for i in range(m)]
    return [be.cast(x, q[i].dtype) for i, x in enumerate(dq)], dk, dv


def run_dist(gen, group=None):
    """Drive a schedule generator over torch.distributed point-to-point ops."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:  # point-to-point peers are named by their global rank
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    try:
        msg = next(gen)
        while True:
            kind, payload = msg
            if kind == "start":
                bufs = [torch.empty_like(t) for t in payload]
                ops = ([dist.P2POp(dist.isend, t, nxt, group) for t in payload] +
                       [dist.P2POp(dist.irecv, b, prv, group) for b in bufs])
                msg = gen.send((dist.batch_isend_irecv(ops), bufs))
            else:
                reqs, bufs = payload
                for r in reqs:
                    r.wait()
                msg = gen.send(bufs)
    except StopIteration as e:
        return e.value


def run_loopback(gens):
    """Drive N ranks' schedule generators in one process (rank r's messages go
    to rank r + 1).  All ranks take the same exchange steps in the same order."""
    world = len(gens)
    results = [None] * world
    msgs = [None] * world
    done = 0
    for r, g in enumerate(gens):
        try:
            msgs[r] = next(g)
        except StopIteration as e:  # a schedule without exchanges (one rank)
            results[r] = e.value
            done += 1
    if done == world:
        return results
    if done:
        raise RuntimeError("ranks out of step")
    while True:
        kinds = {m[0] for m in msgs}
        if len(kinds) != 1:
            raise RuntimeError("ranks out of step")
        kind = kinds.pop()
        if kind == "start":
            sent = [m[1] for m in msgs]
            handles = [[t.clone() for t in sent[(r - 1) % world]] for r in range(world)]
        else:
            handles = [m[1] for m in msgs]
        done = 0
        for r in range(world):
            try:
                msgs[r] = gens[r].send(handles[r])
            except StopIteration as e:
                results[r] = e.value
                done += 1
        if done == world:
            return results
        if done:
            raise RuntimeError("ranks out of step")


def _drive(make_gen, group):
    """Run a schedule over torch.distributed, or as a single rank when no
    process group is initialised (no exchanges then)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return run_dist(make_gen(dist.get_rank(group), dist.get_world_size(group)), group)
    return run_loopback([make_gen(0, 1)])[0]


def ring_fwd(q, k, v, causal=True, scale=None, group=None):
    """Ring forward of this rank: q, k, v are its chunk tensors (local_chunks
    order).  Returns lists (o, lse) per own chunk."""
    scale = float(scale if scale is not None else q[0].shape[-1] ** -0.5)
    be = CudaBlocks(scale)
    out = _drive(lambda r, n: fwd_schedule(r, n, q, k, v, causal, be), group)
    return [o for o, _ in out], [l for _, l in out]


def ring_bwd(q, k, v, o, lse, do, causal=True, scale=None, group=None):
    """Ring backward of this rank: returns lists (dq, dk, dv) per own chunk."""
    scale = float(scale if scale is not None else q[0].shape[-1] ** -0.5)
    be = CudaBlocks(scale)
    return _drive(lambda r, n: bwd_schedule(r, n, q, k, v, o, lse, do, causal, be), group)
