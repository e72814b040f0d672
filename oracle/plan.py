"""Plan oracle: the zigzag chunk ownership and the ring block schedule, restated
in plain Python.  TEST INFRASTRUCTURE ONLY (tests/ and bench.py's baseline leg).

Rules, from "Configuring RingAttention+FlashAttention for CP" (devpress.csdn.net):
  * section 5, item 1: with N ranks and a causal mask the sequence is cut into
    2N chunks and rank r holds chunks r and 2N-1-r (worked example N=4:
    GPU0 {0,7}, GPU1 {1,6}, GPU2 {2,5}, GPU3 {3,4});
  * section 3 code: at ring step t rank r works on the K/V of rank
    (r - t) mod N;
  * section 3, note 2: the causal mask must be exact: a (q chunk a, kv chunk b)
    block is SKIP when a < b, DIAG when a == b, FULL when a > b.
Without a causal mask the split is contiguous (rank r holds chunk r) and every
block is FULL.

Row format (one per (rank, step, q-slot, kv-slot), SKIP rows included):
  (rank, step, q_chunk, kv_chunk, src_rank, kind)   kind: 0 SKIP, 1 FULL, 2 DIAG
"""

SKIP, FULL, DIAG = 0, 1, 2


def owned_chunks(rank: int, cp_size: int, causal: bool):
    if causal:
        return [rank, 2 * cp_size - 1 - rank]
    return [rank]


def chunk_owner(chunk: int, cp_size: int, causal: bool) -> int:
    for r in range(cp_size):
        if chunk in owned_chunks(r, cp_size, causal):
            return r
    raise ValueError("chunk out of range")


def block_kind(a: int, b: int, causal: bool) -> int:
    if not causal:
        return FULL
    if a < b:
        return SKIP
    if a == b:
        return DIAG
    return FULL


def plan_rows(S: int, cp_size: int, causal: bool):
    n_chunks = 2 * cp_size if causal else cp_size
    if cp_size < 1 or S % n_chunks != 0:
        raise ValueError("S must be a multiple of the chunk count")
    rows = []
    for r in range(cp_size):
        for t in range(cp_size):
            src = (r - t) % cp_size
            for a in owned_chunks(r, cp_size, causal):
                for b in owned_chunks(src, cp_size, causal):
                    rows.append((r, t, a, b, src, block_kind(a, b, causal)))
    return rows


def chunk_len(S: int, cp_size: int, causal: bool) -> int:
    return S // (2 * cp_size if causal else cp_size)
