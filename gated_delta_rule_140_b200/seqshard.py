"""Sequence-sharded prefill: one long sequence (or a batch of equally long ones)
split into contiguous segments, one per rank, with one exchange of per-segment
affine state maps.

Over a segment the recurrence S_t = S_{t-1} A_t + beta_t v_t k_t^T, with
A_t = Diag(alpha_t)(I - beta_t k_t k_t^T) (FG2-GDN section 1; GDN's scalar decay
is the special case), is affine in the state it starts from:

    S_end = S_start M + B,   M = A_1 ... A_n,   B = S_end from S_start = 0.

Each rank r >= 1 computes its segment's map with two prefill calls of its own
tokens (B from a zero state; M from the identity with v = 0: every row of the
state is a probe vector); rank 0, whose start is the sequence's initial state,
runs its segment directly and publishes (M, B) = (0, its final state).  One
all-gather shares the maps (2 x H x d_k x d_k fp32 per sequence and rank); each
rank composes its true start S_start(r) = S_start(r - 1) M_{r-1} + B_{r-1} with
the compose kernel and reruns its segment from it, which gives its outputs and
its final state.  Ranks >= 1 do three passes over their segment, rank 0 one:
``balanced_bounds`` splits a sequence so that rank 0 takes three times the tokens of
each other rank, which balances the passes.

Every step runs in libgdn.so's kernels (gdn_chunk_fwd, gdn_state_identity,
gdn_state_compose); the collective is torch.distributed's all-gather (NCCL over
NVLink between GPUs).  The ``prefill``, ``compose`` and ``identity`` arguments
exist so that the exchange can be run on CPU ranks with other implementations of
the same three operations; their defaults are the library's.
"""


def balanced_bounds(T, world, chunk=64):
    """Token boundaries [0, b_1, ..., T] of ``world`` segments that balance the
    passes: rank 0 runs its segment once, the others three times (two map passes
    and the rerun), so rank 0 takes about three times the tokens of each other
    rank, T / (world + 2) per pass.  Boundaries fall on multiples of ``chunk``
    where the lengths allow, so that no segment but the last ends in a partial
    chunk.  With one rank the whole sequence is rank 0's."""
    if world < 1 or T < 0:
        raise ValueError("world >= 1 and T >= 0")
    if world == 1:
        return [0, T]
    unit = T / (world + 2)
    bounds = [0]
    for r in range(1, world):
        b = int(round((3 + (r - 1)) * unit / chunk)) * chunk
        bounds.append(min(max(b, bounds[-1]), T))
    bounds.append(T)
    return bounds


def _default_ops():
    from . import _native as nat

    def prefill(q, k, v, log_alpha, beta, s0):
        return nat.chunk_fwd(q, k, v, log_alpha, beta, s0, check=True)

    def compose(s, m, b):
        return nat.state_compose(s, m, b)

    def identity(n, h, d, like):
        return nat.state_identity(n, h, d, like.device)

    return prefill, compose, identity


def segment_map(q, k, v, log_alpha, beta, *, prefill=None, identity=None):
    """(M, B) of one segment: B = the final state from a zero state, M = the final
    state from the identity with v = 0 ([B,H,d_k,d_k])."""
    import torch
    dp, _, di = _default_ops() if prefill is None or identity is None else (None, None, None)
    prefill = prefill or dp
    identity = identity or di
    n, _, h, dk = q.shape
    _, b_map = prefill(q, k, v, log_alpha, beta, None)
    zv = torch.zeros(v.shape[:-1] + (dk,), dtype=v.dtype, device=v.device)
    _, m_map = prefill(q, k, zv, log_alpha, beta, identity(n, h, dk, b_map))
    return m_map, b_map


def start_state(maps, rank, *, compose=None):
    """S_start(rank) from the maps (M_j, B_j) of segments j < rank, where segment 0
    publishes (0, its final state): B_0, then S <- S M_j + B_j for j = 1 .. rank - 1."""
    if rank == 0:
        raise ValueError("rank 0 starts from the sequence's initial state")
    compose = compose or _default_ops()[1]
    s = maps[0][1]
    for j in range(1, rank):
        s = compose(s, maps[j][0], maps[j][1])
    return s


def sequence_sharded_prefill(q, k, v, log_alpha, beta, initial_state=None, *, group=None,
                             prefill=None, compose=None, identity=None):
    """This rank's segment of a sequence-sharded prefill.

    q, k [B,T_r,H,d_k], v [B,T_r,H,d_v], log_alpha [B,T_r,H] or [B,T_r,H,d_k],
    beta [B,T_r,H]: rank r's contiguous tokens of B sequences (ranks in token
    order; d_v == d_k).  ``initial_state`` [B,H,d_v,d_k] (rank 0's; ignored
    elsewhere).  Returns (o [B,T_r,H,d_v], the state after this segment); the last
    rank's is the sequences' final state.  Every rank of ``group`` must call it."""
    import torch
    import torch.distributed as dist
    dp, dc, di = _default_ops() if None in (prefill, compose, identity) else (None, None, None)
    prefill, compose, identity = prefill or dp, compose or dc, identity or di
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    n, _, h, dk = q.shape
    if v.shape[-1] != dk:
        raise ValueError("sequence sharding needs d_v == d_k (the maps are d_k x d_k)")
    if rank == 0:
        o, s_end = prefill(q, k, v, log_alpha, beta, initial_state)
        m_map, b_map = torch.zeros_like(s_end), s_end
    else:
        m_map, b_map = segment_map(q, k, v, log_alpha, beta, prefill=prefill, identity=identity)
    m_all = [torch.empty_like(m_map) for _ in range(world)]
    b_all = [torch.empty_like(b_map) for _ in range(world)]
    dist.all_gather(m_all, m_map.contiguous(), group=group)
    dist.all_gather(b_all, b_map.contiguous(), group=group)
    if rank == 0:
        return o, s_end
    s0 = start_state(list(zip(m_all, b_all)), rank, compose=compose)
    return prefill(q, k, v, log_alpha, beta, s0)
