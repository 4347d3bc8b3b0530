"""Host-side data parallelism for the layer: independent (batch, KV head) chains.

Each KV head's memory (and the query heads that read it) is independent of
every other head and batch row: the method keeps one compressive memory per
head ("Leave No Context Behind" explainer, section "メモリ構造").  So the work
splits across ranks with no data-path exchange.  The (batch row, KV head)
chains form a B x H_kv grid; a rank takes one rectangular block of it (a run
of batch rows times a run of KV heads, with every query head of those KV
heads' groups), runs the forward on its own GPU on contiguous copies of its
block, and results are assembled by an all-gather.  Splitting along the KV
heads comes first, so a single long stream (B = 1, the 1M-token shape) also
splits.  The only collectives are for timing (max over ranks) and, when a
caller wants the full result on one rank, the gather.

Sequence parallelism for the linear rule.  Under the linear rule the memory
after a run of segments is the memory before it plus a sum over the run's
tokens ("Hugging Face Infini-Attention 再現分析", Memory Update: the
outer-product contributions accumulate; z is the running sum of sigma(K)).
So a sequence cut at segment boundaries into one contiguous run per rank
needs one exchange: every rank computes its run's update from a zero state,
the updates are all-gathered, each rank adds those of the ranks before it to
the initial state (an exclusive prefix, in rank order, so every rank forms
the same sums; the library's infini_attn_state_sum does the additions) and
then runs the forward over its own segments from there.  The delta rule's
update depends on the memory it starts from, so it stays sequential in the
segments and is sharded by chains only.
"""

import torch
import torch.distributed as dist


def batch_range(B, world, rank):
    """Contiguous batch rows [b0, b1) for `rank` of `world` (near-equal split)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(B, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)


def shard_batch(t, world, rank, dim=0):
    """The rank's slice of a [B, ...] tensor along `dim` (a view)."""
    b0, b1 = batch_range(t.shape[dim], world, rank)
    return t.narrow(dim, b0, b1 - b0)


def gather_batch(local, B, world, group=None):
    """All-gather per-rank batch slices (possibly unequal) into the full tensor."""
    sizes = [batch_range(B, world, r)[1] - batch_range(B, world, r)[0] for r in range(world)]
    width = max(sizes)
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:n] for p, n in zip(parts, sizes)], dim=0)


def split_factors(B, H_kv, world):
    """(wb, wh) with wb * wh == world: ranks along the batch rows and along the
    KV heads.  Each is at most its extent; splits that divide both extents
    evenly come first, then the larger head split."""
    best = None
    for wh in range(min(world, H_kv), 0, -1):
        if world % wh:
            continue
        wb = world // wh
        if wb > B:
            continue
        key = (H_kv % wh == 0 and B % wb == 0, wh)
        if best is None or key > best[0]:
            best = (key, (wb, wh))
    if best is None:
        raise ValueError(f"{world} ranks cannot each take a block of {B} batch rows x {H_kv} KV heads")
    return best[1]


def chain_block(B, H_kv, world, rank):
    """`rank`'s block of (batch row, KV head) chains: rows [b0, b1) and KV heads
    [h0, h1) (near-equal splits; together the blocks tile the B x H_kv grid)."""
    wb, wh = split_factors(B, H_kv, world)
    if not 0 <= rank < world:
        raise ValueError("bad rank")
    rb, rh = divmod(rank, wh)
    b0, b1 = batch_range(B, wb, rb)
    h0, h1 = batch_range(H_kv, wh, rh)
    return b0, b1, h0, h1


def shard_chains(t, block, group_size=1):
    """Contiguous copy of the block's part of a [B, heads, ...] tensor, where
    each KV head owns `group_size` consecutive heads of `t` (the query heads of
    its group for q, out and beta's broadcast; 1 for k, v, M and z)."""
    b0, b1, h0, h1 = block
    return t[b0:b1, h0 * group_size:h1 * group_size].contiguous()


def gather_chains(local, B, H_kv, world, group_size=1, group=None):
    """All-gather every rank's block (from shard_chains layout, possibly of
    unequal sizes) into the full [B, H_kv * group_size, ...] tensor."""
    blocks = [chain_block(B, H_kv, world, r) for r in range(world)]
    nb = max(b1 - b0 for b0, b1, _, _ in blocks)
    nh = max(h1 - h0 for _, _, h0, h1 in blocks) * group_size
    rest = tuple(local.shape[2:])
    pad = torch.zeros((nb, nh) + rest, dtype=local.dtype, device=local.device)
    pad[: local.shape[0], : local.shape[1]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    full = torch.empty((B, H_kv * group_size) + rest, dtype=local.dtype, device=local.device)
    for part, (b0, b1, h0, h1) in zip(parts, blocks):
        full[b0:b1, h0 * group_size:h1 * group_size] = part[: b1 - b0, : (h1 - h0) * group_size]
    return full


def max_over_ranks(value, device=None, group=None):
    """Max of a per-rank float (e.g. elapsed ms), identical on every rank."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def segment_range(L, S, world, rank):
    """Token rows [l0, l1) of `rank`'s contiguous run of whole segments (a
    near-equal split of the T = ceil(L / S) segments; only the last run may
    end in the shorter final segment, and a run may be empty)."""
    if S < 1 or L < 1:
        raise ValueError("bad L/S")
    T = -(-L // S)
    s0, s1 = batch_range(T, world, rank)
    return min(s0 * S, L), min(s1 * S, L)


def local_state_update(k, v, seg_len, state_update, dtype=torch.float32):
    """This rank's linear-rule update from a zero state, packed flat:
    [dM (B*H_kv*d_k*d_v), dz (B*H_kv*d_k)] in the state's dtype (float32 for
    the library).  `state_update` is the library call
    (k, v, M_in, z_in, seg_len, rule) -> (M_out, z_out)."""
    B, H_kv, L, d_k = k.shape
    d_v = v.shape[3]
    M0 = torch.zeros((B, H_kv, d_k, d_v), dtype=dtype, device=k.device)
    z0 = torch.zeros((B, H_kv, d_k), dtype=dtype, device=k.device)
    if L == 0:
        return torch.cat([M0.flatten(), z0.flatten()])
    dM, dz = state_update(k, v, M0, z0, seg_len, "linear")
    return torch.cat([dM.flatten(), dz.flatten()])


def prefix_states(updates, rank, M0, z0, state_sum):
    """(M_in, z_in) of `rank` and the final (M_T, z_T) from the gathered
    per-rank updates (`updates`: [world, packed], rank order): M0 plus the
    updates of ranks before `rank`, and plus all of them.  `state_sum` is the
    library call (M_base, z_base, parts, n_parts) -> (M, z), which adds the
    parts in order (api.state_sum)."""
    M_in, z_in = state_sum(M0, z0, updates, rank)
    M_T, z_T = state_sum(M0, z0, updates, updates.shape[0])
    return M_in, z_in, M_T, z_T


def all_gather_flat(t, group=None):
    """All-gather equal-size flat tensors into one [world, n] tensor in rank
    order (one rank: [1, n])."""
    t = t.contiguous().view(1, -1)
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return t
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, t, group=group)
    return torch.cat(parts, dim=0)


def sequence_parallel_forward(q, k, v, beta, M0, z0, seg_len, forward, state_update, state_sum,
                              group=None):
    """Linear-rule forward of this rank's run of segments.

    q, k, v: the rank's token rows [l0, l1) from segment_range (B, heads and d
    as for the whole sequence); M0, z0: the state before token 0.  `forward`,
    `state_update` and `state_sum` are the library calls (api.forward,
    api.state_update, api.state_sum).  Returns (out for the rank's rows, M_T,
    z_T) with the state after the whole sequence on every rank.  One
    all-gather of B * H_kv * (d_k d_v + d_k) floats per rank is the only
    exchange.
    """
    updates = all_gather_flat(local_state_update(k, v, seg_len, state_update, M0.dtype), group)
    rank = dist.get_rank(group) if dist.is_available() and dist.is_initialized() else 0
    M_in, z_in, M_T, z_T = prefix_states(updates, rank, M0, z0, state_sum)
    if q.shape[2] == 0:
        return q.new_empty(q.shape[:3] + (v.shape[3],)), M_T, z_T
    out, _, _ = forward(q, k, v, beta, M_in, z_in, seg_len, "linear")
    return out, M_T, z_T
