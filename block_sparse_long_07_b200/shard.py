"""One MoBA prefill split across ranks by kv-head group.

At very long contexts (10M tokens: 256 blocks of 40960 keys, top-k fixed)
one problem no longer fits one GPU, and the method's authors extend tensor
parallelism to the query heads (wispaper.ai blog, "Efficiency and
Implementation").  Every step of the MoBA forward is independent per kv
head and its group of query heads: the block means, the gate, the bucketing,
the attention and the merge of head g read only q heads g*G .. g*G+G-1 and
kv head g.  So rank r of P takes the contiguous kv-head range

    [r * Hkv // P, (r + 1) * Hkv // P)

with its q heads, runs the ordinary library forward on that slice alone (no
collective inside the attention, and no rank ever reads another rank's
memory), and the outputs are concatenated along the head axis.  The only
exchange is that final gather of o and lse (and, optionally, the selection),
done with torch.distributed all_gather on whatever backend the process
group uses.

Nothing here computes any part of the method: it slices, calls a forward
function it is given (the library's, on the GPU) and concatenates.
"""


def kv_head_range(rank, world, num_kv_heads):
    """Contiguous kv heads [g0, g1) of `rank`; ranks differ by at most one head.
    Every rank must own at least one kv head."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("rank %d of %d" % (rank, world))
    if world > num_kv_heads:
        raise ValueError("%d ranks for %d kv heads: a rank would own none" %
                         (world, num_kv_heads))
    return rank * num_kv_heads // world, (rank + 1) * num_kv_heads // world


def q_head_range(rank, world, num_q_heads, num_kv_heads):
    """q heads [h0, h1) that read the kv heads of `rank` (contiguous GQA groups)."""
    if num_q_heads % num_kv_heads:
        raise ValueError("q heads must be a multiple of kv heads")
    G = num_q_heads // num_kv_heads
    g0, g1 = kv_head_range(rank, world, num_kv_heads)
    return g0 * G, g1 * G


def shard_inputs(q, k, v, rank, world):
    """This rank's slice of [b, N, H, d] (or packed [T, H, d]) inputs: q heads
    of its groups, kv heads of its range.  Returns contiguous tensors."""
    Hq, Hkv = q.shape[-2], k.shape[-2]
    h0, h1 = q_head_range(rank, world, Hq, Hkv)
    g0, g1 = kv_head_range(rank, world, Hkv)
    return (q[..., h0:h1, :].contiguous(), k[..., g0:g1, :].contiguous(),
            v[..., g0:g1, :].contiguous())


def _head_axis_of_lse(lse, batch_layout):
    # batch: lse [b, Hq, N]; packed (varlen): lse [Hq, T]
    return 1 if batch_layout else 0


def gather_heads(local, world, dist, axis, group=None):
    """Concatenate every rank's `local` tensor along `axis` in rank order.
    Ranks may hold different sizes along `axis` (uneven head splits): sizes
    are exchanged first and the pieces padded to the largest."""
    import torch
    n_local = torch.tensor([local.shape[axis]], dtype=torch.int64, device=local.device)
    sizes = [torch.zeros_like(n_local) for _ in range(world)]
    dist.all_gather(sizes, n_local, group=group)
    sizes = [int(s.item()) for s in sizes]
    m = max(sizes)
    if local.shape[axis] < m:
        pad_shape = list(local.shape)
        pad_shape[axis] = m - local.shape[axis]
        local = torch.cat([local, local.new_zeros(pad_shape)], dim=axis)
    local = local.contiguous()
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local, group=group)
    parts = [p.narrow(axis, 0, s) for p, s in zip(parts, sizes)]
    return torch.cat(parts, dim=axis)


def run_shard(forward_fn, q_r, k_r, v_r, world, dist, batch_layout=True, group=None):
    """Run `forward_fn(q_r, k_r, v_r) -> (o_r, lse_r[, sel_r])` on this
    rank's head slice (already sliced, e.g. generated per kv-head group) and
    return the full (o, lse[, sel]) gathered from all ranks, heads in order.
    Layouts: batch o [b, N, Hq, d], lse [b, Hq, N], sel [b, Hq, N, k];
    packed o [T, Hq, d], lse [Hq, T], sel [Hq, T, k]."""
    out = forward_fn(q_r, k_r, v_r)
    o_r, lse_r = out[0], out[1]
    o = gather_heads(o_r, world, dist, axis=o_r.dim() - 2, group=group)
    lse = gather_heads(lse_r, world, dist, axis=_head_axis_of_lse(lse_r, batch_layout),
                       group=group)
    res = [o, lse]
    if len(out) > 2 and out[2] is not None:
        res.append(gather_heads(out[2], world, dist, axis=1 if batch_layout else 0,
                                group=group))
    return tuple(res)


def forward_sharded(forward_fn, q, k, v, rank, world, dist, batch_layout=True, group=None):
    """run_shard on this rank's slice of the full inputs q, k, v."""
    qr, kr, vr = shard_inputs(q, k, v, rank, world)
    return run_shard(forward_fn, qr, kr, vr, world, dist, batch_layout, group)
