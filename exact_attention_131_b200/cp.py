"""Context-parallel attention forward: the sequence is cut into equal chunks, one
per rank, and the K/V chunks travel around a ring of ranks.

"TransformerEngine: FA4 in context-parallel attention" (flowchart): each rank
keeps its query chunk, computes attention against every K/V chunk it may see as
the chunks pass by, and merges the partial results by their log-sum-exps
(``arc_attn_merge``).  With a causal mask over the whole sequence, query chunk
r sees its own chunk under the causal mask, every earlier chunk in full and no
later chunk.  A sink, if any, enters once, in the merge.

Transport is ``torch.distributed`` point-to-point (NCCL over NVLink between
GPUs): every step each rank sends the chunk it holds to rank + 1 and receives
the next one from rank - 1 into its own memory, so a kernel only ever reads
local HBM.  The exchange of step s + 1 is posted before the attention of step s
runs.  All ranks take the same steps in the same order.
"""
from __future__ import annotations


from . import attn_fwd, attn_merge


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, src, mask)] for one rank: at step s it holds the K/V chunk of rank
    src = (rank - s) mod world; mask is True (causal within the chunk), False
    (no mask) or None (the chunk is invisible and is skipped)."""
    out = []
    for step in range(world):
        src = (rank - step) % world
        if not causal:
            mask = False
        elif src == rank:
            mask = True
        elif src < rank:
            mask = False
        else:
            mask = None
        out.append((step, src, mask))
    return out


def _default_attn(q, k, v, *, causal, scale):
    return attn_fwd(q, k, v, scale=scale, causal=causal)


def _default_merge(o_parts, lse_parts, *, sinks, sink_rows):
    return attn_merge(o_parts, lse_parts, sinks=sinks, sink_rows=sink_rows)


def ring_attention_forward(q, k, v, *, group=None, causal=True, scale=None, sinks=None, attn=None, merge=None):
    """O, LSE of this rank's query chunk over the whole sequence.

    q [B, H, L, D], k [B, Hkv, L, D], v [B, Hkv, L, Dv]: this rank's chunk (rank r
    holds positions r*L .. r*L + L - 1).  sinks: optional [H] fp32 sink logits.
    attn / merge: the per-chunk attention and the merge; the library's kernels by
    default (tests substitute others to check the schedule without a GPU).
    """
    import torch
    import torch.distributed as dist

    attn = attn or _default_attn
    merge = merge or _default_merge
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    k_shape, v_shape = k.shape, v.shape
    cur = torch.cat([k.contiguous().reshape(-1), v.contiguous().reshape(-1)])   # one buffer per hop
    nk = k.numel()
    q = q.contiguous()
    o_parts, lse_parts = [], []
    for step, src, mask in ring_schedule(rank, world, causal):
        reqs, nxt_buf = [], None
        if step + 1 < world:
            nxt_buf = torch.empty_like(cur)
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, cur, nxt, group),
                                           dist.P2POp(dist.irecv, nxt_buf, prv, group)])
        if mask is not None:
            k_s = cur[:nk].view(k_shape)
            v_s = cur[nk:].view(v_shape)
            o_i, l_i = attn(q, k_s, v_s, causal=mask, scale=scale)
            o_parts.append(o_i)
            lse_parts.append(l_i)
        for r in reqs:
            r.wait()
        if nxt_buf is not None:
            cur = nxt_buf
    return merge(o_parts, lse_parts, sinks=sinks, sink_rows=q.shape[2])


def context_parallel_forward_local(q, k, v, world, *, causal=True, scale=None, sinks=None):
    """The ring forward for every rank, run on one device without communication:
    q, k, v are whole sequences [B, *, world*L, *]; returns the per-rank (O, LSE)
    chunks, computed by the same schedule and kernels as ring_attention_forward."""
    T = q.shape[2]
    if T % world:
        raise ValueError("the sequence length must divide into world equal chunks")
    L = T // world
    chunk = lambda x, r: x[:, :, r * L:(r + 1) * L].contiguous()
    out = []
    for rank in range(world):
        qr = chunk(q, rank)
        o_parts, lse_parts = [], []
        for _, src, mask in ring_schedule(rank, world, causal):
            if mask is not None:
                o_i, l_i = _default_attn(qr, chunk(k, src), chunk(v, src), causal=mask, scale=scale)
                o_parts.append(o_i)
                lse_parts.append(l_i)
        out.append(_default_merge(o_parts, lse_parts, sinks=sinks, sink_rows=L))
    return out
