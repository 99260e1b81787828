"""Ring attention forward across the ranks of a torch.distributed process group.

The "相关工作" page (paper 7, "Ring Attention with Blockwise Transformers") describes
distributing the key/value blocks of a sequence over devices connected in a ring: every
device keeps its own query block and attends it to the K/V block it currently holds, then
passes that block to the next device, so after W hops every query block has seen every
K/V block while each device only ever holds two of them.  The local step is the forward
kernel; the per-hop partial results are folded together with the exact merge of
``attn_merge_partial`` (the tutorial's 修正公式 applied to whole blocks).

Layout: a batch of B sequences of length W * n is cut into W contiguous chunks of n
tokens; rank r holds tokens [r n, (r+1) n) of every sequence, packed token-major by
sequence (q [B n, Hq, d], k and v [B n, Hkv, d]).  Under the causal mask a chunk is
fully visible to the later chunks, causally visible to itself and hidden from the
earlier ones.  Communication is NCCL point-to-point (over NVLink between the GPUs of one
node); the K/V transfer of the next hop runs while the current hop is computed.

The backward walks the same ring.  With the full forward's O and LSE of this rank's rows
(what ``ring_attn_fwd`` returns), the gradient over one K/V block is exactly the backward
of the (query chunk, K/V block) pair given those O and LSE (the tutorial's 反向重算流程:
P is recomputed from the saved LSE, D from the saved O), so dQ is the sum of the per-hop
dQ, and each block's dK / dV accumulate as the block travels: they are passed on with it
after every hop and arrive back at the block's owner after the last one.  The sums are
float32 throughout: every hop's backward adds straight into them (attn_bwd_accumulate),
and they are rounded to bf16 once, at the end.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import attn_bwd_accumulate, attn_fwd, attn_merge_finish, attn_merge_partial


def ring_schedule(rank: int, world: int, causal: bool):
    """For hop s = 0..world-1: (index of the K/V chunk rank `rank` holds at that hop, mask),
    mask being "causal" (its own chunk), "full" (an earlier chunk, or any chunk without the
    causal mask) or None (a later chunk under the causal mask: nothing to compute)."""
    hops = []
    for s in range(world):
        j = (rank - s) % world
        if not causal:
            kind = "full"
        elif j == rank:
            kind = "causal"
        else:
            kind = "full" if j < rank else None
        hops.append((j, kind))
    return hops


def ring_attn_fwd(q, k, v, batch, scale=None, causal=False, group=None, local_fwd=None, merge=None, finish=None,
                  acc_dtype=torch.float32):
    """Attention of this rank's query chunk over the whole sequences.  Returns
    (o [B n, Hq, d] bf16, lse [Hq, B n] float32), the rows of the full forward that belong
    to this rank.  ``local_fwd(q, k, v, causal) -> (o, lse)``, ``merge(o_acc, lse_acc,
    o, lse, first)`` and ``finish(o_acc) -> o`` default to the library's CUDA kernels
    (attn_fwd, attn_merge_partial, attn_merge_finish), whose accumulators are float32
    (``acc_dtype``)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if local_fwd is None:
        def local_fwd(q_, k_, v_, c_):
            return attn_fwd(q_, k_, v_, scale=scale, causal=c_, batch=batch)
    if merge is None:
        merge = attn_merge_partial
    if finish is None:
        finish = attn_merge_finish
    T, hq, _ = q.shape
    o_acc = torch.empty(q.shape, dtype=acc_dtype, device=q.device)
    lse_acc = torch.empty(hq, T, dtype=acc_dtype, device=q.device)
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    k_cur, v_cur = k.contiguous(), v.contiguous()
    first = True
    for s, (_, kind) in enumerate(ring_schedule(rank, world, causal)):
        reqs = []
        if s + 1 < world:
            # pass the block on while it is being used; receive the previous rank's
            k_nxt, v_nxt = torch.empty_like(k_cur), torch.empty_like(v_cur)
            reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, k_cur, nxt, group), dist.P2POp(dist.irecv, k_nxt, prv, group),
                dist.P2POp(dist.isend, v_cur, nxt, group), dist.P2POp(dist.irecv, v_nxt, prv, group)])
        if kind is not None:
            o_p, lse_p = local_fwd(q, k_cur, v_cur, kind == "causal")
            merge(o_acc, lse_acc, o_p, lse_p, first)
            first = False
        for r in reqs:
            r.wait()
        if s + 1 < world:
            k_cur, v_cur = k_nxt, v_nxt
    return finish(o_acc), lse_acc


def ring_attn_bwd(q, k, v, o, do, lse, batch, scale=None, causal=False, group=None, local_bwd=None, finish=None,
                  acc_dtype=torch.float32):
    """Gradients of the ring forward for this rank: (dq [B n, Hq, d] for its query chunk,
    dk, dv [B n, Hkv, d] for its K/V chunk).  ``o`` / ``lse`` are this rank's rows of the
    full forward (``ring_attn_fwd``'s outputs), ``do`` their upstream gradient.
    ``local_bwd(q, k, v, causal, dq_acc, dk_acc, dv_acc)`` adds the pair's gradients into the
    ``acc_dtype`` accumulators; it defaults to the library's attn_bwd_accumulate with the given
    o, do, lse.  ``finish(acc) -> tensor`` turns an accumulator into the result; by default
    the library's attn_merge_finish (float32 to bf16)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if local_bwd is None:
        def local_bwd(q_, k_, v_, c_, dq_a, dk_a, dv_a):
            attn_bwd_accumulate(q_, k_, v_, o, do, lse, dq_a, dk_a, dv_a, scale=scale, causal=c_, batch=batch)
    if finish is None:
        finish = attn_merge_finish
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    dq_acc = torch.zeros(q.shape, dtype=acc_dtype, device=q.device)
    k_cur, v_cur = k.contiguous(), v.contiguous()
    dk_cur = torch.zeros(k.shape, dtype=acc_dtype, device=k.device)
    dv_cur = torch.zeros(v.shape, dtype=acc_dtype, device=v.device)
    for s, (_, kind) in enumerate(ring_schedule(rank, world, causal)):
        kv_reqs = []
        if s + 1 < world:
            # the next hop's block moves while this hop is computed
            k_nxt, v_nxt = torch.empty_like(k_cur), torch.empty_like(v_cur)
            kv_reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, k_cur, nxt, group), dist.P2POp(dist.irecv, k_nxt, prv, group),
                dist.P2POp(dist.isend, v_cur, nxt, group), dist.P2POp(dist.irecv, v_nxt, prv, group)])
        if kind is not None:
            local_bwd(q, k_cur, v_cur, kind == "causal", dq_acc, dk_cur, dv_cur)
        # the block's gradients so far go on with it (after the last hop: to its owner)
        g_reqs = []
        if world > 1:
            dk_in, dv_in = torch.empty_like(dk_cur), torch.empty_like(dv_cur)
            g_reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, dk_cur, nxt, group), dist.P2POp(dist.irecv, dk_in, prv, group),
                dist.P2POp(dist.isend, dv_cur, nxt, group), dist.P2POp(dist.irecv, dv_in, prv, group)])
        for r in kv_reqs + g_reqs:
            r.wait()
        if world > 1:
            dk_cur, dv_cur = dk_in, dv_in
        if s + 1 < world:
            k_cur, v_cur = k_nxt, v_nxt
    return finish(dq_acc), finish(dk_cur), finish(dv_cur)
