"""Ring attention forward and backward across the ranks of a torch.distributed process group.

The "相关工作" page (paper 7, "Ring Attention with Blockwise Transformers") describes
distributing the key/value blocks of a sequence over devices connected in a ring: every
device keeps its own query block and attends it to the K/V block it currently holds, then
passes that block to the next device, so after W hops every query block has seen every
K/V block while each device only ever holds two of them.  The local step is the forward
kernel; the per-hop partial results are folded together with the exact merge of
``attn_merge_partial`` (the tutorial's 修正公式 applied to whole blocks).

Two layouts of a batch of B sequences over W ranks:

* ``"contiguous"``: each sequence is cut into W chunks of n tokens; rank r holds chunk r of
  every sequence, packed token-major by sequence (q [B n, Hq, d], k and v [B n, Hkv, d]).
  Under the causal mask rank r has r + 1 blocks to compute and rank W - 1 has W: the last
  rank sets the pace.
* ``"zigzag"``: each sequence is cut into 2W chunks of c tokens; rank r holds chunks r and
  2W - 1 - r, stored half-major (q [2, B c, Hq, d]: the B sequences' chunk r, then their
  chunk 2W - 1 - r; k and v likewise).  Under the causal mask every rank then has the same
  work, 2W - 1 full (c x c) blocks and 2 diagonal ones: a query chunk x sees the x chunks
  before it in full and itself causally, and x + (2W - 1 - x) is the same for every rank.
  ``zigzag_shard`` / ``zigzag_unshard`` convert between this layout and whole sequences.

A chunk is fully visible to the later chunks, causally visible to itself and hidden from
the earlier ones.  Communication is NCCL point-to-point (over NVLink between the GPUs of one
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

LAYOUTS = ("contiguous", "zigzag")


def _kind(kv_chunk, q_chunk, causal):
    """Mask of a (query chunk, K/V chunk) pair: "full", "causal" (the same chunk) or None
    (a later K/V chunk under the causal mask: nothing to compute)."""
    if not causal or kv_chunk < q_chunk:
        return "full"
    return "causal" if kv_chunk == q_chunk else None


def ring_schedule(rank: int, world: int, causal: bool):
    """Contiguous layout.  For hop s = 0..world-1: (index of the K/V chunk rank `rank`
    holds at that hop, mask), mask being "causal" (its own chunk), "full" (an earlier
    chunk, or any chunk without the causal mask) or None (nothing to compute)."""
    return [((rank - s) % world, _kind((rank - s) % world, rank, causal)) for s in range(world)]


def zigzag_schedule(rank: int, world: int, causal: bool):
    """Zig-zag layout.  For hop s = 0..world-1: the list of (query half a, K/V half b, mask)
    to compute, a and b in {0, 1} (half 0 of a rank is its chunk r, half 1 its chunk
    2W - 1 - r; at hop s the visiting block is rank (rank - s) mod W's)."""
    hops = []
    for s in range(world):
        j = (rank - s) % world
        q_chunks = (rank, 2 * world - 1 - rank)
        kv_chunks = (j, 2 * world - 1 - j)
        hops.append([(a, b, _kind(kv_chunks[b], q_chunks[a], causal))
                     for a in (0, 1) for b in (0, 1) if _kind(kv_chunks[b], q_chunks[a], causal) is not None])
    return hops


def zigzag_shard(x, batch, rank, world):
    """This rank's zig-zag part of a whole-sequence tensor x [B N, H, d] (N divisible by
    2W): [2, B c, H, d], half 0 = chunk rank of every sequence, half 1 = chunk 2W-1-rank."""
    BN = x.shape[0]
    c = BN // batch // (2 * world)
    xs = x.reshape(batch, 2 * world, c, *x.shape[1:])
    return torch.stack([xs[:, rank], xs[:, 2 * world - 1 - rank]]).reshape(2, batch * c, *x.shape[1:])


def zigzag_unshard(parts, batch):
    """Whole-sequence [B N, H, d] from every rank's zig-zag part (a list over ranks of
    [2, B c, H, d])."""
    world = len(parts)
    c = parts[0].shape[1] // batch
    chunks = [None] * (2 * world)
    for r, p in enumerate(parts):
        p = p.reshape(2, batch, c, *p.shape[2:])
        chunks[r], chunks[2 * world - 1 - r] = p[0], p[1]
    return torch.stack(chunks, dim=1).reshape(batch * 2 * world * c, *parts[0].shape[2:])


def _finish_rows(finish, acc):
    """finish() over all rows of an accumulator [halves, T, H, d] at once (it takes [rows,
    H, d]), in the accumulator's shape."""
    return finish(acc.reshape(-1, *acc.shape[-2:])).reshape(acc.shape)


def _peers(group, world, rank):
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    return nxt, prv


def _exchange(tensors, nxt, prv, group):
    """Send each tensor to the next rank and receive its counterpart from the previous
    one; returns (received tensors, requests)."""
    received = [torch.empty_like(t) for t in tensors]
    ops = []
    for t, r in zip(tensors, received):
        ops += [dist.P2POp(dist.isend, t, nxt, group), dist.P2POp(dist.irecv, r, prv, group)]
    return received, dist.batch_isend_irecv(ops)


def ring_attn_fwd(q, k, v, batch, scale=None, causal=False, group=None, local_fwd=None, merge=None, finish=None,
                  acc_dtype=torch.float32, layout="contiguous"):
    """Attention of this rank's query rows over the whole sequences.  Contiguous layout:
    returns (o [B n, Hq, d] bf16, lse [Hq, B n] float32), the rows of the full forward that
    belong to this rank.  Zig-zag layout (q [2, B c, Hq, d], k, v [2, B c, Hkv, d]): returns
    (o [2, B c, Hq, d], lse [2, Hq, B c]), half by half.  ``local_fwd(q, k, v, causal) ->
    (o, lse)``, ``merge(o_acc, lse_acc, o, lse, first)`` and ``finish(o_acc) -> o`` default
    to the library's CUDA kernels (attn_fwd, attn_merge_partial, attn_merge_finish), whose
    accumulators are float32 (``acc_dtype``)."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {LAYOUTS}")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if local_fwd is None:
        def local_fwd(q_, k_, v_, c_):
            return attn_fwd(q_, k_, v_, scale=scale, causal=c_, batch=batch)
    if merge is None:
        merge = attn_merge_partial
    if finish is None:
        finish = attn_merge_finish
    nxt, prv = _peers(group, world, rank)
    halves = 2 if layout == "zigzag" else 1
    q = q.contiguous()
    qh = q if layout == "zigzag" else q.unsqueeze(0)
    T, hq = qh.shape[1], qh.shape[2]
    o_acc = torch.empty(qh.shape, dtype=acc_dtype, device=q.device)
    lse_acc = torch.empty(halves, hq, T, dtype=acc_dtype, device=q.device)
    first = [True] * halves
    if layout == "zigzag":
        hops = zigzag_schedule(rank, world, causal)
    else:
        hops = [[(0, 0, kind)] if kind is not None else [] for _, kind in ring_schedule(rank, world, causal)]
    k_cur, v_cur = k.contiguous(), v.contiguous()
    for s, pairs in enumerate(hops):
        reqs = []
        if s + 1 < world:
            # pass the block on while it is being used; receive the previous rank's
            (k_nxt, v_nxt), reqs = _exchange([k_cur, v_cur], nxt, prv, group)
        kh = k_cur if layout == "zigzag" else k_cur.unsqueeze(0)
        vh = v_cur if layout == "zigzag" else v_cur.unsqueeze(0)
        for a, b, kind in pairs:
            o_p, lse_p = local_fwd(qh[a], kh[b], vh[b], kind == "causal")
            merge(o_acc[a], lse_acc[a], o_p, lse_p, first[a])
            first[a] = False
        for r in reqs:
            r.wait()
        if s + 1 < world:
            k_cur, v_cur = k_nxt, v_nxt
    o = _finish_rows(finish, o_acc)
    if layout == "zigzag":
        return o, lse_acc
    return o[0], lse_acc[0]


def ring_attn_bwd(q, k, v, o, do, lse, batch, scale=None, causal=False, group=None, local_bwd=None, finish=None,
                  acc_dtype=torch.float32, layout="contiguous"):
    """Gradients of the ring forward for this rank: dq for its query rows, dk, dv for its
    K/V rows, in the layout of q, k, v (contiguous: [B n, H, d]; zig-zag: [2, B c, H, d]).
    ``o`` / ``lse`` are this rank's rows of the full forward (``ring_attn_fwd``'s outputs),
    ``do`` their upstream gradient.  ``local_bwd(q, k, v, o, do, lse, causal, dq_acc,
    dk_acc, dv_acc)`` adds one (query rows, K/V block) pair's gradients into the
    ``acc_dtype`` accumulators; it defaults to the library's attn_bwd_accumulate.
    ``finish(acc) -> tensor`` turns an accumulator into the result; by default the
    library's attn_merge_finish (float32 to bf16)."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {LAYOUTS}")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if local_bwd is None:
        def local_bwd(q_, k_, v_, o_, do_, lse_, c_, dq_a, dk_a, dv_a):
            attn_bwd_accumulate(q_, k_, v_, o_, do_, lse_, dq_a, dk_a, dv_a, scale=scale, causal=c_, batch=batch)
    if finish is None:
        finish = attn_merge_finish
    nxt, prv = _peers(group, world, rank)
    zz = layout == "zigzag"
    q, o, do, lse = (t.contiguous() for t in (q, o, do, lse))
    qh, oh, doh = (t if zz else t.unsqueeze(0) for t in (q, o, do))
    lseh = lse if zz else lse.unsqueeze(0)
    if zz:
        hops = zigzag_schedule(rank, world, causal)
    else:
        hops = [[(0, 0, kind)] if kind is not None else [] for _, kind in ring_schedule(rank, world, causal)]
    dq_acc = torch.zeros(qh.shape, dtype=acc_dtype, device=q.device)
    k_cur, v_cur = k.contiguous(), v.contiguous()
    dk_cur = torch.zeros(k.shape, dtype=acc_dtype, device=k.device)
    dv_cur = torch.zeros(v.shape, dtype=acc_dtype, device=v.device)
    for s, pairs in enumerate(hops):
        kv_reqs = []
        if s + 1 < world:
            # the next hop's block moves while this hop is computed
            (k_nxt, v_nxt), kv_reqs = _exchange([k_cur, v_cur], nxt, prv, group)
        kh, vh, dkh, dvh = (t if zz else t.unsqueeze(0) for t in (k_cur, v_cur, dk_cur, dv_cur))
        for a, b, kind in pairs:
            local_bwd(qh[a], kh[b], vh[b], oh[a], doh[a], lseh[a], kind == "causal", dq_acc[a], dkh[b], dvh[b])
        # the block's gradients so far go on with it (after the last hop: to its owner)
        g_reqs = []
        if world > 1:
            (dk_in, dv_in), g_reqs = _exchange([dk_cur, dv_cur], nxt, prv, group)
        for r in kv_reqs + g_reqs:
            r.wait()
        if world > 1:
            dk_cur, dv_cur = dk_in, dv_in
        if s + 1 < world:
            k_cur, v_cur = k_nxt, v_nxt
    dq = _finish_rows(finish, dq_acc)
    if zz:
        return dq, _finish_rows(finish, dk_cur), _finish_rows(finish, dv_cur)
    return dq[0], finish(dk_cur), finish(dv_cur)
