"""Ring attention's GPU arithmetic: the forward and backward on chunk pairs and the merge
kernels.

This run has one GPU, so the ranks of the ring are emulated in turn in one process: for
every rank the hops of ``ring_schedule`` are executed with the library's kernels
(attn_fwd on the (query chunk, K/V chunk) pair, attn_merge_partial, attn_merge_finish),
and the rows of all ranks together must match the fp64 oracle over the whole sequences
with the forward's tolerances; the backward's per-hop gradients, summed the way the
travelling dK / dV are, must match the oracle's gradient at the backward's tolerance.
The point-to-point passing of the blocks between real ranks is covered by the gloo test
on the CPU; the ring functions themselves run here as a one-rank NCCL group.
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
import oracle
from io_aware_exact_qk_b200.ring import (ring_attn_bwd, ring_attn_fwd, ring_schedule, zigzag_schedule, zigzag_shard,
                                         zigzag_unshard)
from tests import parity

pytestmark = pytest.mark.gpu


def _inputs(batch, N, hq, hkv, d, seed):
    w = W.custom("ring", [N] * batch, hq, hkv, d, False, seed)
    q, k, v, _, cu = W.make_inputs(w, with_grad=False)
    return w, q, k, v, cu


def _chunks(t, batch, N, world):
    n = N // world
    t = t.reshape(batch, N, *t.shape[1:])
    return [t[:, r * n:(r + 1) * n].reshape(batch * n, *t.shape[2:]).contiguous().cuda() for r in range(world)]


@pytest.mark.parametrize("world,causal,d", [(2, False, 128), (4, True, 128), (3, True, 64), (5, False, 32)])
def test_emulated_ring_matches_full_attention(world, causal, d):
    batch, n, hq, hkv = 2, 256 if d == 128 else 200, 8, 2
    N = world * n
    w, q, k, v, cu = _inputs(batch, N, hq, hkv, d, 3100 + world)
    qs, ks, vs = (_chunks(t, batch, N, world) for t in (q, k, v))
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, cu.numpy(), scale=w.scale, causal=causal)
    o_ref = o_ref.reshape(batch, N, hq, d)
    lse_ref = lse_ref.reshape(hq, batch, N)
    for r in range(world):
        o_acc = torch.empty(batch * n, hq, d, dtype=torch.float32, device="cuda")
        lse_acc = torch.empty(hq, batch * n, dtype=torch.float32, device="cuda")
        first = True
        for j, kind in ring_schedule(r, world, causal):
            if kind is None:
                continue
            o_p, lse_p = attn.attn_fwd(qs[r], ks[j], vs[j], scale=w.scale, causal=kind == "causal", batch=batch)
            attn.attn_merge_partial(o_acc, lse_acc, o_p, lse_p, first=first)
            first = False
        o = attn.attn_merge_finish(o_acc)
        attn.attn_get_device_error()
        mine = slice(r * n, (r + 1) * n)
        parity.check_fwd_bf16(parity.to_np(o).reshape(batch, n, hq, d), parity.to_np(lse_acc).reshape(hq, batch, n),
                              o_ref[:, mine], lse_ref[:, :, mine], tag=f"rank {r}")


@pytest.mark.parametrize("world,causal,d", [(2, True, 128), (3, False, 64), (4, True, 32)])
def test_emulated_ring_backward_matches_the_gradient(world, causal, d):
    """Every rank's hops run attn_bwd_accumulate on its (query chunk, K/V block) pairs with
    its rows of the full forward's O and LSE, adding into float32 sums: dQ over the rank's
    hops, dK / dV of a block over the ranks it visits (as ring_attn_bwd does).  The stored O
    (bf16) and LSE (fp32) are the oracle's forward, given to the oracle's backward as well
    (the backward as a function of its inputs)."""
    batch, n, hq, hkv = 2, 256 if d == 128 else 200, 8, 2
    N = world * n
    w = W.custom("ring-bwd", [N] * batch, hq, hkv, d, causal, 3300 + world)
    q, k, v, do, cu = W.make_inputs(w)
    o_or, lse_or = oracle.attn_fwd(q, k, v, cu.numpy(), scale=w.scale, causal=causal)
    o_st = torch.from_numpy(o_or).to(torch.bfloat16)
    lse_st = torch.from_numpy(lse_or).to(torch.float32)
    qs, ks, vs, dos, os_ = (_chunks(t, batch, N, world) for t in (q, k, v, do, o_st))
    lse_b = lse_st.reshape(hq, batch, N)
    lses = [lse_b[:, :, r * n:(r + 1) * n].reshape(hq, batch * n).contiguous().cuda() for r in range(world)]
    dq = [torch.zeros(batch * n, hq, d, device="cuda") for _ in range(world)]
    dk = [torch.zeros(batch * n, hkv, d, device="cuda") for _ in range(world)]
    dv = [torch.zeros(batch * n, hkv, d, device="cuda") for _ in range(world)]
    for r in range(world):
        for j, kind in ring_schedule(r, world, causal):
            if kind is None:
                continue
            attn.attn_bwd_accumulate(qs[r], ks[j], vs[j], os_[r], dos[r], lses[r], dq[r], dk[j], dv[j],
                                     scale=w.scale, causal=kind == "causal", batch=batch)
    attn.attn_get_device_error()
    dq_r, dk_r, dv_r, _, _ = oracle.attn_bwd(q, k, v, do, cu.numpy(), scale=w.scale, causal=causal,
                                             o=o_st.double().numpy(), lse=lse_st.double().numpy())

    def whole(parts, h):
        return torch.stack([p.cpu().reshape(batch, n, h, d) for p in parts], dim=1).reshape(batch * N, h, d)

    parity.check_grads_bf16((whole(dq, hq), whole(dk, hkv), whole(dv, hkv)), (dq_r, dk_r, dv_r),
                            tag=f"ring bwd W={world}")


@pytest.mark.parametrize("world,d", [(2, 128), (3, 64), (4, 128)])
def test_emulated_zigzag_ring_causal(world, d):
    """The zig-zag layout under the causal mask, ranks emulated in turn with the library's
    kernels: each rank's hops of ``zigzag_schedule`` (attn_fwd on each (query half, K/V
    half) pair, merged per query half), then its backward pairs adding into float32 sums
    (dK / dV into the visiting block's halves); all rows against the oracle."""
    batch, c, hq, hkv = 2, 128, 8, 2
    N = 2 * world * c
    w = W.custom("zz", [N] * batch, hq, hkv, d, True, 3400 + world)
    q, k, v, do, cu = W.make_inputs(w)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, cu.numpy(), scale=w.scale, causal=True)
    shard = [[zigzag_shard(t, batch, r, world).cuda() for r in range(world)] for t in (q, k, v, do)]
    qs, ks, vs, dos = shard
    os_, lses = [], []
    for r in range(world):
        o_acc = torch.empty(2, batch * c, hq, d, device="cuda")
        lse_acc = torch.empty(2, hq, batch * c, device="cuda")
        first = [True, True]
        for s, pairs in enumerate(zigzag_schedule(r, world, True)):
            j = (r - s) % world
            for a, b, kind in pairs:
                o_p, lse_p = attn.attn_fwd(qs[r][a], ks[j][b], vs[j][b], scale=w.scale, causal=kind == "causal",
                                           batch=batch)
                attn.attn_merge_partial(o_acc[a], lse_acc[a], o_p, lse_p, first=first[a])
                first[a] = False
        os_.append(attn.attn_merge_finish(o_acc.reshape(-1, hq, d)).reshape(2, batch * c, hq, d))
        lses.append(lse_acc)
    attn.attn_get_device_error()
    o = zigzag_unshard([t.cpu() for t in os_], batch)
    lse = zigzag_unshard([t.cpu().transpose(1, 2) for t in lses], batch).T
    parity.check_fwd_bf16(parity.to_np(o), parity.to_np(lse), o_ref, lse_ref, tag=f"zigzag W={world}")
    # backward on the device forward's O and LSE, as a caller of ring_attn_bwd would
    dq = [torch.zeros(2, batch * c, hq, d, device="cuda") for _ in range(world)]
    dk = [torch.zeros(2, batch * c, hkv, d, device="cuda") for _ in range(world)]
    dv = [torch.zeros(2, batch * c, hkv, d, device="cuda") for _ in range(world)]
    for r in range(world):
        for s, pairs in enumerate(zigzag_schedule(r, world, True)):
            j = (r - s) % world
            for a, b, kind in pairs:
                attn.attn_bwd_accumulate(qs[r][a], ks[j][b], vs[j][b], os_[r][a], dos[r][a],
                                         lses[r][a].contiguous(), dq[r][a], dk[j][b], dv[j][b], scale=w.scale,
                                         causal=kind == "causal", batch=batch)
    attn.attn_get_device_error()
    ref = oracle.attn_bwd(q, k, v, do, cu.numpy(), scale=w.scale, causal=True)
    got = tuple(zigzag_unshard([t.cpu() for t in g], batch) for g in (dq, dk, dv))
    parity.check_grads_bf16(got, ref[:3], tag=f"zigzag bwd W={world}")


def test_merge_kernel_edge_cases():
    T, hq, d = 37, 4, 128
    g = torch.Generator().manual_seed(5)
    o_acc = torch.randn(T, hq, d, generator=g).cuda()
    lse_acc = torch.randn(hq, T, generator=g).cuda()
    o_p = torch.randn(T, hq, d, generator=g).to(torch.bfloat16).cuda()
    # a partial without visible keys leaves the accumulator as it is
    before = (o_acc.clone(), lse_acc.clone())
    attn.attn_merge_partial(o_acc, lse_acc, o_p, torch.full((hq, T), -np.inf, device="cuda"))
    torch.testing.assert_close(o_acc, before[0], rtol=0, atol=0)
    torch.testing.assert_close(lse_acc, before[1], rtol=0, atol=0)
    # first=True starts from the partial; equal LSEs average the two partials
    lse_p = torch.randn(hq, T, generator=g).cuda()
    attn.attn_merge_partial(o_acc, lse_acc, o_p, lse_p, first=True)
    torch.testing.assert_close(o_acc, o_p.float(), rtol=0, atol=0)
    torch.testing.assert_close(lse_acc, lse_p, rtol=0, atol=0)
    o_q = torch.randn(T, hq, d, generator=g).to(torch.bfloat16).cuda()
    attn.attn_merge_partial(o_acc, lse_acc, o_q, lse_p)
    torch.testing.assert_close(o_acc, (o_p.float() + o_q.float()) / 2, rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(lse_acc, lse_p + float(np.log(2.0)), rtol=1e-6, atol=1e-6)
    assert torch.equal(attn.attn_merge_finish(o_acc), o_acc.to(torch.bfloat16))
    attn.attn_get_device_error()


def test_driver_as_a_one_rank_nccl_group():
    """The ring functions' own code path (defaults = the library's kernels) on one rank."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        batch, N, hq, hkv, d = 2, 384, 8, 4, 128
        w, q, k, v, cu = _inputs(batch, N, hq, hkv, d, 3200)
        o, lse = ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), batch, scale=w.scale, causal=True)
        attn.attn_get_device_error()
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, cu.numpy(), scale=w.scale, causal=True)
        parity.check_fwd_bf16(o, lse, o_ref, lse_ref, tag="one-rank ring")
        # the backward driver on the oracle's stored forward
        do = W.make_inputs(W.custom("ring-do", [N] * batch, hq, hkv, d, True, 3201))[3]
        o_st = torch.from_numpy(o_ref).to(torch.bfloat16)
        lse_st = torch.from_numpy(lse_ref).to(torch.float32)
        dq, dk, dv = ring_attn_bwd(q.cuda(), k.cuda(), v.cuda(), o_st.cuda(), do.cuda(), lse_st.cuda(), batch,
                                   scale=w.scale, causal=True)
        attn.attn_get_device_error()
        dq_r, dk_r, dv_r, _, _ = oracle.attn_bwd(q, k, v, do, cu.numpy(), scale=w.scale, causal=True,
                                                 o=o_st.double().numpy(), lse=lse_st.double().numpy())
        parity.check_grads_bf16((dq, dk, dv), (dq_r, dk_r, dv_r), tag="one-rank ring bwd")
        # the zig-zag layout through the same drivers (one rank: chunks 0 and 1)
        qz, kz, vz, oz, doz = (zigzag_shard(t, batch, 0, 1).cuda() for t in (q, k, v, o_st, do))
        o2, lse2 = ring_attn_fwd(qz, kz, vz, batch, scale=w.scale, causal=True, layout="zigzag")
        attn.attn_get_device_error()
        o2 = zigzag_unshard([o2.cpu()], batch)
        lse2 = zigzag_unshard([lse2.cpu().transpose(1, 2)], batch).T
        parity.check_fwd_bf16(o2, lse2, o_ref, lse_ref, tag="one-rank zigzag ring")
        lsez = zigzag_shard(lse_st.T.contiguous(), batch, 0, 1).transpose(1, 2).contiguous().cuda()
        dq2, dk2, dv2 = ring_attn_bwd(qz, kz, vz, oz, doz, lsez, batch, scale=w.scale, causal=True, layout="zigzag")
        attn.attn_get_device_error()
        got = tuple(zigzag_unshard([t.cpu()], batch) for t in (dq2, dk2, dv2))
        parity.check_grads_bf16(got, (dq_r, dk_r, dv_r), tag="one-rank zigzag ring bwd")
    finally:
        dist.destroy_process_group()
