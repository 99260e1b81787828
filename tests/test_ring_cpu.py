"""The ring-attention drivers over a real multi-process group (gloo on CPU).

Each rank holds one chunk of every sequence and runs ``ring_attn_fwd`` and
``ring_attn_bwd``, the same drivers the GPUs run, with their compute steps swapped for
CPU stand-ins (the local attention and its backward from the fp64 oracle, the merge in
float64) -- the schedule, the masks of every hop, the point-to-point passing of the K/V
blocks and of their travelling dK / dV are what is under test here.  The rows gathered
from all ranks must equal the oracle's forward and gradient over the whole sequences.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from io_aware_exact_qk_b200.ring import ring_schedule, zigzag_schedule, zigzag_shard, zigzag_unshard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _local_oracle(batch, scale):
    def f(q, k, v, causal):
        n = q.shape[0] // batch
        cu = np.arange(batch + 1, dtype=np.int32) * n
        o, lse = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), cu, scale=scale, causal=causal, threads=1)
        return torch.from_numpy(o), torch.from_numpy(lse)
    return f


def _merge64(o_acc, lse_acc, o_p, lse_p, first):
    o_p, lse_p = o_p.double(), lse_p.double()
    if first:
        o_acc.copy_(o_p)
        lse_acc.copy_(lse_p)
        return
    la, lp = lse_acc.clone(), lse_p
    m = torch.maximum(la, lp)
    wa = torch.where(la == -np.inf, 0.0, torch.exp(la - m))
    wp = torch.where(lp == -np.inf, 0.0, torch.exp(lp - m))
    s = wa + wp
    # [hq, T] weights -> [T, hq, 1]
    o_acc.mul_((wa / s).T[:, :, None]).add_(o_p * (wp / s).T[:, :, None])
    lse_acc.copy_(m + torch.log(s))


def _local_oracle_bwd(batch, scale):
    def f(q, k, v, o, do, lse, causal, dq_acc, dk_acc, dv_acc):
        n = q.shape[0] // batch
        cu = np.arange(batch + 1, dtype=np.int32) * n
        dq, dk, dv, _, _ = oracle.attn_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), cu, scale=scale,
                                           causal=causal, threads=1, o=o.numpy(), lse=lse.numpy())
        for acc, g in ((dq_acc, dq), (dk_acc, dk), (dv_acc, dv)):
            acc.add_(torch.from_numpy(g))
    return f


def _full_inputs(batch, N, hq, hkv, d):
    g = torch.Generator().manual_seed(77)
    q = torch.randn(batch, N, hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(batch, N, hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(batch, N, hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(batch, N, hq, d, generator=g, dtype=torch.float64)
    return q, k, v, do


def _worker(rank, world, port, batch, n, hq, hkv, d, causal, out, layout="contiguous"):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        from io_aware_exact_qk_b200.ring import ring_attn_bwd, ring_attn_fwd
        q, k, v, do = _full_inputs(batch, world * n, hq, hkv, d)
        if layout == "zigzag":
            qc, kc, vc, doc = (zigzag_shard(t.reshape(-1, t.shape[2], d), batch, rank, world) for t in (q, k, v, do))
        else:
            mine = slice(rank * n, (rank + 1) * n)
            qc, kc, vc, doc = (t[:, mine].reshape(batch * n, t.shape[2], d).contiguous() for t in (q, k, v, do))
        scale = 1.0 / np.sqrt(d)
        o, lse = ring_attn_fwd(qc, kc, vc, batch, scale=scale, causal=causal, local_fwd=_local_oracle(batch, scale),
                               merge=_merge64, finish=lambda oa: oa, acc_dtype=torch.float64, layout=layout)
        dq, dk, dv = ring_attn_bwd(qc, kc, vc, o, doc, lse, batch, scale=scale, causal=causal,
                                   local_bwd=_local_oracle_bwd(batch, scale), finish=lambda a: a,
                                   acc_dtype=torch.float64, layout=layout)
        out[rank] = (o.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_forward_and_backward_equal_full_attention(world, causal):
    batch, n, hq, hkv, d = 2, 5, 4, 2, 8
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as man:
        out = man.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, batch, n, hq, hkv, d, causal, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    N = world * n
    q, k, v, do = _full_inputs(batch, N, hq, hkv, d)
    cu = np.arange(batch + 1, dtype=np.int32) * N
    dq_ref, dk_ref, dv_ref, o_ref, lse_ref = oracle.attn_bwd(
        q.reshape(-1, hq, d).numpy(), k.reshape(-1, hkv, d).numpy(), v.reshape(-1, hkv, d).numpy(),
        do.reshape(-1, hq, d).numpy(), cu, causal=causal)
    o_ref, dq_ref = o_ref.reshape(batch, N, hq, d), dq_ref.reshape(batch, N, hq, d)
    dk_ref, dv_ref = dk_ref.reshape(batch, N, hkv, d), dv_ref.reshape(batch, N, hkv, d)
    lse_ref = lse_ref.reshape(hq, batch, N)
    for r in range(world):
        o, lse, dq, dk, dv = res[r]
        mine = slice(r * n, (r + 1) * n)
        np.testing.assert_allclose(o.reshape(batch, n, hq, d), o_ref[:, mine], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse.reshape(hq, batch, n), lse_ref[:, :, mine], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dq.reshape(batch, n, hq, d), dq_ref[:, mine], rtol=0, atol=1e-10)
        np.testing.assert_allclose(dk.reshape(batch, n, hkv, d), dk_ref[:, mine], rtol=0, atol=1e-10)
        np.testing.assert_allclose(dv.reshape(batch, n, hkv, d), dv_ref[:, mine], rtol=0, atol=1e-10)


def test_ring_schedule_visits_every_block_once():
    for world in (1, 2, 5):
        for causal in (False, True):
            for r in range(world):
                hops = ring_schedule(r, world, causal)
                assert sorted(j for j, _ in hops) == list(range(world))
                assert hops[0] == (r, "causal" if causal else "full")   # own block first
                for j, kind in hops:
                    assert kind == ("full" if not causal or j < r else ("causal" if j == r else None))


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_ring_equals_full_attention(world, causal):
    """The zig-zag layout (rank r holds chunks r and 2W-1-r of every sequence): the rows
    of all ranks, put back in sequence order, equal the oracle's forward and gradient."""
    batch, c, hq, hkv, d = 2, 3, 4, 2, 8
    N = 2 * world * c
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as man:
        out = man.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, batch, N // world, hq, hkv, d, causal, out,
                                                   "zigzag"))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    q, k, v, do = _full_inputs(batch, N, hq, hkv, d)
    cu = np.arange(batch + 1, dtype=np.int32) * N
    dq_ref, dk_ref, dv_ref, o_ref, lse_ref = oracle.attn_bwd(
        q.reshape(-1, hq, d).numpy(), k.reshape(-1, hkv, d).numpy(), v.reshape(-1, hkv, d).numpy(),
        do.reshape(-1, hq, d).numpy(), cu, causal=causal)

    def whole(i):
        return zigzag_unshard([torch.from_numpy(res[r][i]) for r in range(world)], batch).numpy()

    lse = zigzag_unshard([torch.from_numpy(res[r][1]).transpose(1, 2) for r in range(world)], batch).T.numpy()
    np.testing.assert_allclose(whole(0), o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(whole(2), dq_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(whole(3), dk_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(whole(4), dv_ref, rtol=0, atol=1e-10)


def test_zigzag_schedule_balances_the_causal_ring():
    """Every (query chunk, K/V chunk) pair a rank can see is visited exactly once, with the
    right mask, and under the causal mask every rank has 2W - 1 full and 2 diagonal blocks."""
    for world in (1, 2, 3, 5):
        for causal in (False, True):
            for r in range(world):
                hops = zigzag_schedule(r, world, causal)
                assert len(hops) == world
                seen = []
                for s, pairs in enumerate(hops):
                    j = (r - s) % world
                    for a, b, kind in pairs:
                        qc = (r, 2 * world - 1 - r)[a]
                        kc = (j, 2 * world - 1 - j)[b]
                        assert kind == ("full" if not causal or kc < qc else "causal"), (world, r, s, a, b)
                        seen.append((qc, kc))
                want = [(qc, kc) for qc in (r, 2 * world - 1 - r) for kc in range(2 * world)
                        if not causal or kc <= qc]
                assert sorted(seen) == sorted(want)
                if causal:
                    kinds = [k for pairs in hops for _, _, k in pairs]
                    assert kinds.count("full") == 2 * world - 1 and kinds.count("causal") == 2


def test_zigzag_shard_round_trip():
    x = torch.arange(2 * 12 * 3 * 4, dtype=torch.float64).reshape(2 * 12, 3, 4)
    for world in (1, 2, 3, 6):
        parts = [zigzag_shard(x, 2, r, world) for r in range(world)]
        assert all(p.shape == (2, 2 * 12 // (2 * world), 3, 4) for p in parts)
        assert torch.equal(zigzag_unshard(parts, 2), x)
        c = 12 // (2 * world)
        assert torch.equal(parts[0][0][:c], x[:c])                     # rank 0 half 0: chunk 0 of sequence 0
        assert torch.equal(parts[0][1][:c], x[12 - c:12])              # rank 0 half 1: the last chunk
