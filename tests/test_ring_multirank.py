"""Ring attention's schedule and exchange on CPU: gloo ranks (world 2 and 3)
run ``ring_attention_fwd`` / ``ring_attention_bwd`` with the fp64 oracle
standing in for the per-chunk device steps, so the test covers the ring's
host logic (who holds which chunk when, what is skipped under causal masking,
the travelling dK/dV accumulators) with real point-to-point messages; the
result must equal full attention over the whole sequence."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_84_b200.ring import ring_schedule


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """Per-chunk steps computed by the fp64 oracle on CPU tensors."""

    def partial_fwd(self, q, k, v, scale, causal):
        from oracle import attn_fwd_ref
        o, lse = attn_fwd_ref(q.numpy(), k.numpy(), v.numpy(), scale, causal)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o, lse, o_part, lse_part):
        from oracle import merge_partials_ref
        mo, ml = merge_partials_ref(o.numpy(), lse.numpy(), o_part.numpy(), lse_part.numpy())
        o.copy_(torch.from_numpy(mo))
        lse.copy_(torch.from_numpy(ml))

    def partial_bwd(self, q, k, v, o, do, lse, scale, causal, out):
        from oracle import attn_bwd_partial_ref
        return tuple(torch.from_numpy(x) for x in attn_bwd_partial_ref(
            q.numpy(), k.numpy(), v.numpy(), o.numpy(), do.numpy(), lse.numpy(), scale, causal))

    def bwd_buffers(self, q, k):
        return None

    def zeros_acc(self, like):
        return torch.zeros(like.shape, dtype=torch.float64)

    def accumulate(self, acc, src):
        acc += src

    def to_dtype(self, x, like):
        return x.clone()


def _full_inputs(world, n, causal):
    g = torch.Generator().manual_seed(1000 + world + 10 * causal)
    return [torch.randn(1, 2, world * n, 4, generator=g, dtype=torch.float64) for _ in range(4)]


def _worker(rank, world, port, n, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from exact_io_aware_84_b200.ring import ring_attention_bwd, ring_attention_fwd
        q, k, v, do = (x[:, :, rank * n:(rank + 1) * n].contiguous() for x in _full_inputs(world, n, causal))
        ops = OracleOps()
        o, lse, o32 = ring_attention_fwd(q, k, v, scale=0.6, causal=causal, ops=ops)
        dq, dk, dv = ring_attention_bwd(q, k, v, o32, do, lse, scale=0.6, causal=causal, ops=ops)
        out[rank] = tuple(t.numpy() for t in (o, lse, dq, dk, dv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_over_gloo_equals_full_attention(world, causal):
    from oracle import attn_bwd_ref, attn_fwd_ref
    n = 5
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, n, causal, out), nprocs=world, join=True)
    q, k, v, do = (x.numpy() for x in _full_inputs(world, n, causal))
    o_ref, lse_ref = attn_fwd_ref(q, k, v, 0.6, causal)
    dq_ref, dk_ref, dv_ref = attn_bwd_ref(q, k, v, do, 0.6, causal)
    cat = lambda i, ax: np.concatenate([out[r][i] for r in range(world)], axis=ax)
    np.testing.assert_allclose(cat(0, -2), o_ref, atol=1e-12)
    np.testing.assert_allclose(cat(1, -1), lse_ref, atol=1e-12)
    np.testing.assert_allclose(cat(2, -2), dq_ref, atol=1e-12)
    np.testing.assert_allclose(cat(3, -2), dk_ref, atol=1e-12)
    np.testing.assert_allclose(cat(4, -2), dv_ref, atol=1e-12)


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
def test_ring_schedule_covers_every_pair_once(world):
    for causal in (False, True):
        seen = set()
        for r in range(world):
            sched = ring_schedule(r, world, causal)
            assert [s for s, *_ in sched] == list(range(world))
            assert sched[0][1] == r and sched[0][2]           # own chunk first, always computed
            for step, src, computed, diag in sched:
                assert src == (r - step) % world
                assert diag == (causal and src == r)
                if computed:
                    assert (r, src) not in seen
                    seen.add((r, src))
        want = {(r, s) for r in range(world) for s in range(world) if not causal or s <= r}
        assert seen == want


def test_ring_schedule_rejects_bad_rank():
    with pytest.raises(ValueError):
        ring_schedule(3, 3, False)


@pytest.mark.parametrize("causal", [False, True])
def test_thread_ring_equals_full_attention(causal):
    # the in-process ring (one host thread per rank) with the oracle as the
    # chunk steps, on CPU tensors
    from oracle import attn_bwd_ref, attn_fwd_ref

    from exact_io_aware_84_b200.ring import ThreadRing, ring_attention_bwd, ring_attention_fwd
    world, n = 4, 3
    q, k, v, do = _full_inputs(world, n, causal)
    ring = ThreadRing(world)
    out = [None] * world

    def run(r):
        sl = slice(r * n, (r + 1) * n)
        lq, lk, lv, ldo = (x[:, :, sl].contiguous() for x in (q, k, v, do))
        comm = ring.comm(r)
        o, lse, o32 = ring_attention_fwd(lq, lk, lv, scale=0.6, causal=causal, ops=OracleOps(), comm=comm)
        out[r] = (o, lse) + ring_attention_bwd(lq, lk, lv, o32, ldo, lse, scale=0.6, causal=causal,
                                               ops=OracleOps(), comm=comm)

    ring.run(run)
    o_ref, lse_ref = attn_fwd_ref(q.numpy(), k.numpy(), v.numpy(), 0.6, causal)
    grads = attn_bwd_ref(q.numpy(), k.numpy(), v.numpy(), do.numpy(), 0.6, causal)
    cat = lambda i, ax: np.concatenate([out[r][i].numpy() for r in range(world)], axis=ax)
    np.testing.assert_allclose(cat(0, -2), o_ref, atol=1e-12)
    np.testing.assert_allclose(cat(1, -1), lse_ref, atol=1e-12)
    for i, ref in zip((2, 3, 4), grads):
        np.testing.assert_allclose(cat(i, -2), ref, atol=1e-12)


def test_thread_ring_reraises_a_rank_error():
    from exact_io_aware_84_b200.ring import ThreadRing
    ring = ThreadRing(3, timeout=10)

    def run(r):
        if r == 1:
            raise RuntimeError("rank 1 failed")
        ring.comm(r).exchange([torch.zeros(2)], [torch.zeros(2)])

    with pytest.raises(RuntimeError, match="rank 1 failed"):
        ring.run(run)
