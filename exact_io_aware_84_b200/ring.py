"""Ring attention (context parallelism) over a process group.

The sequence is split into equal, contiguous chunks, one per rank; rank r
holds query, key and value chunk r ([B, H, n, d] each, n = N / world).  Each
rank keeps its query chunk and computes attention block by block against the
key/value chunks as they pass around the ring (ultralytics glossary "Flash
Attention", "Flash Attention and related terms", ring attention): at step s
rank r holds the chunk that started on rank (r - s) mod world, computes the
partial result of its queries over those keys, and meanwhile sends the chunk
on to rank r + 1 and receives the next one from rank r - 1.

Partial results over disjoint key sets combine by the online-softmax
recurrence taken one chunk at a time (marketmaker.cc "Online softmax
recurrence"): LSE = ln(e^{LSE_a} + e^{LSE_b}), O = e^{LSE_a - LSE} O_a +
e^{LSE_b - LSE} O_b.  With causal masking a chunk after the query chunk has
no visible key and is skipped; the query chunk's own key chunk is computed
with the causal mask; earlier chunks in full.

Backward: the same ring, now carrying each key/value chunk together with fp32
accumulators of its dK and dV.  At every step the rank adds its partial
gradients (computed from the merged O and LSE of its rows: P = exp(S - LSE),
D = rowsum(dO o O)) to the travelling accumulators and sends them on; after
``world`` hops every chunk's accumulators are back on its own rank.  dQ is
summed locally.

Everything on the device runs in libfa's kernels (fa_fwd / fa_bwd on the
chunk pair, fa_merge, fa_grad_accumulate, fa_convert); the exchange is
torch.distributed point-to-point (NCCL over NVLink on GPUs), issued before
each step's compute so that the transfer overlaps it.

``ops`` and ``comm`` are parameters so that the schedule can run with other
compute or transport (the CPU tests use them); by default they are the CUDA
kernels and the process group.
"""

from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

__all__ = ["ring_schedule", "RingComm", "ThreadRing", "CudaChunkOps", "ring_attention_fwd", "ring_attention_bwd"]


def ring_schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, int, bool, bool]]:
    """(step, source chunk, computed, chunk-causal) for every step of ``rank``.

    At step s the rank holds the key/value chunk of rank (rank - s) mod world.
    With causal masking a chunk after the rank's own has no key at or before
    any of its queries (not computed); its own chunk is causal; earlier
    chunks are attended in full.
    """
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a ring of {world}")
    out = []
    for step in range(world):
        src = (rank - step) % world
        computed = not (causal and src > rank)
        out.append((step, src, computed, causal and src == rank))
    return out


class RingComm:
    """Send to the next rank and receive from the previous one, over a
    torch.distributed process group (NCCL for CUDA tensors, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist

        self._dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        to_global = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
        self.next = to_global((self.rank + 1) % self.world)
        self.prev = to_global((self.rank - 1) % self.world)

    def exchange(self, send: Sequence, recv: Sequence):
        """Start sending ``send`` to the next rank and receiving ``recv`` from
        the previous one; returns handles for ``wait``."""
        dist = self._dist
        ops = [dist.P2POp(dist.isend, t, self.next, self.group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, self.prev, self.group) for t in recv]
        return dist.batch_isend_irecv(ops)

    @staticmethod
    def wait(handles):
        for h in handles or ():
            h.wait()


class ThreadRing:
    """A ring of ``world`` ranks emulated by host threads of one process on
    one device (one thread per rank, all launching on the same stream).
    ``comm(rank)`` gives rank ``rank`` its end: ``exchange`` posts the
    tensors to send, waits for every rank at a barrier, copies the
    predecessor's tensors into the receive buffers (device copies on the
    shared stream, so they run after the kernels that produced them) and
    meets the others at a second barrier before anyone may overwrite what it
    posted.  The device never waits on anything: the ranks' kernels run one
    after another."""

    def __init__(self, world: int, timeout: float = 120.0):
        import threading

        self.world = world
        self.slots = [None] * world
        self.barrier = threading.Barrier(world, timeout=timeout)

    def comm(self, rank: int):
        return _ThreadComm(self, rank)

    def run(self, fn):
        """Run ``fn(rank)`` for every rank on its own thread; re-raise the
        first error (breaking the barrier, so that the other ranks stop)."""
        import threading

        errs = []

        def body(r):
            try:
                fn(r)
            except BaseException as e:  # noqa: BLE001 - re-raised below
                errs.append(e)
                self.barrier.abort()

        threads = [threading.Thread(target=body, args=(r,)) for r in range(self.world)]
        for t in threads:
            t.start()
        for t in threads:
            t.join()
        if errs:
            raise errs[0]


class _ThreadComm:
    def __init__(self, ring: ThreadRing, rank: int):
        self.ring, self.rank, self.world = ring, rank, ring.world

    def exchange(self, send: Sequence, recv: Sequence):
        ring = self.ring
        ring.slots[self.rank] = list(send)
        ring.barrier.wait()
        for r, s in zip(recv, ring.slots[(self.rank - 1) % self.world]):
            r.copy_(s)
        ring.barrier.wait()
        return None

    @staticmethod
    def wait(handles):
        pass


class CudaChunkOps:
    """The device steps of the ring, all in libfa."""

    def __init__(self):
        from . import load_library

        load_library()  # fail now, loudly, if the CUDA library is missing

    def partial_fwd(self, q, k, v, scale, causal):
        from . import fa_fwd

        return fa_fwd(q, k, v, scale=scale, causal=causal, o_fp32=True)

    def merge(self, o, lse, o_part, lse_part):
        from . import fa_merge

        fa_merge(o, lse, o_part, lse_part)

    def partial_bwd(self, q, k, v, o, do, lse, scale, causal, out):
        from . import fa_bwd

        dq, dk, dv, ws = out
        fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, scale=scale, causal=causal)
        return dq, dk, dv

    def bwd_buffers(self, q, k):
        import torch

        from . import fa_bwd_workspace_size

        B, H, n, d = q.shape
        ws = torch.empty(fa_bwd_workspace_size(B, H, n, d), dtype=torch.uint8, device=q.device)
        return torch.empty_like(q), torch.empty_like(k), torch.empty_like(k), ws

    def zeros_acc(self, like):
        import torch

        return torch.zeros(like.shape, dtype=torch.float32, device=like.device)

    def accumulate(self, acc, src):
        from . import fa_grad_accumulate

        fa_grad_accumulate(acc, src)

    def to_dtype(self, x32, like):
        from . import fa_convert

        return fa_convert(x32, like.dtype)


def _check(q, k, v):
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("ring attention takes local [B, H, n, d] chunks of equal shape")


def ring_attention_fwd(q, k, v, scale: Optional[float] = None, causal: bool = False, group=None,
                       ops=None, comm=None):
    """Forward of this rank's query chunk over the whole sequence.

    Returns (O in the input type, LSE fp32 [B, H, n], O fp32) -- the fp32 O
    and the LSE are what ``ring_attention_bwd`` needs.
    """
    import torch

    _check(q, k, v)
    ops = ops or CudaChunkOps()
    comm = comm or RingComm(group)
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    sched = ring_schedule(comm.rank, comm.world, causal)
    cur = (k, v)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    o32 = lse = None
    for step, _src, computed, diag in sched:
        nxt = bufs[step % 2]
        passing = step + 1 < comm.world
        if passing:
            handles = comm.exchange(cur, nxt)  # overlaps this step's compute
        if computed:
            o_p, l_p = ops.partial_fwd(q, cur[0], cur[1], scale, diag)
            if o32 is None:
                o32, lse = o_p, l_p
            else:
                ops.merge(o32, lse, o_p, l_p)
        if passing:
            comm.wait(handles)
            cur = nxt
    # every rank computes at least its own chunk, so o32 is set
    return ops.to_dtype(o32, q), lse, o32


def ring_attention_bwd(q, k, v, o32, do, lse, scale: Optional[float] = None, causal: bool = False, group=None,
                       ops=None, comm=None):
    """Backward of ``ring_attention_fwd``: returns (dQ, dK, dV) of this rank's
    chunks in the input type."""
    import torch

    _check(q, k, v)
    ops = ops or CudaChunkOps()
    comm = comm or RingComm(group)
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    world = comm.world
    sched = ring_schedule(comm.rank, world, causal)
    dq_acc = ops.zeros_acc(q)
    kv_cur = (k, v)
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    acc_cur = (ops.zeros_acc(k), ops.zeros_acc(v))   # accumulators of the chunk held now
    acc_bufs = [(ops.zeros_acc(k), ops.zeros_acc(v)) for _ in range(2)]
    part = ops.bwd_buffers(q, k)
    acc_handles = None
    for step, _src, computed, diag in sched:
        kv_nxt = kv_bufs[step % 2]
        passing = step + 1 < world
        if passing:
            kv_handles = comm.exchange(kv_cur, kv_nxt)
        if computed:
            gq, gk, gv = ops.partial_bwd(q, kv_cur[0], kv_cur[1], o32, do, lse, scale, diag, part)
        # this step's accumulators arrive from the previous rank (sent at the
        # end of its previous step); the sends of our previous step must also
        # be done before their buffers are reused
        comm.wait(acc_handles)
        if computed:
            ops.accumulate(dq_acc, gq)
            ops.accumulate(acc_cur[0], gk)
            ops.accumulate(acc_cur[1], gv)
        if world > 1:  # pass the accumulators on (the last hop brings them home)
            acc_nxt = acc_bufs[step % 2]
            acc_handles = comm.exchange(acc_cur, acc_nxt)
            acc_cur = acc_nxt
        if passing:
            comm.wait(kv_handles)
            kv_cur = kv_nxt
    comm.wait(acc_handles)
    # after world hops the accumulators held are those of this rank's chunk
    return ops.to_dtype(dq_acc, q), ops.to_dtype(acc_cur[0], k), ops.to_dtype(acc_cur[1], v)
