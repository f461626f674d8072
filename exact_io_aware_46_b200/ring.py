"""Ring attention: the forward over a sequence split across the ranks of a
process group (context parallelism, the third ledger of "FlashAttention and
long context: separate the three ledgers", where RingAttention passes K/V
blocks around the devices and computes blockwise attention).

Rank r holds one contiguous chunk of the sequence: its query rows and its
keys/values, all chunks of equal length.  In ``world`` steps every K/V chunk
visits every rank: at step s rank r holds the chunk of rank (r - s) mod world,
computes the partial attention of its queries against it with ``attn_fwd``
(on the GPU kernels) and folds the partial into an fp32 accumulator with the
normalised merge rule in LSE form -- in the forward kernel's epilogue
(``attn_fwd_merge``), so a step is one kernel launch.  While a step
computes, the next chunk is already in flight: each rank sends the chunk it
holds to rank r + 1 and receives the next from rank r - 1 with point-to-point
operations of ``torch.distributed`` (NCCL between GPUs over NVLink; gloo on
CPU), into a second buffer.  Under the causal mask a chunk from a later rank is
entirely masked and skipped (its exchange still runs, so every rank takes the
same collective steps in the same order), the diagonal chunk is causal and the
earlier chunks are fully visible.

The backward (``ring_attn_bwd``) runs the same ring with the forward's global O
and LSE: the partial gradients of a (query chunk, key chunk) pair from
``attn_bwd`` are exact pieces of the whole-sequence gradients, since P and
D = rowsum(dO o O) only need the global LSE and O.  dQ sums locally; the running
sums of a chunk's dK and dV travel with that chunk (each rank adds its share
before passing them on) and one extra pass at the end brings them home.  The sums
are kept in fp32 by ``attn_accumulate``.

For the causal mask there is also a zigzag layout (``ring_attn_fwd_zigzag``,
``ring_attn_bwd_zigzag``): the sequence is cut into 2 * world chunks and rank r
holds chunks r and 2 * world - 1 - r, which gives every rank the same work at
every step.

The exchange moves K/V (and gradient sums) between ranks and the kernels compute;
there is no compute on the host and no fallback: ``ring_attn_fwd`` and
``ring_attn_bwd`` need the CUDA library.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

FULL, CAUSAL, SKIP = "full", "causal", "skip"


def ring_steps(rank: int, world: int, causal: bool):
    """The schedule of one rank: a list of (step, source rank, kind), where
    kind is FULL (every key of the chunk visible), CAUSAL (the rank's own
    chunk, the causal mask inside it) or SKIP (every key masked)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    out = []
    for s in range(world):
        src = (rank - s) % world
        if not causal or src < rank:
            kind = FULL
        elif src == rank:
            kind = CAUSAL
        else:
            kind = SKIP
        out.append((s, src, kind))
    return out


class RingExchange:
    """Double-buffered ring pass of a tuple of tensors: ``start()`` posts the
    send of the held tensors to rank + 1 and the receive of the next ones from
    rank - 1; ``finish()`` waits for both and makes the received tensors the
    held ones.  Works on any backend with point-to-point operations.

    NCCL moves CUDA tensors device to device (over NVLink between GPUs).  A
    gloo group cannot send CUDA tensors, so there the pass is staged through
    pinned host buffers: ``start()`` copies the held tensors to the host (after
    the work already queued on the current stream, which wrote them) and sends
    the bytes; ``finish()`` copies what arrived back into the device buffer.
    The staged path exists for process groups without a device transport (and
    for testing the drivers with several processes on one GPU); its host copies
    are not overlapped with the compute."""

    def __init__(self, tensors, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        # the first held tensors are the caller's: they are sent but never
        # received into (the caller still owns them after the pass)
        self.cur = [t.contiguous() for t in tensors]
        self.borrowed = True
        self.nxt = [torch.empty_like(t) for t in self.cur]
        self.reqs = None
        self.staged = (any(t.is_cuda for t in self.cur)
                       and dist.get_backend(group) == dist.Backend.GLOO)
        if self.staged:
            pin = torch.cuda.is_available()
            self.h_send = [torch.empty(t.shape, dtype=t.dtype, pin_memory=pin) for t in self.cur]
            self.h_recv = [torch.empty(t.shape, dtype=t.dtype, pin_memory=pin) for t in self.cur]

    def _peer(self, r):
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def start(self):
        if self.reqs is not None:
            raise RuntimeError("a ring step is already in flight")
        to = self._peer((self.rank + 1) % self.world)
        frm = self._peer((self.rank - 1) % self.world)
        send, recv = self.cur, self.nxt
        if self.staged:
            for h, t in zip(self.h_send, self.cur):
                h.copy_(t)  # waits for the stream's writes of t
            # bytes on the wire: the transport need not know the element type
            send = [h.view(torch.uint8) for h in self.h_send]
            recv = [h.view(torch.uint8) for h in self.h_recv]
        ops = [dist.P2POp(dist.isend, t, to, self.group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, frm, self.group) for t in recv]
        self.reqs = dist.batch_isend_irecv(ops)

    def finish(self):
        for r in self.reqs:
            r.wait()
        self.reqs = None
        if self.staged:
            for t, h in zip(self.nxt, self.h_recv):
                t.copy_(h)
        old = self.cur
        self.cur = self.nxt
        if self.borrowed:
            self.nxt = [torch.empty_like(t) for t in old]
            self.borrowed = False
        else:
            self.nxt = old


def fold_chunk(q, kc, vc, kind, O_acc, lse_acc, first, O_out=None, scale=None, workspace=None):
    """One ring step's compute: the partial attention of q against the K/V chunk
    (kc, vc) held at this step (kind FULL or CAUSAL), folded into the fp32
    accumulator (O_acc, lse_acc) by the forward kernel itself; ``first``
    initialises it, ``O_out`` (bf16) receives the merged O at the last step."""
    from . import attn_fwd_merge

    if kind == SKIP:
        return
    attn_fwd_merge(q, kc, vc, O_acc, lse_acc, init=first, O_out=O_out, scale=scale,
                   causal=(kind == CAUSAL), workspace=workspace)


def ring_attn_fwd(q, k, v, group=None, causal=True, scale=None):
    """Ring-attention forward.  q [B, Hq, Lc, d], k/v [B, Hkv, Lc, d] bf16 CUDA
    tensors: this rank's chunk (rows [rank * Lc, (rank + 1) * Lc) of the whole
    sequence); every rank passes the same shapes.  Returns this rank's
    (O bf16 [B, Hq, Lc, d], LSE fp32 [B, Hq, Lc]) of attention over the whole
    sequence."""
    if not q.is_cuda:
        raise ValueError("ring_attn_fwd runs on the CUDA kernels")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    steps = ring_steps(rank, world, causal)
    last = max(s for s, _, kind in steps if kind != SKIP)
    O_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    O = torch.empty_like(q)
    ex = RingExchange((k, v), group)
    for s, _, kind in steps:
        if s + 1 < world:
            ex.start()
        kc, vc = ex.cur
        fold_chunk(q, kc, vc, kind, O_acc, lse_acc, first=(s == 0),
                   O_out=O if s == last else None, scale=scale)
        if s + 1 < world:
            ex.finish()
    return O, lse_acc


def bwd_chunk(q, kc, vc, o, do, lse, kind, scale=None, workspace=None):
    """One ring step's backward: the partial (dQ, dK, dV) (bf16) of this rank's
    query chunk against the K/V chunk held at this step, from the whole-sequence
    O and LSE of this rank's rows; None for a SKIP step."""
    from . import attn_bwd

    if kind == SKIP:
        return None
    return attn_bwd(q, kc, vc, o, do, lse, scale=scale, causal=(kind == CAUSAL),
                    workspace=workspace)


def ring_bwd_pass(kv, grads, steps, compute, add, group=None):
    """The backward's data movement.  ``kv``: this rank's K/V chunk tensors, sent
    around the ring one step ahead as in the forward; ``grads``: zeroed running
    sums of this chunk's gradients, which travel with their chunk.  At each step
    ``compute(kind, src, kv_held)`` returns this rank's partial for the held
    chunk (or None) while the previous step's sums are still in flight, then
    ``add(partial, grads_held)`` adds it into the held chunk's sums, which are
    passed on.  Returns this rank's own chunk's sums after the closing pass."""
    world = len(steps)
    kvx = RingExchange(kv, group)
    if world == 1:  # nothing travels: the rank's own chunk is the whole sequence
        grads = [t.contiguous() for t in grads]
        part = compute(steps[0][2], steps[0][1], kvx.cur)
        if part is not None:
            add(part, grads)
        return grads
    gx = RingExchange(grads, group)
    for s, src, kind in steps:
        if s + 1 < world:
            kvx.start()
        part = compute(kind, src, kvx.cur)
        if s > 0:
            gx.finish()
        if part is not None:
            add(part, gx.cur)
        gx.start()
        if s + 1 < world:
            kvx.finish()
    gx.finish()
    return gx.cur


def ring_attn_bwd(q, k, v, o, do, lse, group=None, causal=True, scale=None):
    """Ring-attention backward.  q, o, do [B, Hq, Lc, d] and lse [B, Hq, Lc] of
    this rank's rows (o and lse from ``ring_attn_fwd``), k/v [B, Hkv, Lc, d] of
    this rank's keys.  Returns this rank's (dQ, dK, dV) bf16 of the whole-sequence
    loss."""
    from . import attn_accumulate

    if not q.is_cuda:
        raise ValueError("ring_attn_bwd runs on the CUDA kernels")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    steps = ring_steps(rank, world, causal)
    dq_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    first = [True]

    def compute(kind, src, kv_held):
        return bwd_chunk(q, kv_held[0], kv_held[1], o, do, lse, kind, scale=scale)

    def add(part, g):
        dqp, dkp, dvp = part
        attn_accumulate(dqp, dq_acc, init=first[0])
        first[0] = False
        attn_accumulate(dkp, g[0], init=False)
        attn_accumulate(dvp, g[1], init=False)

    zeros = (torch.zeros(k.shape, dtype=torch.float32, device=k.device),
             torch.zeros(v.shape, dtype=torch.float32, device=v.device))
    gk, gv = ring_bwd_pass((k, v), zeros, steps, compute, add, group)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    attn_accumulate(None, dq_acc, init=False, out=dq)
    attn_accumulate(None, gk, init=False, out=dk)
    attn_accumulate(None, gv, init=False, out=dv)
    return dq, dk, dv


# ---------------------------------------------------------------- zigzag layout
# Under the causal mask, contiguous chunks leave rank r with r + 1 chunk
# computations and the last rank with world of them.  In the zigzag layout the
# sequence is cut into 2 * world chunks and rank r holds chunks r and
# 2 * world - 1 - r (an early and a late one); K/V chunk pairs travel the ring
# as before.  Every rank then computes two full-chunk equivalents per step: at
# step 0 its two diagonal chunks (causal) and late-on-early (full), at every
# other step two full chunk pairs; the other two pairs of the step are masked.


def zigzag_chunks(rank: int, world: int):
    """The two global chunk indices (of 2 * world) that rank ``rank`` holds."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank, 2 * world - 1 - rank


def ring_steps_zigzag(rank: int, world: int):
    """The causal zigzag schedule of one rank: a list of (step, source rank,
    [(q, kv, kind), ...]) where q and kv index this rank's query chunk and the
    held K/V chunk (0 = the early one, 1 = the late one) and kind is FULL or
    CAUSAL; masked pairs are left out."""
    mine = zigzag_chunks(rank, world)
    out = []
    for s in range(world):
        src = (rank - s) % world
        held = zigzag_chunks(src, world)
        pairs = []
        for qi, a in enumerate(mine):
            for ki, b in enumerate(held):
                if a > b:
                    pairs.append((qi, ki, FULL))
                elif a == b:
                    pairs.append((qi, ki, CAUSAL))
        out.append((s, src, pairs))
    return out


def zigzag_folds(rank: int, world: int):
    """The folds of one rank in order: (step, source rank, q, kv, kind, first,
    last), with first / last marking the first and the last fold into query
    chunk q (the first initialises its accumulator, the last writes O)."""
    flat = [(s, src, qi, ki, kind) for s, src, pairs in ring_steps_zigzag(rank, world)
            for qi, ki, kind in pairs]
    out = []
    for i, (s, src, qi, ki, kind) in enumerate(flat):
        first = all(f[2] != qi for f in flat[:i])
        last = all(f[2] != qi for f in flat[i + 1:])
        out.append((s, src, qi, ki, kind, first, last))
    return out


def ring_attn_fwd_zigzag(q, k, v, group=None, scale=None):
    """Causal ring-attention forward in the zigzag layout.  q, k, v: pairs of
    bf16 CUDA tensors, this rank's early and late chunk (global chunks r and
    2 * world - 1 - r of equal length): q [B, Hq, Lc, d], k/v [B, Hkv, Lc, d].
    Returns (O pair, LSE pair) for the two query chunks."""
    if not q[0].is_cuda:
        raise ValueError("ring_attn_fwd_zigzag runs on the CUDA kernels")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    folds = zigzag_folds(rank, world)
    O_acc = [torch.empty(t.shape, dtype=torch.float32, device=t.device) for t in q]
    lse_acc = [torch.empty(t.shape[:-1], dtype=torch.float32, device=t.device) for t in q]
    O = [torch.empty_like(t) for t in q]
    ex = RingExchange((k[0], k[1], v[0], v[1]), group)
    # the folds into the two query chunks' accumulators are independent: the
    # late chunk's run on a side stream (its own scheduler workspace), so one
    # launch's last partial wave overlaps the other's; both join before the
    # exchange reuses the chunk buffers
    main = torch.cuda.current_stream(q[0].device)
    side = torch.cuda.Stream(device=q[0].device)
    ws = [torch.zeros(256, dtype=torch.uint8, device=q[0].device) for _ in range(2)]
    for s in range(world):
        if s + 1 < world:
            ex.start()
        k0, k1, v0, v1 = ex.cur
        side.wait_stream(main)
        for _, _, qi, ki, kind, first, last in (f for f in folds if f[0] == s):
            with torch.cuda.stream(side if qi == 1 else main):
                fold_chunk(q[qi], (k0, k1)[ki], (v0, v1)[ki], kind, O_acc[qi], lse_acc[qi],
                           first=first, O_out=O[qi] if last else None, scale=scale,
                           workspace=ws[qi])
        main.wait_stream(side)
        if s + 1 < world:
            ex.finish()
    return tuple(O), tuple(lse_acc)


def ring_attn_bwd_zigzag(q, k, v, o, do, lse, group=None, scale=None):
    """Causal ring-attention backward in the zigzag layout.  q, o, do, lse, k,
    v: pairs (this rank's early and late chunk) shaped as in ``ring_attn_bwd``,
    o and lse from ``ring_attn_fwd_zigzag``.  Returns (dQ pair, dK pair, dV pair)
    bf16.  The running sums of the held chunks' dK and dV (four fp32 tensors)
    travel with the K/V pair."""
    from . import attn_accumulate

    if not q[0].is_cuda:
        raise ValueError("ring_attn_bwd_zigzag runs on the CUDA kernels")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    steps = ring_steps_zigzag(rank, world)  # the pair list rides in the "kind" slot
    dq_acc = [torch.empty(t.shape, dtype=torch.float32, device=t.device) for t in q]
    first = [True, True]

    def compute(pairs, src, kv_held):
        k0, k1, v0, v1 = kv_held
        return [(qi, ki, bwd_chunk(q[qi], (k0, k1)[ki], (v0, v1)[ki], o[qi], do[qi], lse[qi],
                                   kind, scale=scale)) for qi, ki, kind in pairs]

    def add(parts, g):
        for qi, ki, (dqp, dkp, dvp) in parts:
            attn_accumulate(dqp, dq_acc[qi], init=first[qi])
            first[qi] = False
            attn_accumulate(dkp, g[ki], init=False)
            attn_accumulate(dvp, g[2 + ki], init=False)

    zeros = tuple(torch.zeros(t.shape, dtype=torch.float32, device=t.device)
                  for t in (k[0], k[1], v[0], v[1]))
    g = ring_bwd_pass((k[0], k[1], v[0], v[1]), zeros, steps, compute, add, group)
    dq = tuple(torch.empty_like(t) for t in q)
    dk = tuple(torch.empty_like(t) for t in k)
    dv = tuple(torch.empty_like(t) for t in v)
    for acc, out in zip((dq_acc[0], dq_acc[1], g[0], g[1], g[2], g[3]),
                        (dq[0], dq[1], dk[0], dk[1], dv[0], dv[1])):
        attn_accumulate(None, acc, init=False, out=out)
    return dq, dk, dv
