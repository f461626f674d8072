"""Ring attention host logic without a GPU: the step schedule (closed forms,
and composed on the fp64 oracle it gives exact attention over the whole
sequence) and the double-buffered K/V ring pass on 2 and 3 gloo ranks."""

import os
import socket

import numpy as np
import pytest

import oracle
import synth
from exact_io_aware_46_b200.ring import CAUSAL, FULL, SKIP, RingExchange, ring_steps


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_visits_every_chunk_once(world, causal):
    for rank in range(world):
        st = ring_steps(rank, world, causal)
        assert [s for s, _, _ in st] == list(range(world))
        assert sorted(src for _, src, _ in st) == list(range(world))
        assert st[0][1] == rank  # a rank starts on its own chunk
        for s, src, kind in st:
            assert src == (rank - s) % world
            if not causal:
                assert kind == FULL
            else:
                assert kind == (CAUSAL if src == rank else FULL if src < rank else SKIP)


def test_schedule_causal_closed_forms():
    assert [k for _, _, k in ring_steps(0, 4, True)] == [CAUSAL, SKIP, SKIP, SKIP]
    assert [k for _, _, k in ring_steps(3, 4, True)] == [CAUSAL, FULL, FULL, FULL]
    assert [k for _, _, k in ring_steps(1, 4, True)] == [CAUSAL, FULL, SKIP, SKIP]
    with pytest.raises(ValueError):
        ring_steps(4, 4, True)


@pytest.mark.parametrize("world,causal", [(3, True), (3, False), (4, True)])
def test_schedule_composes_exact_attention_on_the_oracle(world, causal):
    """Each rank's chunk partials (oracle forward per step kind), merged with
    the oracle's normalised merge rule in step order, equal the oracle's
    attention over the whole sequence for that rank's rows."""
    Lc, d = 37, 8
    L = world * Lc
    Q = synth.bf16_bits_to_f64(synth.normal_bf16(611, (1, 2, L, d)))
    K = synth.bf16_bits_to_f64(synth.normal_bf16(612, (1, 1, L, d)))
    V = synth.bf16_bits_to_f64(synth.normal_bf16(613, (1, 1, L, d)))
    Oref, Lref = oracle.fwd(Q, K, V, 0.3, causal=causal)
    for rank in range(world):
        q = Q[:, :, rank * Lc:(rank + 1) * Lc]
        acc = None
        for _, src, kind in ring_steps(rank, world, causal):
            if kind == SKIP:
                continue
            kc = K[:, :, src * Lc:(src + 1) * Lc]
            vc = V[:, :, src * Lc:(src + 1) * Lc]
            Op, lp = oracle.fwd(q, kc, vc, 0.3, causal=(kind == CAUSAL))
            if acc is None:
                acc = [Op.copy(), lp.copy()]
                continue
            for h in range(2):
                for i in range(Lc):
                    m, l, o = oracle.merge(acc[1][0, h, i], 1.0, acc[0][0, h, i],
                                           lp[0, h, i], 1.0, Op[0, h, i])
                    acc[0][0, h, i] = o
                    acc[1][0, h, i] = m + np.log(l)
        rows = slice(rank * Lc, (rank + 1) * Lc)
        assert np.max(np.abs(acc[0] - Oref[:, :, rows])) <= 1e-12
        assert np.max(np.abs(acc[1] - Lref[:, :, rows])) <= 1e-12


def _exchange_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    k = torch.full((3, 5), float(rank))
    v = torch.full((2, 7), 10.0 * rank)
    ex = RingExchange((k, v))
    seen = []
    for s in range(world):
        if s + 1 < world:
            ex.start()
        seen.append((float(ex.cur[0][0, 0]), float(ex.cur[1][1, 6])))
        if s + 1 < world:
            ex.finish()
    dist.barrier()
    dist.destroy_process_group()
    with open(out + f".{rank}", "w") as f:
        f.write(repr(seen))


def _caller_tensors_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    from exact_io_aware_46_b200.ring import ring_bwd_pass

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    k = torch.full((3, 5), float(rank))
    v = torch.full((2, 7), 10.0 * rank)
    ex = RingExchange((k, v))
    for s in range(world):
        if s + 1 < world:
            ex.start()
            ex.finish()
    g = torch.zeros(4)
    ring_bwd_pass((k, v), (g,), ring_steps(rank, world, False), lambda *a: None,
                  lambda part, gs: None)
    dist.barrier()
    dist.destroy_process_group()
    with open(out + f".{rank}", "w") as f:
        f.write(repr((float(k.min()), float(k.max()), float(v.min()), float(v.max()),
                      float(g.abs().max()))))


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_pass_leaves_the_callers_tensors_alone(tmp_path, world):
    """A full ring pass (forward exchange, then the backward's two exchanges)
    sends the caller's K/V but never receives into them: a driver's caller can
    run the backward on the same K/V tensors after the forward.  (Receiving into
    the first held tensors broke this from the second swap on, i.e. from three
    ranks.)"""
    import torch.multiprocessing as mp

    out = str(tmp_path / "c")
    mp.start_processes(_caller_tensors_main, args=(world, _free_port(), out), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        kmin, kmax, vmin, vmax, g = eval(open(out + f".{rank}").read())
        assert (kmin, kmax, vmin, vmax) == (rank, rank, 10.0 * rank, 10.0 * rank)
        assert g == 0.0


@pytest.mark.parametrize("world", [1, 2, 3])
def test_ring_exchange_on_gloo_ranks(tmp_path, world):
    """At step s every rank holds the chunk of rank (rank - s) mod world."""
    import torch.multiprocessing as mp

    out = str(tmp_path / "x")
    mp.start_processes(_exchange_main, args=(world, _free_port(), out), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        seen = eval(open(out + f".{rank}").read())
        assert seen == [(float((rank - s) % world), 10.0 * ((rank - s) % world))
                        for s in range(world)]


def _bwd_pass_main(rank, world, port, out, causal):
    import datetime

    import torch
    import torch.distributed as dist

    from exact_io_aware_46_b200.ring import ring_bwd_pass

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    steps = ring_steps(rank, world, causal)
    seen = []

    def compute(kind, src, kv_held):
        seen.append(float(kv_held[0][0]))  # the K/V chunk held at this step
        return None if kind == SKIP else float(rank + 1)

    def add(part, g):
        g[0] += part

    kv = (torch.full((4,), float(rank)),)
    sums = ring_bwd_pass(kv, (torch.zeros(4),), steps, compute, add)
    dist.barrier()
    dist.destroy_process_group()
    with open(out + f".{rank}", "w") as f:
        f.write(repr((seen, float(sums[0][0]))))


@pytest.mark.parametrize("world,causal", [(1, True), (2, True), (3, True), (3, False)])
def test_ring_backward_gradient_sums_travel_home(tmp_path, world, causal):
    """Every rank adds its share to the sums of the chunk it holds; after the
    closing pass each rank holds its own chunk's total: the shares of every rank
    whose step on that chunk was not skipped."""
    import torch.multiprocessing as mp

    out = str(tmp_path / "g")
    mp.start_processes(_bwd_pass_main, args=(world, _free_port(), out, causal), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        seen, total = eval(open(out + f".{rank}").read())
        assert seen == [float((rank - s) % world) for s in range(world)]
        contributors = [r for r in range(world) if not causal or r >= rank]
        assert total == float(sum(r + 1 for r in contributors))


# ---------------------------------------------------------------- zigzag layout

from exact_io_aware_46_b200.ring import ring_steps_zigzag, zigzag_chunks  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_schedule_is_balanced_and_complete(world):
    """Every visible (query chunk, key chunk) pair of the causal 2*world-chunk
    sequence is computed exactly once, by the rank holding the query chunk, and
    every rank computes two full-chunk equivalents per step (a causal diagonal
    pair counts one half)."""
    seen = set()
    for rank in range(world):
        mine = zigzag_chunks(rank, world)
        for s, src, pairs in ring_steps_zigzag(rank, world):
            held = zigzag_chunks(src, world)
            assert src == (rank - s) % world
            work = 0.0
            for qi, ki, kind in pairs:
                a, b = mine[qi], held[ki]
                assert (kind == CAUSAL) == (a == b) and a >= b
                assert (a, b) not in seen
                seen.add((a, b))
                work += 0.5 if kind == CAUSAL else 1.0
            assert work == 2.0
    n = 2 * world
    assert seen == {(a, b) for a in range(n) for b in range(a + 1)}


@pytest.mark.parametrize("world", [2, 3])
def test_zigzag_schedule_composes_exact_attention_on_the_oracle(world):
    """Each rank's zigzag partials (oracle forward per pair), merged in fold
    order with the oracle's merge rule, equal the oracle's causal attention over
    the whole sequence for the rank's two chunks."""
    Lc, d = 23, 8
    L = 2 * world * Lc
    Q = synth.bf16_bits_to_f64(synth.normal_bf16(631, (1, 2, L, d)))
    K = synth.bf16_bits_to_f64(synth.normal_bf16(632, (1, 1, L, d)))
    V = synth.bf16_bits_to_f64(synth.normal_bf16(633, (1, 1, L, d)))
    Oref, Lref = oracle.fwd(Q, K, V, 0.4, causal=True)
    ch = lambda t, c: t[:, :, c * Lc:(c + 1) * Lc]
    for rank in range(world):
        mine = zigzag_chunks(rank, world)
        acc = [None, None]
        for _, src, pairs in ring_steps_zigzag(rank, world):
            held = zigzag_chunks(src, world)
            for qi, ki, kind in pairs:
                Op, lp = oracle.fwd(ch(Q, mine[qi]), ch(K, held[ki]), ch(V, held[ki]), 0.4,
                                    causal=(kind == CAUSAL))
                if acc[qi] is None:
                    acc[qi] = [Op.copy(), lp.copy()]
                    continue
                for h in range(2):
                    for i in range(Lc):
                        m, l, o = oracle.merge(acc[qi][1][0, h, i], 1.0, acc[qi][0][0, h, i],
                                               lp[0, h, i], 1.0, Op[0, h, i])
                        acc[qi][0][0, h, i] = o
                        acc[qi][1][0, h, i] = m + np.log(l)
        for qi in (0, 1):
            assert np.max(np.abs(acc[qi][0] - ch(Oref, mine[qi]))) <= 1e-12
            assert np.max(np.abs(acc[qi][1] - ch(Lref, mine[qi]))) <= 1e-12


def test_zigzag_folds_mark_first_and_last():
    from exact_io_aware_46_b200.ring import zigzag_folds

    for world in (1, 2, 4):
        for rank in range(world):
            folds = zigzag_folds(rank, world)
            for qi in (0, 1):
                mine = [f for f in folds if f[2] == qi]
                assert mine[0][5] and not any(f[5] for f in mine[1:])
                assert mine[-1][6] and not any(f[6] for f in mine[:-1])
            assert [f[0] for f in folds] == sorted(f[0] for f in folds)  # step order


def _zigzag_bwd_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    from exact_io_aware_46_b200.ring import ring_bwd_pass

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    mine = zigzag_chunks(rank, world)
    steps = ring_steps_zigzag(rank, world)

    def compute(pairs, src, kv_held):
        held = zigzag_chunks(src, world)
        assert [float(kv_held[i][0]) for i in (0, 1)] == [float(c) for c in held]
        return [(ki, float(mine[qi] + 1)) for qi, ki, _ in pairs]

    def add(parts, g):
        for ki, val in parts:
            g[ki] += val

    kv = tuple(torch.full((4,), float(c)) for c in mine)
    sums = ring_bwd_pass(kv, (torch.zeros(4), torch.zeros(4)), steps, compute, add)
    dist.barrier()
    dist.destroy_process_group()
    with open(out + f".{rank}", "w") as f:
        f.write(repr([float(t[0]) for t in sums]))


@pytest.mark.parametrize("world", [2, 3])
def test_zigzag_backward_sums_travel_home(tmp_path, world):
    """Zigzag backward routing: every query chunk a adds a + 1 to the sums of each
    key chunk b <= a it meets; after the closing pass a rank holds, for each of
    its two chunks b, the total over a >= b."""
    import torch.multiprocessing as mp

    out = str(tmp_path / "z")
    mp.start_processes(_zigzag_bwd_main, args=(world, _free_port(), out), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        got = eval(open(out + f".{rank}").read())
        want = [float(sum(a + 1 for a in range(b, 2 * world))) for b in zigzag_chunks(rank, world)]
        assert got == want
