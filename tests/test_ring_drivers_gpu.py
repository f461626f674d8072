"""The ring-attention drivers themselves, end to end on the CUDA kernels.

RingAttention (the third ledger of "FlashAttention and long context: three
ledgers": K/V blocks passed around the devices, attention computed
blockwise) is run exactly as a user runs it: 2 and 3 processes, each one rank of
a gloo group, each calling ``ring_attn_fwd`` / ``ring_attn_bwd`` (contiguous
chunks) and ``ring_attn_fwd_zigzag`` / ``ring_attn_bwd_zigzag`` on its own
chunks.  Every rank computes on ``cuda:0`` (a run here has one GPU); the K/V
chunks and the travelling gradient sums move between the processes through the
exchange's host-staged gloo path.  No kernel waits on another process: the
exchange happens on the host between launches.

The ranks' outputs, put back in sequence order, are compared element by element
with the fp64 oracle's attention and gradients over the whole sequence, at the
same bars as every other parity test: O max-abs <= 1e-2 and rel-L2 <= 5e-3, LSE
max-abs <= 1e-3, gradients rel-L2 <= 1e-2."""

import datetime
import math
import os
import socket

import numpy as np
import pytest

import oracle
import synth
from tests._util import GRAD_REL_L2, assert_lse_close, assert_out_close, rel_l2

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed, Hq, Hkv, L, d):
    Q = synth.normal_bf16(seed * 8 + 1, (1, Hq, L, d))
    K = synth.normal_bf16(seed * 8 + 2, (1, Hkv, L, d))
    V = synth.normal_bf16(seed * 8 + 3, (1, Hkv, L, d))
    dO = synth.normal_bf16(seed * 8 + 4, (1, Hq, L, d))
    return Q, K, V, dO


def _rank_main(rank, world, port, out, cfg):
    import torch
    import torch.distributed as dist

    from exact_io_aware_46_b200.ring import (ring_attn_bwd, ring_attn_bwd_zigzag, ring_attn_fwd,
                                             ring_attn_fwd_zigzag, zigzag_chunks)

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    Hq, Hkv, L, d, causal = cfg["Hq"], cfg["Hkv"], cfg["L"], cfg["d"], cfg["causal"]
    Q, K, V, dO = (synth.to_torch_bf16(x).cuda() for x in _inputs(cfg["seed"], Hq, Hkv, L, d))
    scale = 1.0 / math.sqrt(d)
    res = {}
    # contiguous chunks: rank r holds rows [r Lc, (r + 1) Lc)
    Lc = L // world
    ch = lambda t, c, n: t[:, :, c * n:(c + 1) * n].contiguous()
    q, k, v, do = (ch(t, rank, Lc) for t in (Q, K, V, dO))
    O, lse = ring_attn_fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = ring_attn_bwd(q, k, v, O, do, lse, causal=causal, scale=scale)
    for name, t in (("O", O), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        res["c_" + name] = t.float().cpu().numpy()
    if cfg["zigzag"]:
        # zigzag: 2 * world chunks, rank r holds chunks r and 2 world - 1 - r
        Lz = L // (2 * world)
        mine = zigzag_chunks(rank, world)
        qz, kz, vz, doz = (tuple(ch(t, c, Lz) for c in mine) for t in (Q, K, V, dO))
        Oz, lz = ring_attn_fwd_zigzag(qz, kz, vz, scale=scale)
        dqz, dkz, dvz = ring_attn_bwd_zigzag(qz, kz, vz, Oz, doz, lz, scale=scale)
        for i in range(2):
            for name, t in (("O", Oz), ("lse", lz), ("dq", dqz), ("dk", dkz), ("dv", dvz)):
                res[f"z{i}_" + name] = t[i].float().cpu().numpy()
    torch.cuda.synchronize()
    dist.barrier()
    dist.destroy_process_group()
    np.savez(out + f".{rank}.npz", **res)


CASES = [
    # world, Hq, Hkv, L, d, causal, zigzag
    (2, 4, 2, 384, 128, True, True),     # GQA, chunks of 192 (zigzag: 96)
    (3, 2, 2, 420, 128, False, True),    # ragged chunks of 140 (zigzag: 70), not causal
    (3, 4, 1, 390, 128, True, False),    # 4 query heads per kv head, chunks of 130
    (2, 2, 1, 300, 64, True, True),      # d = 64, chunks of 150 (zigzag: 75)
]


@pytest.mark.parametrize("world,Hq,Hkv,L,d,causal,zigzag", CASES)
def test_ring_drivers_match_whole_sequence(tmp_path, world, Hq, Hkv, L, d, causal, zigzag):
    import torch.multiprocessing as mp

    cfg = dict(Hq=Hq, Hkv=Hkv, L=L, d=d, causal=causal, zigzag=zigzag,
               seed=9900 + 10 * world + d + L)
    out = str(tmp_path / "ring")
    mp.start_processes(_rank_main, args=(world, _free_port(), out, cfg), nprocs=world,
                       join=True, start_method="spawn")
    res = [dict(np.load(out + f".{r}.npz")) for r in range(world)]

    Q, K, V, dO = _inputs(cfg["seed"], Hq, Hkv, L, d)
    scale = 1.0 / math.sqrt(d)

    def check(what, chunks, n, mask_causal):
        """chunks[c] = (rank, prefix) holding global chunk c of n rows."""
        Oref, Lref = oracle.fwd(Q, K, V, scale, causal=mask_causal)
        gref = oracle.bwd(Q, K, V, dO, scale, causal=mask_causal)
        order = np.concatenate([np.arange(c * n, (c + 1) * n) for c in range(len(chunks))])
        cat = lambda key: np.concatenate([res[r][f"{p}_{key}"] for r, p in chunks], axis=2)
        assert_out_close(cat("O"), Oref[:, :, order], f"{what} O")
        assert_lse_close(cat("lse"), Lref[:, :, order])
        for gi, g in enumerate(("dq", "dk", "dv")):
            err = rel_l2(cat(g), gref[gi][:, :, order])
            assert err <= GRAD_REL_L2, f"{what} {g}: rel-L2 {err:.3e}"

    # contiguous: global chunk c lives on rank c
    check("contiguous", [(r, "c") for r in range(world)], L // world, causal)
    if zigzag:
        # zigzag (causal): chunk c < world is rank c's early chunk, chunk
        # c >= world is rank 2 world - 1 - c's late chunk
        chunks = [(c, "z0") if c < world else (2 * world - 1 - c, "z1")
                  for c in range(2 * world)]
        check("zigzag", chunks, L // (2 * world), True)
