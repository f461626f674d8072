"""Parity at the exact shapes, seeds and launch configurations of the bench lines
that the other full-size tests do not already cover: the d = 64 forward, the
sliding-window forward, the packed (varlen) prefill and ring attention's
decomposition of the long-context workload (forward against the oracle, backward
against the undivided call).  Sampled outputs are compared with the fp64 oracle
at the bars every parity test uses."""

import math

import numpy as np
import pytest

import bench
import oracle
import synth
from tests._util import GRAD_REL_L2, assert_lse_close, assert_out_close, bits, rel_l2, to_f64

pytestmark = pytest.mark.gpu


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


def _rows(L, seed, extra=()):
    rng = np.random.default_rng(seed)
    r = {0, 1, 127, 128, L - 129, L - 128, L - 1, *extra}
    r |= set(rng.choice(L, 24, replace=False).tolist())
    return np.array(sorted(x for x in r if 0 <= x < L), dtype=np.int32)


def _check_heads(q, k, v, O, Lse, heads, rows, causal=True, window=0):
    G = q.shape[1] // k.shape[1]
    d = q.shape[3]
    for b, h in heads:
        Qh = bits(q[b:b + 1, h:h + 1])
        Kh = bits(k[b:b + 1, h // G:h // G + 1])
        Vh = bits(v[b:b + 1, h // G:h // G + 1])
        Oref, Lref = oracle.fwd(Qh, Kh, Vh, 1 / math.sqrt(d), causal=causal, rows=rows,
                                window=window)
        assert_out_close(to_f64(O[b, h, rows]), Oref[0, 0], f"O[{b},{h}]")
        assert_lse_close(to_f64(Lse[b, h, rows]), Lref[0, 0])


def test_d64_forward_bench_workload():
    """The bench's d = 64 line: causal B4 H16 L4096 d64, its own inputs."""
    import torch

    attn = _lib()
    c = bench.FWD
    shp = (c["B"], c["Hq"], c["L"], 64)
    q, k, v = (synth.normal_bf16_device(synth.workload_seed(2, t) ^ 64, shp, "cuda")
               for t in ("q", "k", "v"))
    O, Lse = attn.attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    _check_heads(q, k, v, O, Lse, [(0, 0), (1, 9), (3, 15)], _rows(c["L"], 6401))


def test_sliding_window_bench_workload():
    """The bench's sliding-window line: B4 H16 L4096 d128, window 1024, the forward
    workload's inputs."""
    import torch

    attn = _lib()
    c, W = bench.FWD, bench.WINDOW
    shp = (c["B"], c["Hq"], c["L"], c["d"])
    q, k, v = (synth.normal_bf16_device(synth.workload_seed(2, t), shp, "cuda")
               for t in ("q", "k", "v"))
    O, Lse = attn.attn_fwd_sliding(q, k, v, W)
    torch.cuda.synchronize()
    rows = _rows(c["L"], 6402, extra=(W - 1, W, W + 1, 2 * W, 2 * W + 127))
    _check_heads(q, k, v, O, Lse, [(0, 0), (2, 5), (3, 15)], rows, window=W)


def test_varlen_bench_workload():
    """The bench's packed prefill: 16 sequences, lengths ~ U[256, 4096] from the
    bench's seed, back to back, H16 d128 causal; the longest, the first and the last
    sequence against the oracle, and bit for bit against attn_fwd on each alone."""
    import torch

    attn = _lib()
    c = bench.VARLEN
    lens = synth.uniform_int(synth.workload_seed(6, "klen"), c["n_seq"], c["lo"], c["hi"])
    total = int(np.sum(lens.astype(np.int64)))
    starts = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    cu = torch.tensor(starts, dtype=torch.int32, device="cuda")
    q, k, v = (synth.normal_bf16_device(synth.workload_seed(6, t), (total, c["H"], c["d"]),
                                        "cuda") for t in ("q", "k", "v"))
    mx = int(lens.max())
    O, Lse = attn.attn_fwd_varlen(q, k, v, cu, cu, mx, mx, causal=True)
    torch.cuda.synchronize()
    for i in sorted({int(np.argmax(lens)), 0, c["n_seq"] - 1}):
        s, e = int(starts[i]), int(starts[i + 1])
        # this sequence as a [1, H, n, d] batch of one
        qs, ks, vs = (t[s:e].permute(1, 0, 2).unsqueeze(0).contiguous() for t in (q, k, v))
        Os = O[s:e].permute(1, 0, 2).unsqueeze(0)
        Ls = Lse[:, s:e].unsqueeze(0)
        O1, L1 = attn.attn_fwd(qs, ks, vs, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(O1, Os) and torch.equal(L1, Ls), f"sequence {i}"
        _check_heads(qs, ks, vs, Os, Ls, [(0, 0), (0, c["H"] - 1)], _rows(e - s, 6403 + i))


def test_ring_decomposition_bench_workload():
    """The bench's ring line: the long-context workload B1 Hq32 Hkv8 L16384 d128,
    causal, in 4 chunks.  Every emulated rank's folds (contiguous and zigzag) against
    the oracle on sampled rows; the backward's chunk-pair decomposition, summed in
    fp32, against the undivided attn_bwd."""
    import torch

    from exact_io_aware_46_b200.ring import (bwd_chunk, fold_chunk, ring_steps, zigzag_chunks,
                                             zigzag_folds)

    attn = _lib()
    c = bench.RING
    W, Lc = c["world"], c["L"] // c["world"]
    dev = torch.device("cuda")
    shp_q = (c["B"], c["Hq"], c["L"], c["d"])
    shp_k = (c["B"], c["Hkv"], c["L"], c["d"])
    q = synth.normal_bf16_device(synth.workload_seed(3, "q"), shp_q, dev)
    k = synth.normal_bf16_device(synth.workload_seed(3, "k"), shp_k, dev)
    v = synth.normal_bf16_device(synth.workload_seed(3, "v"), shp_k, dev)
    chunk = lambda t, i, n: t[:, :, i * n:(i + 1) * n].contiguous()
    heads = [(0, 0), (0, 13), (0, 31)]
    rows_c = _rows(Lc, 6404)
    # contiguous layout: rank r holds chunk r
    O = torch.empty_like(q)
    Lse = torch.empty((c["B"], c["Hq"], c["L"]), dtype=torch.float32, device=dev)
    for r in range(W):
        qr = chunk(q, r, Lc)
        O_acc = torch.empty(qr.shape, dtype=torch.float32, device=dev)
        lse_acc = torch.empty((c["B"], c["Hq"], Lc), dtype=torch.float32, device=dev)
        Or = torch.empty_like(qr)
        steps = ring_steps(r, W, True)
        last = max(s for s, _, kind in steps if kind != "skip")
        for s, src, kind in steps:
            fold_chunk(qr, chunk(k, src, Lc), chunk(v, src, Lc), kind, O_acc, lse_acc,
                       first=(s == 0), O_out=Or if s == last else None)
        O[:, :, r * Lc:(r + 1) * Lc] = Or
        Lse[:, :, r * Lc:(r + 1) * Lc] = lse_acc
    torch.cuda.synchronize()
    rows = np.concatenate([r * Lc + rows_c for r in range(W)]).astype(np.int32)
    _check_heads(q, k, v, O, Lse, heads, rows)
    # zigzag layout: 2W chunks, rank r holds chunks r and 2W - 1 - r
    Lz = c["L"] // (2 * W)
    Oz = torch.empty_like(q)
    Lsez = torch.empty_like(Lse)
    for r in range(W):
        mine = zigzag_chunks(r, W)
        acc = [(torch.empty((c["B"], c["Hq"], Lz, c["d"]), dtype=torch.float32, device=dev),
                torch.empty((c["B"], c["Hq"], Lz), dtype=torch.float32, device=dev))
               for _ in range(2)]
        outs = [torch.empty((c["B"], c["Hq"], Lz, c["d"]), dtype=torch.bfloat16, device=dev)
                for _ in range(2)]
        for _, src, qi, ki, kind, first, last in zigzag_folds(r, W):
            g = zigzag_chunks(src, W)[ki]
            fold_chunk(chunk(q, mine[qi], Lz), chunk(k, g, Lz), chunk(v, g, Lz), kind,
                       acc[qi][0], acc[qi][1], first=first, O_out=outs[qi] if last else None)
        for qi in range(2):
            Oz[:, :, mine[qi] * Lz:(mine[qi] + 1) * Lz] = outs[qi]
            Lsez[:, :, mine[qi] * Lz:(mine[qi] + 1) * Lz] = acc[qi][1]
    torch.cuda.synchronize()
    _check_heads(q, k, v, Oz, Lsez, heads, rows)
    # backward: every rank's chunk pairs through attn_bwd, summed in fp32, against the
    # undivided call (itself checked against the oracle at full size elsewhere)
    dO = synth.normal_bf16_device(synth.workload_seed(3, "do"), shp_q, dev)
    O1, L1 = attn.attn_fwd(q, k, v, causal=True)
    dq1, dk1, dv1 = attn.attn_bwd(q, k, v, O1, dO, L1, causal=True)
    dq = [None] * W
    dk = [None] * W
    dv = [None] * W
    for r in range(W):
        first = True
        for _, src, kind in ring_steps(r, W, True):
            part = bwd_chunk(chunk(q, r, Lc), chunk(k, src, Lc), chunk(v, src, Lc),
                             chunk(O1, r, Lc), chunk(dO, r, Lc), chunk(L1, r, Lc), kind)
            if part is None:
                continue
            if first:
                dq[r] = torch.zeros(part[0].shape, dtype=torch.float32, device=dev)
                first = False
            attn.attn_accumulate(part[0], dq[r], init=False)
            for acc_list, g in ((dk, part[1]), (dv, part[2])):
                if acc_list[src] is None:
                    acc_list[src] = torch.zeros(g.shape, dtype=torch.float32, device=dev)
                attn.attn_accumulate(g, acc_list[src], init=False)
    torch.cuda.synchronize()
    for name, parts, whole in (("dQ", dq, dq1), ("dK", dk, dk1), ("dV", dv, dv1)):
        got = torch.cat(parts, dim=2)
        err = rel_l2(to_f64(got), to_f64(whole))
        assert err <= GRAD_REL_L2, f"ring {name}: rel-L2 {err:.3e} against the undivided call"
    del q, k, v, dO, O, O1, dq1, dk1, dv1
    torch.cuda.empty_cache()
