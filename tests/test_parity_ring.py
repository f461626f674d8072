"""Ring attention on one GPU: the merge kernel (attn_merge_partial) against
the oracle's normalised merge rule, and the ring decomposition -- every rank's
steps from ring_steps, each computed by fold_chunk on the CUDA kernels, with
the chunks taken from one tensor instead of arriving over the ring -- against
the oracle's attention over the whole sequence.  (The exchange itself is
covered on gloo ranks in test_ring.py; several GPUs are not available here.)"""

import math

import numpy as np
import pytest

import oracle
import synth
from exact_io_aware_46_b200.ring import ring_steps, fold_chunk
from tests._util import assert_lse_close, assert_out_close, dev_bf16, to_f64

pytestmark = pytest.mark.gpu


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


@pytest.mark.parametrize("d", [64, 128, 256, 8])
def test_merge_kernel_matches_oracle_merge(d):
    import torch

    attn = _lib()
    rows = 1000
    rng = np.random.default_rng(d)
    Oa = rng.standard_normal((rows, d)).astype(np.float32)
    la = (rng.standard_normal(rows) * 3).astype(np.float32)
    Ob_bits = synth.normal_bf16(900 + d, (rows, d))
    Ob = synth.bf16_bits_to_f64(Ob_bits)
    lb = (rng.standard_normal(rows) * 3).astype(np.float32)
    la[::7] = -np.inf      # accumulator without keys
    lb[::5] = -np.inf      # partial without keys (rows 0, 35, ... have neither)
    O_acc = torch.from_numpy(Oa).cuda()
    lse_acc = torch.from_numpy(la).cuda()
    O_out = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    attn.attn_merge_partial(dev_bf16(Ob_bits), torch.from_numpy(lb).cuda(), O_acc, lse_acc,
                            init=False, O_out=O_out)
    torch.cuda.synchronize()
    got_O, got_l = to_f64(O_acc), to_f64(lse_acc)
    for i in range(rows):
        m, l, o = oracle.merge(float(la[i]), 1.0, Oa[i].astype(np.float64), float(lb[i]), 1.0,
                               Ob[i])
        ref_l = m + math.log(l) if l > 0 else -math.inf
        assert got_l[i] == ref_l or abs(got_l[i] - ref_l) <= 1e-5, i
        assert np.max(np.abs(got_O[i] - o)) <= 1e-5 * (1 + np.max(np.abs(o))), i
    assert torch.equal(O_out, O_acc.to(torch.bfloat16))


def test_merge_init_copies_the_partial():
    import torch

    attn = _lib()
    Ob_bits = synth.normal_bf16(77, (3, 5, 128))
    lb = torch.tensor(np.arange(15, dtype=np.float32).reshape(3, 5), device="cuda")
    lb[1, 2] = -float("inf")
    O_acc = torch.full((3, 5, 128), 9.0, device="cuda")
    lse_acc = torch.full((3, 5), 9.0, device="cuda")
    Ob = dev_bf16(Ob_bits)
    attn.attn_merge_partial(Ob, lb, O_acc, lse_acc, init=True)
    torch.cuda.synchronize()
    ref = Ob.float()
    ref[1, 2] = 0.0  # a row without keys is O = 0
    assert torch.equal(O_acc, ref) and torch.equal(lse_acc, lb)


@pytest.mark.parametrize("world,causal,Hq,Hkv,Lc,d", [
    (2, True, 4, 2, 300, 128),
    (3, True, 2, 2, 256, 128),
    (4, False, 2, 1, 130, 64),
    (3, False, 4, 4, 200, 128),
])
def test_ring_decomposition_matches_whole_sequence(world, causal, Hq, Hkv, Lc, d):
    import torch

    L = world * Lc
    seed = 9100 + world * 10 + Lc
    Q = synth.normal_bf16(seed * 4 + 1, (1, Hq, L, d))
    K = synth.normal_bf16(seed * 4 + 2, (1, Hkv, L, d))
    V = synth.normal_bf16(seed * 4 + 3, (1, Hkv, L, d))
    q_all, k_all, v_all = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    scale = 1.0 / math.sqrt(d)
    Oref, Lref = oracle.fwd(Q, K, V, scale, causal=causal)
    for rank in range(world):
        rows = slice(rank * Lc, (rank + 1) * Lc)
        q = q_all[:, :, rows].contiguous()
        O_acc = torch.empty((1, Hq, Lc, d), dtype=torch.float32, device="cuda")
        lse_acc = torch.empty((1, Hq, Lc), dtype=torch.float32, device="cuda")
        O = torch.empty((1, Hq, Lc, d), dtype=torch.bfloat16, device="cuda")
        steps = ring_steps(rank, world, causal)
        last = max(s for s, _, kind in steps if kind != "skip")
        for s, src, kind in steps:
            kc = k_all[:, :, src * Lc:(src + 1) * Lc].contiguous()
            vc = v_all[:, :, src * Lc:(src + 1) * Lc].contiguous()
            fold_chunk(q, kc, vc, kind, O_acc, lse_acc, first=(s == 0),
                       O_out=O if s == last else None, scale=scale)
        torch.cuda.synchronize()
        assert_out_close(to_f64(O), Oref[:, :, rows], f"O[rank {rank}]")
        assert_lse_close(to_f64(lse_acc), Lref[:, :, rows])


def test_fwd_merge_rows_without_keys_keep_the_accumulator():
    """attn_fwd_merge with a chunk whose keys are all padded away for one
    sequence (k_lens = 0): that sequence's accumulator is unchanged; the other
    sequence gets attention over both chunks.  Also init with no keys gives
    O = 0, LSE = -inf."""
    import torch

    attn = _lib()
    B, H, Lq, LA, LB, d = 2, 2, 150, 200, 180, 128
    Q = synth.normal_bf16(9301, (B, H, Lq, d))
    KA = synth.normal_bf16(9302, (B, H, LA, d))
    VA = synth.normal_bf16(9303, (B, H, LA, d))
    KB = synth.normal_bf16(9304, (B, H, LB, d))
    VB = synth.normal_bf16(9305, (B, H, LB, d))
    scale = 1.0 / math.sqrt(d)
    acc = torch.empty((B, H, Lq, d), dtype=torch.float32, device="cuda")
    lacc = torch.empty((B, H, Lq), dtype=torch.float32, device="cuda")
    O = torch.empty((B, H, Lq, d), dtype=torch.bfloat16, device="cuda")
    q = dev_bf16(Q)
    attn.attn_fwd_merge(q, dev_bf16(KA), dev_bf16(VA), acc, lacc, init=True, scale=scale)
    kl = torch.tensor([0, 150], dtype=torch.int32, device="cuda")
    attn.attn_fwd_merge(q, dev_bf16(KB), dev_bf16(VB), acc, lacc, init=False, O_out=O,
                        scale=scale, k_lens=kl)
    torch.cuda.synchronize()
    K = np.concatenate([KA, KB], axis=2)
    V = np.concatenate([VA, VB], axis=2)
    Oref, Lref = oracle.fwd(Q, K, V, scale, k_lens=[LA, LA + 150])
    assert_out_close(to_f64(O), Oref)
    assert_lse_close(to_f64(lacc), Lref)
    # init from a chunk with no visible key at all
    attn.attn_fwd_merge(q, dev_bf16(KB), dev_bf16(VB), acc, lacc, init=True, O_out=O,
                        scale=scale, k_lens=torch.zeros(2, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.all(acc == 0) and torch.all(O == 0) and torch.all(torch.isneginf(lacc))


def test_fwd_merge_buffers_aligned_to_16_bytes_only():
    """The fused fold with O_acc and O_out 16-byte but not 32-byte aligned (the
    boundary asks for 16): the epilogue then moves 16 bytes at a time; the results
    are bit-identical to buffers at 32-byte boundaries."""
    import torch

    attn = _lib()
    B, H, Lq, LA, LB, d = 1, 2, 200, 260, 140, 128
    Q = synth.normal_bf16(9311, (B, H, Lq, d))
    KA, VA = synth.normal_bf16(9312, (B, H, LA, d)), synth.normal_bf16(9313, (B, H, LA, d))
    KB, VB = synth.normal_bf16(9314, (B, H, LB, d)), synth.normal_bf16(9315, (B, H, LB, d))
    q = dev_bf16(Q)
    n = B * H * Lq * d
    outs = []
    for shift in (0, 4):  # 0 or 4 fp32 (16 bytes) past a 32-byte boundary
        acc_big = torch.empty(n + 8, dtype=torch.float32, device="cuda")
        o_big = torch.empty(n + 16, dtype=torch.bfloat16, device="cuda")
        acc = acc_big[shift:shift + n].view(B, H, Lq, d)
        O = o_big[2 * shift:2 * shift + n].view(B, H, Lq, d)
        assert acc.data_ptr() % 32 == 4 * shift and O.data_ptr() % 32 == 4 * shift
        lacc = torch.empty((B, H, Lq), dtype=torch.float32, device="cuda")
        attn.attn_fwd_merge(q, dev_bf16(KA), dev_bf16(VA), acc, lacc, init=True)
        attn.attn_fwd_merge(q, dev_bf16(KB), dev_bf16(VB), acc, lacc, init=False, O_out=O)
        torch.cuda.synchronize()
        outs.append((acc.clone(), lacc.clone(), O.clone()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)
    Oref, Lref = oracle.fwd(Q, np.concatenate([KA, KB], axis=2), np.concatenate([VA, VB], axis=2),
                            1.0 / math.sqrt(d))
    assert_out_close(to_f64(outs[1][2]), Oref)
    assert_lse_close(to_f64(outs[1][1]), Lref)


def test_merge_and_accumulate_accumulators_aligned_to_16_bytes_only():
    """attn_merge_partial and attn_accumulate with fp32 accumulators 16-byte but not
    32-byte aligned (the boundary asks for 16): bit-identical results to accumulators
    at 32-byte boundaries (the kernels then move 16 bytes at a time)."""
    import torch

    attn = _lib()
    rows, d = 700, 128
    Ob = dev_bf16(synth.normal_bf16(9500, (rows, d)))
    lb = torch.from_numpy((np.random.default_rng(9501).standard_normal(rows) * 3)
                          .astype(np.float32)).cuda()
    A0 = torch.from_numpy(np.random.default_rng(9502).standard_normal((rows, d))
                          .astype(np.float32)).cuda()
    l0 = torch.from_numpy(np.random.default_rng(9503).standard_normal(rows)
                          .astype(np.float32)).cuda()
    parts = [dev_bf16(synth.normal_bf16(9510 + i, (rows, d))) for i in range(2)]
    results = []
    for shift in (0, 4):  # fp32 elements past a 32-byte boundary
        big = torch.empty(rows * d + 8, dtype=torch.float32, device="cuda")
        acc = big[shift:shift + rows * d].view(rows, d)
        assert acc.data_ptr() % 32 == 4 * shift
        acc.copy_(A0)
        lacc = l0.clone()
        attn.attn_merge_partial(Ob, lb, acc, lacc, init=False)
        merged = acc.clone()
        attn.attn_accumulate(parts[0], acc, init=True)
        attn.attn_accumulate(parts[1], acc, init=False)
        torch.cuda.synchronize()
        results.append((merged, lacc.clone(), acc.clone()))
    for a, b in zip(results[0], results[1]):
        assert torch.equal(a, b)
    assert torch.equal(results[1][2], parts[0].float() + parts[1].float())


def test_accumulate_kernel():
    import torch

    attn = _lib()
    parts = [dev_bf16(synth.normal_bf16(9400 + i, (3, 5, 64))) for i in range(3)]
    acc = torch.full((3, 5, 64), 7.0, device="cuda")
    out = torch.empty((3, 5, 64), dtype=torch.bfloat16, device="cuda")
    attn.attn_accumulate(parts[0], acc, init=True)
    attn.attn_accumulate(parts[1], acc, init=False)
    attn.attn_accumulate(parts[2], acc, init=False, out=out)
    torch.cuda.synchronize()
    ref = parts[0].float() + parts[1].float() + parts[2].float()
    assert torch.equal(acc, ref) and torch.equal(out, ref.to(torch.bfloat16))
    attn.attn_accumulate(None, acc, init=False, out=out)  # convert only
    torch.cuda.synchronize()
    assert torch.equal(acc, ref)


@pytest.mark.parametrize("world,causal,Hq,Hkv,Lc,d", [
    (2, True, 4, 2, 200, 128),
    (3, True, 2, 2, 130, 128),
    (3, False, 2, 1, 150, 128),   # the backward kernels take d = 128
])
def test_ring_backward_decomposition_matches_whole_sequence(world, causal, Hq, Hkv, Lc, d):
    """Each rank's steps (bwd_chunk from the whole-sequence O and LSE, partials
    summed in fp32 by attn_accumulate; each key chunk's dK/dV summed over every
    rank) against the oracle's gradients of the whole sequence."""
    import torch

    from exact_io_aware_46_b200.ring import bwd_chunk

    attn = _lib()
    L = world * Lc
    seed = 9500 + world * 10 + Lc
    Q = synth.normal_bf16(seed * 8 + 1, (1, Hq, L, d))
    K = synth.normal_bf16(seed * 8 + 2, (1, Hkv, L, d))
    V = synth.normal_bf16(seed * 8 + 3, (1, Hkv, L, d))
    dO = synth.normal_bf16(seed * 8 + 4, (1, Hq, L, d))
    q, k, v, do = (dev_bf16(x) for x in (Q, K, V, dO))
    scale = 1.0 / math.sqrt(d)
    O, Lse = attn.attn_fwd(q, k, v, scale=scale, causal=causal)
    rQ, rK, rV = oracle.bwd(Q, K, V, dO, scale, causal=causal)
    sl = [slice(c * Lc, (c + 1) * Lc) for c in range(world)]
    dk_acc = [torch.zeros((1, Hkv, Lc, d), device="cuda") for _ in range(world)]
    dv_acc = [torch.zeros((1, Hkv, Lc, d), device="cuda") for _ in range(world)]
    dq = torch.empty_like(q)
    for rank in range(world):
        qr, orr, dor = (t[:, :, sl[rank]].contiguous() for t in (q, O, do))
        lr = Lse[:, :, sl[rank]].contiguous()
        dq_acc = torch.empty((1, Hq, Lc, d), device="cuda")
        first = True
        for _, src, kind in ring_steps(rank, world, causal):
            part = bwd_chunk(qr, k[:, :, sl[src]].contiguous(), v[:, :, sl[src]].contiguous(),
                             orr, dor, lr, kind, scale=scale)
            if part is None:
                continue
            attn.attn_accumulate(part[0], dq_acc, init=first)
            first = False
            attn.attn_accumulate(part[1], dk_acc[src], init=False)
            attn.attn_accumulate(part[2], dv_acc[src], init=False)
        out = torch.empty_like(qr)
        attn.attn_accumulate(None, dq_acc, init=False, out=out)
        dq[:, :, sl[rank]] = out
    torch.cuda.synchronize()
    dk = torch.cat(dk_acc, dim=2)
    dv = torch.cat(dv_acc, dim=2)
    from tests._util import GRAD_REL_L2, rel_l2
    for got, ref, what in ((dq, rQ, "dQ"), (dk, rK, "dK"), (dv, rV, "dV")):
        assert rel_l2(to_f64(got), ref) <= GRAD_REL_L2, f"{what}: {rel_l2(to_f64(got), ref):.3e}"


@pytest.mark.parametrize("world,Hq,Hkv,Lc", [(2, 4, 2, 150), (3, 2, 2, 130)])
def test_ring_zigzag_decomposition_matches_whole_sequence(world, Hq, Hkv, Lc):
    """The causal zigzag layout (rank r holds chunks r and 2*world-1-r): every
    rank's folds from zigzag_folds on the CUDA kernels, chunks taken from one
    tensor, against the oracle's whole-sequence attention."""
    import torch

    from exact_io_aware_46_b200.ring import zigzag_chunks, zigzag_folds

    d = 128
    L = 2 * world * Lc
    seed = 9700 + world * 10 + Lc
    Q = synth.normal_bf16(seed * 4 + 1, (1, Hq, L, d))
    K = synth.normal_bf16(seed * 4 + 2, (1, Hkv, L, d))
    V = synth.normal_bf16(seed * 4 + 3, (1, Hkv, L, d))
    q_all, k_all, v_all = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    scale = 1.0 / math.sqrt(d)
    Oref, Lref = oracle.fwd(Q, K, V, scale, causal=True)
    ch = lambda t, c: t[:, :, c * Lc:(c + 1) * Lc]
    for rank in range(world):
        mine = zigzag_chunks(rank, world)
        qs = [ch(q_all, c).contiguous() for c in mine]
        acc = [torch.empty((1, Hq, Lc, d), device="cuda") for _ in range(2)]
        lacc = [torch.empty((1, Hq, Lc), device="cuda") for _ in range(2)]
        O = [torch.empty((1, Hq, Lc, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        for _, src, qi, ki, kind, first, last in zigzag_folds(rank, world):
            c = zigzag_chunks(src, world)[ki]
            fold_chunk(qs[qi], ch(k_all, c).contiguous(), ch(v_all, c).contiguous(), kind,
                       acc[qi], lacc[qi], first=first, O_out=O[qi] if last else None,
                       scale=scale)
        torch.cuda.synchronize()
        for qi in (0, 1):
            assert_out_close(to_f64(O[qi]), ch(Oref, mine[qi]), f"O[rank {rank}, chunk {qi}]")
            assert_lse_close(to_f64(lacc[qi]), ch(Lref, mine[qi]))


@pytest.mark.parametrize("world,Hq,Hkv,Lc", [(2, 4, 2, 140), (3, 2, 2, 100)])
def test_ring_zigzag_backward_matches_whole_sequence(world, Hq, Hkv, Lc):
    """Zigzag backward decomposition: every rank's pairs (bwd_chunk from the
    whole-sequence O and LSE) summed in fp32, each key chunk's dK/dV over every
    rank, against the oracle's whole-sequence gradients."""
    import torch

    from exact_io_aware_46_b200.ring import bwd_chunk, ring_steps_zigzag, zigzag_chunks

    attn = _lib()
    d = 128
    L = 2 * world * Lc
    seed = 9900 + world * 10 + Lc
    Q = synth.normal_bf16(seed * 8 + 1, (1, Hq, L, d))
    K = synth.normal_bf16(seed * 8 + 2, (1, Hkv, L, d))
    V = synth.normal_bf16(seed * 8 + 3, (1, Hkv, L, d))
    dO = synth.normal_bf16(seed * 8 + 4, (1, Hq, L, d))
    q, k, v, do = (dev_bf16(x) for x in (Q, K, V, dO))
    scale = 1.0 / math.sqrt(d)
    O, Lse = attn.attn_fwd(q, k, v, scale=scale, causal=True)
    rQ, rK, rV = oracle.bwd(Q, K, V, dO, scale, causal=True)
    ch = lambda t, c: t[:, :, c * Lc:(c + 1) * Lc].contiguous()
    n = 2 * world
    dq_acc = [torch.empty((1, Hq, Lc, d), device="cuda") for _ in range(n)]
    dk_acc = [torch.zeros((1, Hkv, Lc, d), device="cuda") for _ in range(n)]
    dv_acc = [torch.zeros((1, Hkv, Lc, d), device="cuda") for _ in range(n)]
    started = set()
    for rank in range(world):
        mine = zigzag_chunks(rank, world)
        for _, src, pairs in ring_steps_zigzag(rank, world):
            held = zigzag_chunks(src, world)
            for qi, ki, kind in pairs:
                a, b = mine[qi], held[ki]
                dqp, dkp, dvp = bwd_chunk(ch(q, a), ch(k, b), ch(v, b), ch(O, a), ch(do, a),
                                          ch(Lse, a), kind, scale=scale)
                attn.attn_accumulate(dqp, dq_acc[a], init=a not in started)
                started.add(a)
                attn.attn_accumulate(dkp, dk_acc[b], init=False)
                attn.attn_accumulate(dvp, dv_acc[b], init=False)
    torch.cuda.synchronize()
    from tests._util import GRAD_REL_L2, rel_l2
    for got, ref, what in ((torch.cat(dq_acc, 2), rQ, "dQ"), (torch.cat(dk_acc, 2), rK, "dK"),
                           (torch.cat(dv_acc, 2), rV, "dV")):
        assert rel_l2(to_f64(got), ref) <= GRAD_REL_L2, f"{what}: {rel_l2(to_f64(got), ref):.3e}"
