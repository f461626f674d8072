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
