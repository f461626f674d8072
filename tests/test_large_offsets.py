"""Tensors of more than 2^31 elements: every element offset on the path is 64-bit.

The forward and the backward run on [1040, 16, 1040, 128] tensors (2.2e9 elements
each, ragged 1040-row tails) and the split decode on a [80, 8, 34000, 128] cache
(2.8e9 elements), contiguous and paged.  The oracle checks sampled outputs of
the first head, of the head whose rows cross element 2^31 and of the last head,
at the same bars as every other parity test."""

import math

import numpy as np
import pytest

import oracle
import synth
from tests._util import GRAD_REL_L2, assert_lse_close, assert_out_close, bits, rel_l2, to_f64

pytestmark = pytest.mark.gpu

B, H, L, D = 1040, 16, 1040, 128
# flat head index 16131 starts at element 16131 * 1040 * 128 = 2^31 - 124928, so its
# rows from 976 on lie past element 2^31; 16639 is the last head
HEADS = ((0, 0), (1008, 3), (1039, 15))


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


def test_fwd_and_bwd_beyond_2_31_elements():
    import torch

    attn = _lib()
    assert B * H * L * D > 2 ** 31 and (1008 * H + 3) * L * D < 2 ** 31 < (1008 * H + 4) * L * D
    seed = 4711
    shp = (B, H, L, D)
    q = synth.normal_bf16_device(seed * 16 + 1, shp, "cuda")
    k = synth.normal_bf16_device(seed * 16 + 2, shp, "cuda")
    v = synth.normal_bf16_device(seed * 16 + 3, shp, "cuda")
    do = synth.normal_bf16_device(seed * 16 + 4, shp, "cuda")
    O, Lse = attn.attn_fwd(q, k, v, causal=True)
    dq, dk, dv = attn.attn_bwd(q, k, v, O, do, Lse, causal=True)
    torch.cuda.synchronize()
    scale = 1 / math.sqrt(D)
    rows = np.array([0, 1, 127, 128, 975, 976, 977, 1023, 1024, L - 1], dtype=np.int32)
    cols = np.array([0, 127, 128, 511, 975, 976, 1024, L - 1], dtype=np.int32)
    for b, h in HEADS:
        sl = lambda t: bits(t[b:b + 1, h:h + 1])
        Qh, Kh, Vh, dOh = sl(q), sl(k), sl(v), sl(do)
        Oref, Lref = oracle.fwd(Qh, Kh, Vh, scale, causal=True, rows=rows)
        assert_out_close(to_f64(O[b, h, rows]), Oref[0, 0], f"O[{b},{h}]")
        assert_lse_close(to_f64(Lse[b, h, rows]), Lref[0, 0])
        rQ, rK, rV = oracle.bwd_sampled(Qh, Kh, Vh, dOh, scale, True, None, 0, 0, rows, cols)
        for name, got, ref in (("dQ", dq[b, h, rows], rQ[0]), ("dK", dk[b, h, cols], rK),
                               ("dV", dv[b, h, cols], rV)):
            err = rel_l2(to_f64(got), ref)
            assert err <= GRAD_REL_L2, f"{name}[{b},{h}]: rel-L2 {err:.3e}"
    del q, k, v, do, O, Lse, dq, dk, dv
    torch.cuda.empty_cache()


def test_decode_contiguous_and_paged_beyond_2_31_elements():
    import torch

    attn = _lib()
    Bd, Hq, Hkv, Lmax, d, page = 80, 32, 8, 34000, 128, 64
    assert Bd * Hkv * Lmax * d > 2 ** 31
    seed = 4712
    dev = torch.device("cuda")
    k_lens = synth.uniform_int(seed * 16 + 5, Bd, 1, Lmax)
    k_lens[-1] = Lmax  # the last sequence reads the cache's last row
    q = synth.normal_bf16_device(seed * 16 + 1, (Bd, Hq, 1, d), dev)
    kc = synth.normal_bf16_device(seed * 16 + 2, (Bd, Hkv, Lmax, d), dev)
    vc = synth.normal_bf16_device(seed * 16 + 3, (Bd, Hkv, Lmax, d), dev)
    kl = torch.from_numpy(k_lens).to(dev)
    O, Lse = attn.attn_fwd_splitkv_decode(q, kc, vc, kl)
    torch.cuda.synchronize()
    for b in (0, Bd - 1):
        n = int(k_lens[b])
        Oref, Lref = oracle.fwd(bits(q[b:b + 1]), bits(kc[b:b + 1, :, :n]),
                                bits(vc[b:b + 1, :, :n]), 1 / math.sqrt(d))
        assert_out_close(to_f64(O[b:b + 1]), Oref, f"O[{b}]")
        assert_lse_close(to_f64(Lse[b:b + 1]), Lref[:, :, 0])
    # the same cache as 64-row pages in a seeded random order: bit-identical results
    nb = (Lmax + page - 1) // page
    order = np.argsort(synth.uniform_u64(seed * 16 + 6, Bd * nb), kind="stable")
    order_t = torch.from_numpy(order.astype(np.int64)).to(dev)
    table = order_t.view(Bd, nb).to(torch.int32).contiguous()

    def scatter(c):
        pad = torch.zeros((Bd, Hkv, nb * page, d), dtype=c.dtype, device=dev)
        pad[:, :, :Lmax] = c
        blocks = pad.view(Bd, Hkv, nb, page, d).permute(0, 2, 1, 3, 4).reshape(Bd * nb, Hkv,
                                                                                page, d)
        out = torch.empty_like(blocks)
        out[order_t] = blocks
        return out

    kp = scatter(kc)
    del kc
    vp = scatter(vc)
    del vc
    torch.cuda.empty_cache()
    Op, Lp = attn.attn_fwd_splitkv_decode_paged(q, kp, vp, table, kl)
    torch.cuda.synchronize()
    assert torch.equal(Op, O) and torch.equal(Lp, Lse)
    del kp, vp
    torch.cuda.empty_cache()
