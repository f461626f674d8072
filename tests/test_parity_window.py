"""Sliding-window (local causal) attention: attn_fwd_sliding / attn_bwd_sliding
against the fp64 oracle with the same window, and the wide-window limit
against the causal entry points."""

import math

import numpy as np
import pytest

import oracle
import synth
from tests._util import (GRAD_REL_L2, assert_lse_close, assert_out_close, dev_bf16, rel_l2,
                         to_f64)

pytestmark = pytest.mark.gpu


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


FWD_CASES = [
    # B, Hq, Hkv, Lq, Lk, d, window, k_lens
    (2, 4, 2, 700, 700, 128, 1, None),          # only the diagonal key
    (2, 4, 2, 700, 700, 128, 100, None),        # window inside one key tile
    (1, 2, 2, 700, 700, 128, 128, None),        # exactly one tile wide
    (1, 2, 1, 700, 700, 128, 129, None),
    (1, 2, 2, 600, 600, 128, 300, [600]),
    (1, 2, 2, 300, 900, 128, 256, None),        # Lq < Lk: bottom-right alignment
    (2, 2, 2, 513, 513, 64, 200, [513, 301]),   # d = 64, key padding
    (1, 2, 2, 500, 300, 128, 64, None),         # Lq > Lk: the first 200 rows see no key
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,window,k_lens", FWD_CASES)
def test_sliding_fwd_matches_oracle(B, Hq, Hkv, Lq, Lk, d, window, k_lens):
    import torch

    attn = _lib()
    seed = 7100 + Lq + Lk + window + d
    Q = synth.normal_bf16(seed * 16 + 1, (B, Hq, Lq, d))
    K = synth.normal_bf16(seed * 16 + 2, (B, Hkv, Lk, d))
    V = synth.normal_bf16(seed * 16 + 3, (B, Hkv, Lk, d))
    scale = 1.0 / math.sqrt(d)
    kl = None if k_lens is None else torch.tensor(k_lens, dtype=torch.int32, device="cuda")
    O, L = attn.attn_fwd_sliding(dev_bf16(Q), dev_bf16(K), dev_bf16(V), window, scale=scale,
                                 k_lens=kl)
    torch.cuda.synchronize()
    Oref, Lref = oracle.fwd(Q, K, V, scale, causal=True, k_lens=k_lens, window=window)
    assert_out_close(to_f64(O), Oref)
    assert_lse_close(to_f64(L), Lref)


def test_wide_window_equals_causal_forward_bitwise():
    import torch

    attn = _lib()
    Q = dev_bf16(synth.normal_bf16(7301, (1, 4, 1000, 128)))
    K = dev_bf16(synth.normal_bf16(7302, (1, 2, 1000, 128)))
    V = dev_bf16(synth.normal_bf16(7303, (1, 2, 1000, 128)))
    O1, L1 = attn.attn_fwd(Q, K, V, causal=True)
    O2, L2 = attn.attn_fwd_sliding(Q, K, V, 1000)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


BWD_CASES = [
    # B, Hq, Hkv, Lq, Lk, window
    (1, 2, 2, 400, 400, 1),
    (1, 2, 2, 400, 400, 150),
    (1, 4, 2, 300, 300, 64),     # grouped heads, window of one query tile
    (1, 2, 2, 200, 500, 200),    # Lq < Lk
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,window", BWD_CASES)
def test_sliding_bwd_matches_oracle(B, Hq, Hkv, Lq, Lk, window):
    import torch

    attn = _lib()
    d = 128
    seed = 7500 + Lq + Lk + window
    Q = synth.normal_bf16(seed * 16 + 1, (B, Hq, Lq, d))
    K = synth.normal_bf16(seed * 16 + 2, (B, Hkv, Lk, d))
    V = synth.normal_bf16(seed * 16 + 3, (B, Hkv, Lk, d))
    dO = synth.normal_bf16(seed * 16 + 4, (B, Hq, Lq, d))
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (dev_bf16(x) for x in (Q, K, V, dO))
    O, L = attn.attn_fwd_sliding(q, k, v, window)
    dq, dk, dv = attn.attn_bwd_sliding(q, k, v, O, do, L, window)
    torch.cuda.synchronize()
    rQ, rK, rV = oracle.bwd(Q, K, V, dO, scale, causal=True, window=window)
    for got, ref, what in ((dq, rQ, "dQ"), (dk, rK, "dK"), (dv, rV, "dV")):
        g = to_f64(got)
        assert np.all(np.isfinite(g)), what
        if np.linalg.norm(ref) == 0:
            # W = 1: dS = P (dP - D) is exactly zero; the GPU leaves rounding noise
            # (D is formed from the bf16 O), orders of magnitude below any real error
            assert np.max(np.abs(g)) <= 1e-5, f"{what}: max {np.max(np.abs(g)):.3e}"
        else:
            assert rel_l2(g, ref) <= GRAD_REL_L2, f"{what}: rel-L2 {rel_l2(g, ref):.3e}"


def test_sliding_fwd_long_sequence_sampled_rows():
    """B=1, H=4, L=8192, window 1024 (a common local-attention width): sampled
    rows, including the first window and tile boundaries, against the oracle."""
    import torch

    attn = _lib()
    H, L, d, W = 4, 8192, 128, 1024
    Q = synth.normal_bf16(7701, (1, H, L, d))
    K = synth.normal_bf16(7702, (1, H, L, d))
    V = synth.normal_bf16(7703, (1, H, L, d))
    O, Lse = attn.attn_fwd_sliding(dev_bf16(Q), dev_bf16(K), dev_bf16(V), W)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 1023, 1024, 1025, 4095, 4096, 5000, 8190, 8191]
    Oref, Lref = oracle.fwd(Q, K, V, 1.0 / math.sqrt(d), causal=True, rows=rows, window=W)
    assert_out_close(to_f64(O)[:, :, rows], Oref)
    assert_lse_close(to_f64(Lse)[:, :, rows], Lref)
