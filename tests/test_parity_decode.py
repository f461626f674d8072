"""Split-KV decode parity: CUDA split + combine kernels against the fp64 oracle."""

import math

import numpy as np
import pytest

import oracle
import synth
from tests._util import assert_lse_close, assert_out_close, bits, dev_bf16, to_f64

pytestmark = pytest.mark.gpu


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


def _run(Q, K, V, k_lens, scale):
    import torch

    attn = _lib()
    kl = torch.tensor(k_lens, dtype=torch.int32, device="cuda")
    O, L = attn.attn_fwd_splitkv_decode(dev_bf16(Q), dev_bf16(K), dev_bf16(V), kl, scale=scale)
    torch.cuda.synchronize()
    return to_f64(O), to_f64(L)


CASES = [
    # B, Hq, Hkv, Lmax, d, k_lens
    (3, 8, 2, 3000, 128, [2500, 1, 2048]),        # chunk boundary, single key, exact chunk
    (1, 4, 1, 5000, 128, [4097]),                 # three chunks, the last holding one key
    (2, 4, 4, 2100, 128, [2049, 2100]),           # G = 1
    (2, 16, 2, 1500, 128, [1500, 777]),           # G = 8
    (2, 4, 2, 1300, 64, [1300, 65]),              # d = 64, G = 2
    (2, 8, 2, 1200, 128, [0, 1200]),              # an empty sequence
    (1, 4, 1, 70, 128, [70]),                     # shorter than one stage
    (2, 4, 2, 2200, 128, [128, 2177]),            # G = 2; one whole 128-key block; a chunk of 129 keys
    (2, 16, 2, 4500, 64, [4500, 2049]),           # d = 64, G = 8: three chunks, the last of one key
    (2, 4, 4, 2100, 64, [0, 2100]),               # d = 64, G = 1: an empty sequence, two chunks
]


@pytest.mark.parametrize("B,Hq,Hkv,Lmax,d,k_lens", CASES)
def test_decode_matches_oracle(B, Hq, Hkv, Lmax, d, k_lens):
    seed = 31 + Lmax + d + Hq
    Q = synth.normal_bf16(seed * 16 + 1, (B, Hq, 1, d))
    K = synth.normal_bf16(seed * 16 + 2, (B, Hkv, Lmax, d))
    V = synth.normal_bf16(seed * 16 + 3, (B, Hkv, Lmax, d))
    scale = 1.0 / math.sqrt(d)
    O, L = _run(Q, K, V, k_lens, scale)
    Oref, Lref = oracle.fwd(Q, K, V, scale, causal=False, k_lens=k_lens)
    assert_out_close(O, Oref)
    assert_lse_close(L, Lref[:, :, 0])


@pytest.mark.parametrize("d", [64, 128])
def test_decode_large_logits(d):
    """Scale 1 (scores of size ~sqrt(d)): each head's probabilities concentrate on a
    few keys across several 2048-key chunks, so the chunks' partial maxima differ by
    tens of log2 units in the combine.  |O| then reaches ~4, so the absolute O bar is
    scaled by max(1, |O_ref|) as in the forward's large-logit test."""
    B, Hq, Hkv, Lmax = 2, 8, 2, 4600
    k_lens = [4600, 2100]
    Q = synth.normal_bf16(9900 + d, (B, Hq, 1, d))
    K = synth.normal_bf16(9910 + d, (B, Hkv, Lmax, d))
    V = synth.normal_bf16(9920 + d, (B, Hkv, Lmax, d))
    O, L = _run(Q, K, V, k_lens, 1.0)
    Oref, Lref = oracle.fwd(Q, K, V, 1.0, causal=False, k_lens=k_lens)
    err = np.abs(O - Oref)
    bound = 1e-2 * np.maximum(1.0, np.abs(Oref))
    assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3f}"
    assert_lse_close(L, Lref[:, :, 0])


def test_decode_deterministic_and_status():
    import torch

    attn = _lib()
    Q = dev_bf16(synth.normal_bf16(1, (2, 4, 1, 128)))
    K = dev_bf16(synth.normal_bf16(2, (2, 1, 900, 128)))
    V = dev_bf16(synth.normal_bf16(3, (2, 1, 900, 128)))
    kl = torch.tensor([900, 901], dtype=torch.int32, device="cuda")
    ws = torch.zeros(attn.attn_decode_workspace_size(2, 4, 1, 900, 128), dtype=torch.uint8,
                     device="cuda")
    O1, L1 = attn.attn_fwd_splitkv_decode(Q, K, V, kl, workspace=ws)
    O2, L2 = attn.attn_fwd_splitkv_decode(Q, K, V, kl, workspace=ws)
    code, st = attn.attn_read_device_status(ws)
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    assert code == attn.ATTN_ERR_INVALID and st & attn.ATTN_DEV_BAD_KLEN
    assert torch.all(O1[1] == 0) and torch.all(torch.isneginf(L1[1]))


def test_decode_full_size_sampled():
    """B=64, Hq=32, Hkv=8, d=128, cache [64,8,32768,128], k_len ~ U[1024, 32768]."""
    import torch

    attn = _lib()
    B, Hq, Hkv, Lmax, d = 64, 32, 8, 32768, 128
    seed = 4604
    k_lens = synth.uniform_int(seed * 16 + 5, B, 1024, Lmax)
    q = synth.normal_bf16_device(seed * 16 + 1, (B, Hq, 1, d), "cuda")
    k = synth.normal_bf16_device(seed * 16 + 2, (B, Hkv, Lmax, d), "cuda")
    v = synth.normal_bf16_device(seed * 16 + 3, (B, Hkv, Lmax, d), "cuda")
    kl = torch.from_numpy(k_lens).to("cuda")
    O, L = attn.attn_fwd_splitkv_decode(q, k, v, kl)
    torch.cuda.synchronize()
    G = Hq // Hkv
    for b in (0, int(np.argmax(k_lens)), int(np.argmin(k_lens)), 37):
        n = int(k_lens[b])
        Qb = bits(q[b:b + 1])
        Kb = bits(k[b:b + 1, :, :n])
        Vb = bits(v[b:b + 1, :, :n])
        Oref, Lref = oracle.fwd(Qb, Kb, Vb, 1 / math.sqrt(d))
        assert_out_close(to_f64(O[b:b + 1]), Oref, f"O[{b}]")
        assert_lse_close(to_f64(L[b:b + 1]), Lref[:, :, 0])
    del q, k, v
    torch.cuda.empty_cache()
