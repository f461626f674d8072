"""Paged-KV split decode: the attention of the contiguous decode, with the cache
read through a block table.  Checked against the fp64 oracle on the logical
cache, and bit for bit against the contiguous entry point (same chunks, same
row order, so the same sums)."""

import math

import numpy as np
import pytest

import oracle
import synth
from tests._util import assert_lse_close, assert_out_close, dev_bf16, to_f64

pytestmark = pytest.mark.gpu

FILL = 0x42C8  # bf16 100.0: pages nobody references hold it, so a misread shows


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


def _page_order(seed, n):
    """A seeded permutation of n page indices."""
    return np.argsort(synth.uniform_u64(seed, n), kind="stable").astype(np.int32)


def _scatter(K, page, order):
    """Logical cache [B,Hkv,Lmax,d] (bf16 bits) -> pages [n_pages,Hkv,page,d] and
    block table [B, max_blocks]; logical block (b, j) goes to page order[b*nb+j]."""
    B, Hkv, Lmax, d = K.shape
    nb = (Lmax + page - 1) // page
    n_pages = len(order)
    P = np.full((n_pages, Hkv, page, d), FILL, dtype=np.uint16)
    table = np.zeros((B, nb), dtype=np.int32)
    for b in range(B):
        for j in range(nb):
            pg = order[b * nb + j]
            table[b, j] = pg
            rows = K[b, :, j * page:min((j + 1) * page, Lmax), :]
            P[pg, :, :rows.shape[1], :] = rows
    return P, table


CASES = [
    # B, Hq, Hkv, Lmax, d, k_lens, page
    (3, 8, 2, 3000, 128, [2500, 1, 2048], 16),     # chunk boundary, single key, small pages
    (2, 4, 4, 2100, 128, [2049, 2100], 64),        # G = 1
    (2, 16, 2, 1500, 128, [1500, 777], 256),       # G = 8, pages larger than a stage
    (2, 4, 2, 1300, 64, [1300, 65], 32),           # d = 64
    (2, 8, 2, 1200, 128, [0, 1200], 128),          # an empty sequence
    (1, 4, 1, 5000, 128, [4097], 1024),            # three chunks inside large pages
    (2, 4, 2, 2200, 128, [128, 2177], 32),         # G = 2; a chunk of 129 keys over 32-row pages
    (2, 16, 2, 4200, 64, [4200, 2048], 16),        # d = 64, G = 8: three chunks over 16-row pages
]


@pytest.mark.parametrize("B,Hq,Hkv,Lmax,d,k_lens,page", CASES)
def test_paged_decode_matches_oracle_and_contiguous(B, Hq, Hkv, Lmax, d, k_lens, page):
    import torch

    attn = _lib()
    seed = 57 + Lmax + d + Hq + page
    Q = synth.normal_bf16(seed * 16 + 1, (B, Hq, 1, d))
    K = synth.normal_bf16(seed * 16 + 2, (B, Hkv, Lmax, d))
    V = synth.normal_bf16(seed * 16 + 3, (B, Hkv, Lmax, d))
    nb = (Lmax + page - 1) // page
    order = _page_order(seed * 16 + 4, B * nb + 3)  # three pages nobody references
    Kp, table = _scatter(K, page, order)
    Vp, _ = _scatter(V, page, order)
    scale = 1.0 / math.sqrt(d)
    kl = torch.tensor(k_lens, dtype=torch.int32, device="cuda")
    Qd = dev_bf16(Q)
    O, L = attn.attn_fwd_splitkv_decode_paged(Qd, dev_bf16(Kp), dev_bf16(Vp),
                                              torch.from_numpy(table).cuda(), kl, scale=scale)
    Oc, Lc = attn.attn_fwd_splitkv_decode(Qd, dev_bf16(K), dev_bf16(V), kl, scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(O, Oc) and torch.equal(L, Lc)
    Oref, Lref = oracle.fwd(Q, K, V, scale, causal=False, k_lens=k_lens)
    assert_out_close(to_f64(O), Oref)
    assert_lse_close(to_f64(L), Lref[:, :, 0])


def test_paged_decode_bad_block_table_entry_is_flagged_not_read():
    import torch

    attn = _lib()
    B, Hq, Hkv, Lmax, d, page = 2, 4, 1, 4096, 128, 64
    Q = synth.normal_bf16(901, (B, Hq, 1, d))
    K = synth.normal_bf16(902, (B, Hkv, Lmax, d))
    V = synth.normal_bf16(903, (B, Hkv, Lmax, d))
    order = _page_order(904, B * (Lmax // page))
    Kp, table = _scatter(K, page, order)
    Vp, _ = _scatter(V, page, order)
    n_pages = Kp.shape[0]
    table[1, 40] = n_pages      # sequence 1, second chunk (rows 2048..4095): out of range
    kl = torch.tensor([Lmax, Lmax], dtype=torch.int32, device="cuda")
    ws = torch.zeros(attn.attn_decode_workspace_size(B, Hq, Hkv, Lmax, d), dtype=torch.uint8,
                     device="cuda")
    O, L = attn.attn_fwd_splitkv_decode_paged(dev_bf16(Q), dev_bf16(Kp), dev_bf16(Vp),
                                              torch.from_numpy(table).cuda(), kl, workspace=ws)
    code, st = attn.attn_read_device_status(ws)
    assert code == attn.ATTN_ERR_INVALID and st & attn.ATTN_DEV_BAD_PAGE
    # sequence 0 is untouched; sequence 1 keeps the contribution of its first chunk
    Oref, Lref = oracle.fwd(Q, K, V, 1.0 / math.sqrt(d), causal=False, k_lens=[Lmax, 2048])
    assert_out_close(to_f64(O), Oref)
    assert_lse_close(to_f64(L), Lref[:, :, 0])


def test_paged_decode_full_size_equals_contiguous():
    """B=64, Hq=32, Hkv=8, d=128, cache 32768, k_len ~ U[1024, 32768], 64-row pages in a
    seeded random order: bit-identical to the contiguous path, which the contiguous
    decode tests check against the oracle at this size."""
    import torch

    attn = _lib()
    B, Hq, Hkv, Lmax, d, page = 64, 32, 8, 32768, 128, 64
    dev = torch.device("cuda")
    k_lens = synth.uniform_int(synth.workload_seed(4, "klen"), B, 1024, Lmax)
    q = synth.normal_bf16_device(synth.workload_seed(4, "q"), (B, Hq, 1, d), dev)
    kc = synth.normal_bf16_device(synth.workload_seed(4, "k"), (B, Hkv, Lmax, d), dev)
    vc = synth.normal_bf16_device(synth.workload_seed(4, "v"), (B, Hkv, Lmax, d), dev)
    kl = torch.from_numpy(k_lens).to(dev)
    nb = Lmax // page
    order = torch.from_numpy(_page_order(77, B * nb).astype(np.int64)).to(dev)
    table = order.view(B, nb).to(torch.int32).contiguous()

    def scatter(c):
        blocks = c.view(B, Hkv, nb, page, d).permute(0, 2, 1, 3, 4).reshape(B * nb, Hkv, page, d)
        out = torch.empty_like(blocks)
        out[order] = blocks
        return out

    kp, vp = scatter(kc), scatter(vc)
    O, L = attn.attn_fwd_splitkv_decode_paged(q, kp, vp, table, kl)
    Oc, Lc = attn.attn_fwd_splitkv_decode(q, kc, vc, kl)
    torch.cuda.synchronize()
    assert torch.equal(O, Oc) and torch.equal(L, Lc)
