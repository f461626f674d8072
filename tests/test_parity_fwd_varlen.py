"""Forward over packed variable-length sequences (attn_fwd_varlen): every
sequence must equal attn_fwd run on that sequence alone (same tiles, same
order, so bit for bit) and the fp64 oracle within the forward tolerances."""

import math

import numpy as np
import pytest

import oracle
import synth
from tests._util import assert_lse_close, assert_out_close, dev_bf16, to_f64

pytestmark = pytest.mark.gpu


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


def _pack(seed, lens, H, d):
    """Per-sequence tensors [1, H, L, d] (bf16 bits) and their packed [sum L, H, d] form."""
    seqs = [synth.normal_bf16(seed + 7 * i, (1, H, L, d)) for i, L in enumerate(lens)]
    packed = np.concatenate([s[0].transpose(1, 0, 2) for s in seqs], axis=0) if lens else None
    return seqs, packed


CASES = [
    # lens_q, lens_k, Hq, Hkv, d, causal
    ([300, 1, 777, 256], [300, 1, 777, 256], 4, 2, 128, True),
    ([300, 1, 777, 256], [300, 1, 777, 256], 4, 2, 128, False),
    ([130, 511], [700, 900], 2, 1, 128, True),     # Lk > Lq: bottom-right causal alignment
    ([0, 200, 0, 129], [0, 330, 5, 129], 4, 4, 64, True),  # empty sequences, d = 64
    ([1000], [1000], 8, 2, 128, True),            # one sequence: same as the batched layout
]


@pytest.mark.parametrize("lens_q,lens_k,Hq,Hkv,d,causal", CASES)
def test_varlen_matches_single_sequence_calls_and_oracle(lens_q, lens_k, Hq, Hkv, d, causal):
    import torch

    attn = _lib()
    seed = 4100 + sum(lens_q) + d + Hq
    qs, Qp = _pack(seed, lens_q, Hq, d)
    ks, Kp = _pack(seed + 1000, lens_k, Hkv, d)
    vs, Vp = _pack(seed + 2000, lens_k, Hkv, d)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32, device="cuda")
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32, device="cuda")
    scale = 1.0 / math.sqrt(d)
    O, L = attn.attn_fwd_varlen(dev_bf16(Qp), dev_bf16(Kp), dev_bf16(Vp), cu_q, cu_k,
                                max(lens_q), max(lens_k), scale=scale, causal=causal)
    torch.cuda.synchronize()
    for i, (lq, lk) in enumerate(zip(lens_q, lens_k)):
        if lq == 0:
            continue
        q0 = int(cu_q[i])
        Oi = O[q0:q0 + lq].permute(1, 0, 2).unsqueeze(0)
        Li = L[:, q0:q0 + lq].unsqueeze(0)
        Os, Ls = attn.attn_fwd(dev_bf16(qs[i]), dev_bf16(ks[i]), dev_bf16(vs[i]), scale=scale,
                               causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(Oi, Os) and torch.equal(Li, Ls), f"sequence {i}"
        Oref, Lref = oracle.fwd(qs[i], ks[i], vs[i], scale, causal=causal)
        assert_out_close(to_f64(Oi), Oref, f"O[seq {i}]")
        assert_lse_close(to_f64(Li), Lref)


def test_varlen_malformed_offsets_are_flagged_and_skipped():
    import torch

    attn = _lib()
    Hq, Hkv, d = 2, 1, 128
    lens = [200, 300]
    qs, Qp = _pack(77, lens, Hq, d)
    ks, Kp = _pack(78, lens, Hkv, d)
    vs, Vp = _pack(79, lens, Hkv, d)
    # sequence 1 claims to end past total_q: skipped, sequence 0 still computed
    cu_q = torch.tensor([0, 200, 600], dtype=torch.int32, device="cuda")
    cu_k = torch.tensor([0, 200, 500], dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    O = torch.full((500, Hq, d), 7.0, dtype=torch.bfloat16, device="cuda")
    O, L = attn.attn_fwd_varlen(dev_bf16(Qp), dev_bf16(Kp), dev_bf16(Vp), cu_q, cu_k, 400, 300,
                                causal=True, O=O, workspace=ws)
    code, st = attn.attn_read_device_status(ws)
    assert code == attn.ATTN_ERR_INVALID and st & attn.ATTN_DEV_BAD_KLEN
    assert torch.all(O[200:] == 7.0)  # the skipped sequence's rows are untouched
    Oref, Lref = oracle.fwd(qs[0], ks[0], vs[0], 1.0 / math.sqrt(d), causal=True)
    assert_out_close(to_f64(O[:200].permute(1, 0, 2).unsqueeze(0)), Oref)
