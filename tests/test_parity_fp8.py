"""8-bit forward (attn_fwd_fp8): E4M3 Q, K, V with one scale per 128-row tile,
against the fp64 oracle's exact attention of the dequantised tensors.

Tolerances (derived from the arithmetic, not fitted): S = Q K^T is exact up to
fp32 summation, so LSE keeps the forward's bar.  P is rounded to E4M3 (3
mantissa bits, relative rounding error at most 2^-4) before O += P V, so an
element of O is off by at most 2^-4 * max|V| plus fp32/bf16 rounding; the
rounding errors of independent probabilities add in quadrature, which puts the
relative L2 error near 2 % (a direct simulation of the rounding on N(0,1)
inputs gives 1.9-2.1 %), and the bar is twice that."""

import math

import numpy as np
import pytest

import oracle
import synth
from tests._util import assert_lse_close, rel_l2, to_f64

pytestmark = pytest.mark.gpu

FP8_O_REL_L2 = 4e-2
FP8_P_ROUNDING = 2.0 ** -4


def _lib():
    import exact_io_aware_46_b200 as attn

    return attn


def _dev(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _inputs(seed, B, Hq, Hkv, Lq, Lk, d=128):
    Q8, qs = synth.normal_e4m3(seed * 16 + 1, (B, Hq, Lq, d))
    K8, ks = synth.normal_e4m3(seed * 16 + 2, (B, Hkv, Lk, d))
    V8, vs = synth.normal_e4m3(seed * 16 + 3, (B, Hkv, Lk, d))
    return Q8, K8, V8, qs, ks, vs


def _check(O, L, Q8, K8, V8, qs, ks, vs, scale, causal, k_lens=None):
    Oref, Lref = oracle.fwd_fp8(Q8, K8, V8, qs, ks, vs, scale, causal=causal, k_lens=k_lens)
    got = to_f64(O)
    vmax = float(np.max(np.abs(oracle.dequant_tiles(V8, vs)))) if V8.size else 0.0
    err = float(np.max(np.abs(got - Oref))) if got.size else 0.0
    assert err <= FP8_P_ROUNDING * vmax + 1e-2, f"O max-abs {err:.3e} (max|V| {vmax:.3f})"
    assert rel_l2(got, Oref) <= FP8_O_REL_L2, f"O rel-L2 {rel_l2(got, Oref):.3e}"
    assert_lse_close(to_f64(L), Lref)


CASES = [
    # B, Hq, Hkv, Lq, Lk, causal, k_lens
    (2, 4, 2, 700, 700, True, None),          # several tiles, ragged tail, grouped heads
    (1, 2, 2, 300, 900, True, None),          # Lq < Lk: bottom-right alignment
    (2, 2, 1, 513, 513, False, [513, 301]),   # key padding, no causal mask
    (1, 2, 2, 128, 128, True, None),          # exactly one tile
    (1, 1, 1, 1, 1, False, None),             # one row, one key
    (1, 2, 2, 500, 300, True, None),          # Lq > Lk: the first 200 rows see no key
    (1, 4, 4, 1000, 1000, False, None),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,causal,k_lens", CASES)
def test_fp8_fwd_matches_oracle(B, Hq, Hkv, Lq, Lk, causal, k_lens):
    import torch

    attn = _lib()
    Q8, K8, V8, qs, ks, vs = _inputs(8100 + Lq + Lk + Hq, B, Hq, Hkv, Lq, Lk)
    scale = 1.0 / math.sqrt(128)
    kl = None if k_lens is None else torch.tensor(k_lens, dtype=torch.int32, device="cuda")
    O, L = attn.attn_fwd_fp8(_dev(Q8), _dev(K8), _dev(V8), _dev(qs), _dev(ks), _dev(vs),
                             scale=scale, causal=causal, k_lens=kl)
    torch.cuda.synchronize()
    _check(O, L, Q8, K8, V8, qs, ks, vs, scale, causal, k_lens)


def test_fp8_fwd_widely_spread_tile_scales():
    """Per-tile scales spread over 2^-6 .. 2^6 (K and V tiles of very different
    magnitude): the V scales are folded into P relative to the largest one."""
    import torch

    attn = _lib()
    Q8, K8, V8, qs, ks, vs = _inputs(8301, 1, 2, 2, 900, 900)
    nt = ks.shape[-1]
    spread = np.exp2(np.array([(j * 5) % 13 - 6 for j in range(nt)], dtype=np.float32))
    ks = (ks * spread[::-1]).astype(np.float32)
    vs = (vs * spread).astype(np.float32)
    O, L = attn.attn_fwd_fp8(_dev(Q8), _dev(K8), _dev(V8), _dev(qs), _dev(ks), _dev(vs),
                             scale=0.1, causal=True)
    torch.cuda.synchronize()
    _check(O, L, Q8, K8, V8, qs, ks, vs, 0.1, True)


def test_fp8_fwd_full_size_sampled():
    """The bench's workload, causal B4 H16 L4096 d128 in E4M3: sampled rows of
    a few heads (tile boundaries, first and last rows) against the oracle."""
    import torch

    attn = _lib()
    B, H, L, d = 4, 16, 4096, 128
    dev = torch.device("cuda")
    q8, qs = synth.normal_e4m3_device(synth.workload_seed(1, "q"), (B, H, L, d), dev)
    k8, ks = synth.normal_e4m3_device(synth.workload_seed(1, "k"), (B, H, L, d), dev)
    v8, vs = synth.normal_e4m3_device(synth.workload_seed(1, "v"), (B, H, L, d), dev)
    O, Lse = attn.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=True)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 255, 256, 1000, 2047, 2048, 3071, 4095]
    for b, h in ((0, 0), (1, 7), (3, 15)):
        sl = slice(h, h + 1)
        args = [t[b:b + 1, sl].cpu().numpy() for t in (q8, k8, v8, qs, ks, vs)]
        Oref, Lref = oracle.fwd_fp8(*args, 1.0 / math.sqrt(d), causal=True, rows=rows)
        got = to_f64(O[b:b + 1, sl][:, :, rows])
        vmax = float(np.max(np.abs(oracle.dequant_tiles(args[2], args[5]))))
        assert np.max(np.abs(got - Oref)) <= FP8_P_ROUNDING * vmax + 1e-2
        assert rel_l2(got, Oref) <= FP8_O_REL_L2, f"({b},{h}) rel-L2 {rel_l2(got, Oref):.3e}"
        assert_lse_close(to_f64(Lse[b:b + 1, sl][:, :, rows]), Lref)


def test_fp8_bad_scale_is_flagged():
    """A zero or NaN scale sets ATTN_DEV_BAD_SCALE (nothing outside the buffers is touched)."""
    import torch

    attn = _lib()
    Q8, K8, V8, qs, ks, vs = _inputs(8401, 1, 2, 2, 300, 300)
    for bad_v in (0.0, float("nan")):
        vs2 = vs.copy()
        vs2[0, 1, 2] = bad_v
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        attn.attn_fwd_fp8(_dev(Q8), _dev(K8), _dev(V8), _dev(qs), _dev(ks), _dev(vs2),
                          causal=True, workspace=ws)
        code, st = attn.attn_read_device_status(ws)
        assert code == attn.ATTN_ERR_INVALID and st & attn.ATTN_DEV_BAD_SCALE
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    attn.attn_fwd_fp8(_dev(Q8), _dev(K8), _dev(V8), _dev(qs), _dev(ks), _dev(vs), causal=True,
                      workspace=ws)
    code, st = attn.attn_read_device_status(ws)
    assert code == attn.ATTN_OK and st == 0


@pytest.mark.parametrize("n_peak", [1, 2, 3])
def test_fp8_fwd_sharply_peaked_softmax(n_peak):
    """Scores dominated by a few keys per row (query i = beta times the sum of
    its n_peak chosen keys, so those keys score ~12 above the N(0,1) rest): the
    probabilities concentrate on n_peak entries, each rounded to E4M3 with a
    relative error of up to 2^-4 that no averaging over many keys hides.

    Bars, derived for this case: every O element stays within 2^-4 max|V|
    (+1e-2); with the mass on few keys, ||O_i - O_ref,i|| <= 2^-4 sum_j P_ij
    ||v_j|| ~ 2^-4 ||O_ref,i||, so the relative L2 error is held to 2^-4 rather
    than the many-key bar; LSE keeps the forward's bar (S is exact up to fp32
    sums)."""
    import torch

    attn = _lib()
    B, H, L, d = 1, 2, 384, 128
    rng = np.random.default_rng(8300 + n_peak)
    Kf = synth.bf16_bits_to_f64(synth.normal_bf16(8310 + n_peak, (B, H, L, d)))
    Vf = synth.bf16_bits_to_f64(synth.normal_bf16(8320 + n_peak, (B, H, L, d)))
    beta = 12.0 * math.sqrt(d) / d  # scale * beta * |k|^2 ~ 12 for |k|^2 ~ d
    Qf = 0.1 * synth.bf16_bits_to_f64(synth.normal_bf16(8330 + n_peak, (B, H, L, d)))
    for h in range(H):
        for i in range(L):
            keys = rng.choice(L, size=n_peak, replace=False)
            Qf[0, h, i] += beta * Kf[0, h, keys].sum(axis=0)
    q8, qs = synth.quantize_e4m3_tiles(torch.from_numpy(Qf.astype(np.float32)))
    k8, ks = synth.quantize_e4m3_tiles(torch.from_numpy(Kf.astype(np.float32)))
    v8, vs = synth.quantize_e4m3_tiles(torch.from_numpy(Vf.astype(np.float32)))
    Q8, K8, V8, QS, KS, VS = (t.numpy() for t in (q8, k8, v8, qs, ks, vs))
    scale = 1.0 / math.sqrt(d)
    O, Lse = attn.attn_fwd_fp8(_dev(Q8), _dev(K8), _dev(V8), _dev(QS), _dev(KS), _dev(VS),
                               scale=scale, causal=False)
    torch.cuda.synchronize()
    Oref, Lref = oracle.fwd_fp8(Q8, K8, V8, QS, KS, VS, scale, causal=False)
    # the construction worked: each row's n_peak largest probabilities hold most of its mass
    P, _ = oracle.probs(oracle.dequant_tiles(Q8, QS)[0, 0], oracle.dequant_tiles(K8, KS)[0, 0],
                        scale)
    top = np.sort(P, axis=1)[:, -n_peak:].sum(axis=1)
    assert np.median(top) > 0.9
    got = to_f64(O)
    vmax = float(np.max(np.abs(oracle.dequant_tiles(V8, VS))))
    err = float(np.max(np.abs(got - Oref)))
    assert err <= FP8_P_ROUNDING * vmax + 1e-2, f"O max-abs {err:.3e} (max|V| {vmax:.3f})"
    assert rel_l2(got, Oref) <= FP8_P_ROUNDING, f"O rel-L2 {rel_l2(got, Oref):.3e}"
    assert_lse_close(to_f64(Lse), Lref)
