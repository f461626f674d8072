"""attn_fwd_splitkv_decode_noalloc: decode for callers that cannot allocate.

Callers inside a runtime whose device memory plan is fixed up front, or
behind an operator interface that passes tensors but no allocator, cannot hand
the library a workspace.  The no-alloc entry point keeps its partials in a
fixed device array instead.  It
must give the same output as the workspace entry point, call after call (the
array keeps the previous call's contents, which must not leak into the next
result).

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""

import ctypes
import math

import numpy as np
import pytest

import synth
from tests._util import assert_lse_close, assert_out_close, dev_bf16, to_f64

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Hq, Hkv, Lmax, d):
    Q = dev_bf16(synth.normal_bf16(seed * 16 + 1, (B, Hq, 1, d)))
    K = dev_bf16(synth.normal_bf16(seed * 16 + 2, (B, Hkv, Lmax, d)))
    V = dev_bf16(synth.normal_bf16(seed * 16 + 3, (B, Hkv, Lmax, d)))
    return Q, K, V


def _noalloc_call(lib, Q, K, V, O, L, k_lens, scale):
    import torch

    B, Hq, _, d = Q.shape
    Hkv, Lmax = K.shape[1], K.shape[2]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.attn_fwd_splitkv_decode_noalloc(
        p(Q), p(K), p(V), p(O), p(L), B, Hq, Hkv, Lmax, d, scale, p(k_lens),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import torch

    import exact_io_aware_46_b200 as attn

    lib = attn.lib()
    B, Hq, Hkv, Lmax, d = 3, 8, 2, 2600, 128
    scale = 1.0 / math.sqrt(d)
    Q, K, V = _inputs(71, B, Hq, Hkv, Lmax, d)
    # two calls in a row with different lengths: stale partials of the first
    # call (two 2048-key chunks of sequence 0) must not reach the second
    for k_lens in ([2600, 1, 1024], [700, 2048, 0]):
        kl = torch.tensor(k_lens, dtype=torch.int32, device="cuda")
        ref_O, ref_L = attn.attn_fwd_splitkv_decode(Q, K, V, kl, scale=scale)
        O = torch.full_like(Q, float("nan"))
        L = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_call(lib, Q, K, V, O, L, kl, scale) == attn.ATTN_OK
        torch.cuda.synchronize()
        assert_out_close(to_f64(O), to_f64(ref_O))
        assert_lse_close(to_f64(L), to_f64(ref_L))


def test_noalloc_rejects_requests_beyond_its_scratch():
    import torch

    import exact_io_aware_46_b200 as attn

    lib = attn.lib()
    # 64 x 32 x 32 chunks of 128 fp32 outputs need ~34 MB > the fixed 16 MiB
    B, Hq, Hkv, Lmax, d = 64, 32, 8, 32768, 128
    Q = torch.zeros((B, Hq, 1, d), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1,), dtype=torch.bfloat16, device="cuda")  # never touched
    O = torch.empty_like(Q)
    kl = torch.zeros((B,), dtype=torch.int32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    code = lib.attn_fwd_splitkv_decode_noalloc(p(Q), p(K), p(K), p(O), None, B, Hq, Hkv, Lmax,
                                               d, 0.1, p(kl), None)
    assert code == attn.ATTN_ERR_CAPACITY
    assert attn.status_string(code).startswith("request exceeds")
