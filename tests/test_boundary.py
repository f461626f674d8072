"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects bad arguments on the host before launching anything."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_46_b200 import build

    build.build()
    import exact_io_aware_46_b200 as attn

    return attn.lib()


def test_every_declared_symbol_is_exported(lib):
    import exact_io_aware_46_b200 as attn

    names = _declared()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} missing from libattn.so"
        assert n in attn.SIGNATURES, f"{n} has no binding signature"


def test_workspace_sizes_are_closed_forms(lib):
    import exact_io_aware_46_b200 as attn

    assert attn.attn_fwd_workspace_size(4, 16, 16, 4096, 4096, 128) == 256
    # decode: fp32 partial output and log-sum-exp per (sequence, head, 2048-key chunk)
    n = 64 * 32 * 16
    assert attn.attn_decode_workspace_size(64, 32, 8, 32768, 128) == 256 + ((n * 128 * 4 + n * 4 + 255) // 256) * 256
    # backward: fp32 dQ accumulator (d columns), log2-LSE and D per query row;
    # nothing of size Lq x Lk
    rows = 2 * 16 * 8192  # query rows, padded per head to a multiple of 128
    assert attn.attn_bwd_workspace_size(2, 16, 16, 8192, 8192, 128) == 256 + ((rows * 128 * 4 + rows * 8 + 255) // 256) * 256
    rows = 1 * 2 * 128  # Lq = 100 pads to 128
    assert attn.attn_bwd_workspace_size(1, 2, 1, 100, 300, 128) == 256 + ((rows * 128 * 4 + rows * 8 + 255) // 256) * 256
    rows = 1 * 2 * 256  # Lq = 200 pads to 256; d = 64 accumulates 64 columns
    assert attn.attn_bwd_workspace_size(1, 2, 1, 200, 300, 64) == 256 + ((rows * 64 * 4 + rows * 8 + 255) // 256) * 256


def test_status_strings(lib):
    import exact_io_aware_46_b200 as attn

    assert attn.status_string(0) == "ok"
    assert attn.status_string(2) == "unsupported"


# Host-side validation happens before any CUDA call, so these run without a GPU.
P = ctypes.c_void_p(256 * 1024)  # a 256-byte aligned non-null stand-in, never dereferenced


def _fwd(lib, **kw):
    a = dict(Q=P, K=P, V=P, O=P, lse=None, B=1, Hq=2, Hkv=1, Lq=8, Lk=8, d=128, scale=0.1,
             mask=0, k_lens=None, ws=P, ws_bytes=256, stream=None)
    a.update(kw)
    return lib.attn_fwd(a["Q"], a["K"], a["V"], a["O"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                        a["Lq"], a["Lk"], a["d"], a["scale"], a["mask"], a["k_lens"], a["ws"],
                        a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(Q=None), 1), (dict(ws=None), 1), (dict(Hq=3, Hkv=2), 1), (dict(B=0), 1),
    (dict(Lq=-1), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(mask=7), 1),
    (dict(ws_bytes=16), 1), (dict(Q=ctypes.c_void_p(256 * 1024 + 8)), 1),
    (dict(ws=ctypes.c_void_p(256 * 1024 + 16)), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(Lq=0), 0),
])
def test_fwd_rejects_on_host(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_decode_and_bwd_reject_on_host(lib):
    # decode: k_lens are required; G = 3 is not a supported group size
    assert lib.attn_fwd_splitkv_decode(P, P, P, P, None, 1, 4, 1, 64, 128, 0.1, None, P,
                                       1 << 20, None) == 1
    assert lib.attn_fwd_splitkv_decode(P, P, P, P, None, 1, 3, 1, 64, 128, 0.1, P, P,
                                       1 << 20, None) == 2
    assert lib.attn_fwd_splitkv_decode(P, P, P, P, None, 1, 4, 1, 64, 72, 0.1, P, P,
                                       1 << 20, None) == 2
    # a cache of more than 65535 chunks of 2048 keys is refused, noalloc entry included
    big = 65535 * 2048 + 1
    assert lib.attn_fwd_splitkv_decode(P, P, P, P, None, 1, 4, 1, big, 128, 0.1, P, P,
                                       1 << 40, None) == 2
    assert lib.attn_fwd_splitkv_decode_noalloc(P, P, P, P, None, 1, 4, 1, big, 128, 0.1, P,
                                               None) == 2
    # bwd: lse is required; d must be 64 or 128
    assert lib.attn_bwd(P, P, P, P, P, None, P, P, P, 1, 1, 1, 8, 8, 128, 0.1, 0, None, P,
                        1 << 20, None) == 1
    assert lib.attn_bwd(P, P, P, P, P, P, P, P, P, 1, 1, 1, 8, 8, 80, 0.1, 0, None, P,
                        1 << 20, None) == 2


def test_paged_decode_rejects_on_host(lib):
    def call(bt=P, max_blocks=4, page=64, n_pages=8, d=128, ws_bytes=1 << 20, Hq=4):
        return lib.attn_fwd_splitkv_decode_paged(P, P, P, bt, max_blocks, page, n_pages, P, None,
                                                 1, Hq, 1, d, 0.1, P, P, ws_bytes, None)
    assert call(bt=None) == 1
    assert call(n_pages=0) == 1 and call(max_blocks=0) == 1
    assert call(page=24) == 2 and call(page=8) == 2 and call(page=1 << 17) == 2
    assert call(ws_bytes=64) == 1
    assert call(d=96) == 2 and call(Hq=3) == 2
    # 65536 pages of 2048 rows: more than 65535 chunks of 2048 keys
    assert call(max_blocks=65536, page=2048, ws_bytes=1 << 40) == 2


def test_varlen_fwd_rejects_on_host(lib):
    def call(cu=P, B=2, Hq=4, Hkv=2, mq=64, mk=64, tq=100, tk=100, d=128, mask=1, ws_bytes=256):
        return lib.attn_fwd_varlen(P, P, P, P, None, cu, cu, B, Hq, Hkv, mq, mk, tq, tk, d, 0.1,
                                   mask, P, ws_bytes, None)
    assert call(cu=None) == 1 and call(Hq=3) == 1 and call(tq=-1) == 1 and call(mask=5) == 1
    assert call(ws_bytes=16) == 1 and call(B=0) == 1
    assert call(d=80) == 2
    assert call(mq=0) == 0 and call(tq=0) == 0  # nothing to compute: returns at once


def test_sliding_rejects_on_host(lib):
    assert lib.attn_fwd_sliding(P, P, P, P, None, 1, 2, 1, 8, 8, 128, 0.1, 0, None, P, 256,
                                None) == 1
    assert lib.attn_fwd_sliding(P, P, P, P, None, 1, 2, 1, 8, 8, 96, 0.1, 4, None, P, 256,
                                None) == 2
    assert lib.attn_bwd_sliding(P, P, P, P, P, P, P, P, P, 1, 1, 1, 8, 8, 128, 0.1, -3, None, P,
                                1 << 20, None) == 1


def test_fp8_fwd_rejects_on_host(lib):
    def call(q=P, qs=P, d=128, mask=1, scale=0.1, ws_bytes=256, Lq=8, Hq=2):
        return lib.attn_fwd_fp8(q, P, P, qs, P, P, P, None, 1, Hq, 1, Lq, 8, d, scale, mask, None,
                                P, ws_bytes, None)
    assert call(q=None) == 1 and call(qs=None) == 1 and call(mask=3) == 1
    assert call(scale=-1.0) == 1 and call(ws_bytes=8) == 1 and call(Hq=0) == 1
    assert call(qs=ctypes.c_void_p(256 * 1024 + 4)) == 1  # scales must be 16-byte aligned
    assert call(d=64) == 2 and call(d=96) == 2
    assert call(Lq=0) == 0


def test_fwd_merge_and_merge_partial_reject_on_host(lib):
    def fm(acc=P, lse=P, init=1, d=128, mask=0, ws_bytes=256):
        return lib.attn_fwd_merge(P, P, P, acc, lse, None, init, 1, 2, 1, 8, 8, d, 0.1, mask,
                                  None, P, ws_bytes, None)
    assert fm(acc=None) == 1 and fm(lse=None) == 1 and fm(init=2) == 1 and fm(mask=4) == 1
    assert fm(ws_bytes=8) == 1 and fm(acc=ctypes.c_void_p(256 * 1024 + 4)) == 1
    assert fm(d=96) == 2

    def mp(d=128, rows=10, init=0, part=P):
        return lib.attn_merge_partial(part, P, P, P, None, rows, d, init, None)
    assert mp(d=96) == 1 and mp(d=512) == 1 and mp(rows=-1) == 1 and mp(init=3) == 1
    assert mp(part=None) == 1 and mp(rows=0) == 0
    # attn_accumulate: n a multiple of 8; no partial only when adding (convert)
    assert lib.attn_accumulate(P, P, None, 12, 0, None) == 1
    assert lib.attn_accumulate(None, P, None, 16, 1, None) == 1
    assert lib.attn_accumulate(P, None, None, 16, 0, None) == 1
    assert lib.attn_accumulate(P, P, None, 0, 0, None) == 0


def test_product_path_does_not_touch_oracle():
    """The CUDA binding must neither import nor load anything from oracle/."""
    pkg = os.path.join(ROOT, "exact_io_aware_46_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "attn_oracle" not in txt, f


def test_binding_refuses_host_tensors():
    """No CPU fallback: every entry point of the binding (and the ring drivers)
    rejects host tensors before anything runs."""
    import torch

    import exact_io_aware_46_b200 as attn
    from exact_io_aware_46_b200 import ring

    b = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    f = torch.zeros((1, 2, 8, 128), dtype=torch.float32)
    l = torch.zeros((1, 2, 8), dtype=torch.float32)
    u8 = torch.zeros((1, 2, 8, 128), dtype=torch.uint8)
    s = torch.ones((1, 2, 1), dtype=torch.float32)
    calls = [
        lambda: attn.attn_fwd(b, b, b),
        lambda: attn.attn_fwd_sliding(b, b, b, 4),
        lambda: attn.attn_bwd(b, b, b, b, b, l),
        lambda: attn.attn_fwd_fp8(u8, u8, u8, s, s, s),
        lambda: attn.attn_fwd_merge(b, b, b, f, l, init=True),
        lambda: attn.attn_merge_partial(b, l, f, l, init=True),
        lambda: attn.attn_accumulate(b, f, init=True),
        lambda: ring.ring_attn_fwd(b, b, b),
        lambda: ring.ring_attn_bwd(b, b, b, b, b, l),
        lambda: ring.ring_attn_fwd_zigzag((b, b), (b, b), (b, b)),
        lambda: ring.ring_attn_bwd_zigzag((b, b), (b, b), (b, b), (b, b), (b, b), (l, l)),
    ]
    for call in calls:
        with pytest.raises(ValueError):
            call()
