"""The Python binding rejects mismatched tensors before any pointer reaches the
library.  A tensor the C side would read or write past its end (V smaller than
K, a short O or LSE), a host or other-GPU tensor the kernels would dereference
(k_lens on the CPU is an illegal address on the GPU), or an int64 k_lens that
the kernels would read as int32 must all raise ValueError on the host.

The tensors here are stand-ins that report a CUDA device, shape, dtype and
contiguity but hold no memory; taking a pointer from one fails the test, so
every rejection is shown to happen before the library is called.  Runs without
a GPU."""

import numpy as np
import pytest
import torch

import exact_io_aware_46_b200 as attn

BF, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


class FakeCuda:
    """Shape/dtype/device/contiguity of a CUDA tensor, without memory."""

    def __init__(self, shape, dtype, device="cuda:0", contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self._contiguous = contiguous

    @property
    def is_cuda(self):
        return self.device.type == "cuda"

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        return int(np.prod(self.shape, dtype=np.int64))

    def data_ptr(self):
        raise AssertionError("a pointer was taken before validation finished")


B, HQ, HKV, L, D = 2, 4, 2, 16, 128


def q():
    return FakeCuda((B, HQ, L, D), BF)


def kv(**kw):
    return FakeCuda((B, HKV, L, D), BF, **kw)


def rejects(fn, *words):
    with pytest.raises(ValueError) as e:
        fn()
    msg = str(e.value)
    for w in words:
        assert w in msg, f"{w!r} not in {msg!r}"


def test_fwd_shapes_dtypes_devices():
    rejects(lambda: attn.attn_fwd(q(), kv(), FakeCuda((B, HKV, L - 1, D), BF)), "V", "shape")
    rejects(lambda: attn.attn_fwd(q(), FakeCuda((B + 1, HKV, L, D), BF), kv()), "K")
    rejects(lambda: attn.attn_fwd(q(), FakeCuda((B, HKV, L, 64), BF), kv()), "K")
    rejects(lambda: attn.attn_fwd(q(), FakeCuda((B, 3, L, D), BF), FakeCuda((B, 3, L, D), BF)),
            "multiple")
    rejects(lambda: attn.attn_fwd(FakeCuda((B, HQ, D), BF), kv(), kv()), "[B, H, L, d]")
    rejects(lambda: attn.attn_fwd(q(), kv(device="cuda:1"), kv()), "K", "cuda:1")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(contiguous=False)), "V", "contiguous")
    rejects(lambda: attn.attn_fwd(q(), kv(), FakeCuda((B, HKV, L, D), F32)), "V", "bfloat16")
    # outputs smaller than the call writes, or of another dtype
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), O=FakeCuda((B, HQ, L - 1, D), BF)), "O")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), O=FakeCuda((B, HQ, L, D), F32)), "O")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), lse=FakeCuda((B, HQ), F32)), "lse")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), lse=FakeCuda((B, HQ, L), BF)), "lse")


def test_k_lens_dtype_length_device():
    # torch.tensor's default integer type is int64: read as int32 it would give
    # wrong lengths without an error
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), k_lens=FakeCuda((B,), torch.int64)),
            "k_lens", "int32")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), k_lens=FakeCuda((B + 1,), I32)), "k_lens")
    # on the host: the kernels would dereference a host pointer
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), k_lens=torch.zeros(B, dtype=I32)),
            "k_lens", "CUDA")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), k_lens=FakeCuda((B,), I32, "cuda:1")),
            "k_lens", "cuda:1")


def test_workspace_checks():
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), workspace=FakeCuda((256,), F32)), "workspace")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), workspace=FakeCuda((256,), U8, "cuda:1")),
            "workspace")
    rejects(lambda: attn.attn_fwd(q(), kv(), kv(), workspace=torch.zeros(256, dtype=U8)),
            "workspace", "CUDA")
    # the backward's workspace holds the fp32 dQ accumulator: 256 bytes are too few
    lse = FakeCuda((B, HQ, L), F32)
    rejects(lambda: attn.attn_bwd(q(), kv(), kv(), q(), q(), lse,
                                  workspace=FakeCuda((256,), U8)), "workspace", "needs")


def test_bwd_and_sliding():
    lse = FakeCuda((B, HQ, L), F32)
    rejects(lambda: attn.attn_bwd(q(), kv(), kv(), FakeCuda((B, HQ, L, 64), BF), q(), lse), "O")
    rejects(lambda: attn.attn_bwd(q(), kv(), kv(), q(), FakeCuda((B, HQ, L + 1, D), BF), lse),
            "dO")
    rejects(lambda: attn.attn_bwd(q(), kv(), kv(), q(), q(), FakeCuda((B, HQ, L - 1), F32)),
            "lse")
    rejects(lambda: attn.attn_bwd(q(), kv(), kv(), q(), q(), lse, dK=q()), "dK")
    rejects(lambda: attn.attn_bwd(q(), kv(), kv(), q(), q(), lse, dQ=kv()), "dQ")
    rejects(lambda: attn.attn_bwd_sliding(q(), kv(), kv(), q(), q(), lse, 8, dV=q()), "dV")
    rejects(lambda: attn.attn_fwd_sliding(q(), kv(), kv(), 8, O=kv()), "O")


def test_decode_and_paged():
    Qd = FakeCuda((B, HQ, 1, D), BF)
    cache = FakeCuda((B, HKV, 4096, D), BF)
    kl = FakeCuda((B,), I32)
    rejects(lambda: attn.attn_fwd_splitkv_decode(q(), cache, cache, kl), "Q", "1")
    rejects(lambda: attn.attn_fwd_splitkv_decode(Qd, cache, FakeCuda((B, HKV, 2048, D), BF), kl),
            "Vcache")
    rejects(lambda: attn.attn_fwd_splitkv_decode(Qd, FakeCuda((B + 1, HKV, 4096, D), BF),
                                                 FakeCuda((B + 1, HKV, 4096, D), BF), kl),
            "Kcache")
    rejects(lambda: attn.attn_fwd_splitkv_decode(Qd, cache, cache, None), "k_lens", "required")
    rejects(lambda: attn.attn_fwd_splitkv_decode(Qd, cache, cache, torch.zeros(B, dtype=I32)),
            "k_lens", "CUDA")
    rejects(lambda: attn.attn_fwd_splitkv_decode(Qd, cache, cache, kl, lse=FakeCuda((B,), F32)),
            "lse")
    rejects(lambda: attn.attn_fwd_splitkv_decode_noalloc(Qd, cache, cache,
                                                         FakeCuda((B,), torch.int64)), "k_lens")
    pages = FakeCuda((64, HKV, 64, D), BF)
    rejects(lambda: attn.attn_fwd_splitkv_decode_paged(Qd, pages, pages,
                                                       FakeCuda((B + 1, 8), I32), kl),
            "block_table")
    rejects(lambda: attn.attn_fwd_splitkv_decode_paged(Qd, pages, pages,
                                                       FakeCuda((B, 8), torch.int64), kl),
            "block_table")
    rejects(lambda: attn.attn_fwd_splitkv_decode_paged(Qd, pages, FakeCuda((64, HKV, 32, D), BF),
                                                       FakeCuda((B, 8), I32), kl), "Vpages")


def test_varlen():
    Qp = FakeCuda((100, HQ, D), BF)
    Kp = FakeCuda((120, HKV, D), BF)
    cu = FakeCuda((B + 1,), I32)
    rejects(lambda: attn.attn_fwd_varlen(Qp, Kp, FakeCuda((119, HKV, D), BF), cu, cu, 64, 64),
            "V")
    rejects(lambda: attn.attn_fwd_varlen(Qp, Kp, Kp, cu, FakeCuda((B + 2,), I32), 64, 64),
            "cu_seqlens_k")
    rejects(lambda: attn.attn_fwd_varlen(Qp, Kp, Kp, FakeCuda((B + 1,), torch.int64), cu, 64, 64),
            "cu_seqlens_q")
    rejects(lambda: attn.attn_fwd_varlen(Qp, Kp, Kp, cu, cu, 64, 64,
                                         lse=FakeCuda((100, HQ), F32)), "lse")


def test_fp8_merge_accumulate():
    q8 = FakeCuda((B, HQ, 200, D), U8)
    k8 = FakeCuda((B, HKV, 300, D), U8)
    qs = FakeCuda((B, HQ, 2), F32)
    ks = FakeCuda((B, HKV, 3), F32)
    rejects(lambda: attn.attn_fwd_fp8(q8, k8, k8, qs, FakeCuda((B, HKV, 2), F32), ks), "k_scale")
    rejects(lambda: attn.attn_fwd_fp8(q8, k8, k8, qs, ks, FakeCuda((B, HKV, 3), BF)), "v_scale")
    rejects(lambda: attn.attn_fwd_fp8(q8, FakeCuda((B, HKV, 300, D), BF), k8, qs, ks, ks), "K8")
    acc = FakeCuda((B, HQ, L, D), F32)
    lacc = FakeCuda((B, HQ, L), F32)
    rejects(lambda: attn.attn_fwd_merge(q(), kv(), kv(), FakeCuda((B, HQ, L, 64), F32), lacc,
                                        init=True), "O_acc")
    rejects(lambda: attn.attn_fwd_merge(q(), kv(), kv(), acc, FakeCuda((B, HQ, L), BF),
                                        init=True), "lse_acc")
    rejects(lambda: attn.attn_accumulate(FakeCuda((B, HQ, L, 64), BF), acc, init=True), "part")
    rejects(lambda: attn.attn_accumulate(q(), acc, init=True, out=FakeCuda((8,), BF)), "out")
    rejects(lambda: attn.attn_merge_partial(q(), FakeCuda((B, HQ), F32), acc, lacc, init=True),
            "lse_part")
    rejects(lambda: attn.attn_merge_partial(q(), lacc, acc, FakeCuda((B, HQ, L + 1), F32),
                                            init=True), "lse_acc")
