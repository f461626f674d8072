"""Python binding of the B200 exact-attention C library (``libattn.so``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/attn.h``.  PyTorch provides device
memory and the stream.  There is no CPU or library fallback: if the compiled
library is missing, every call raises.

The functions carry the C entry points' names:

* ``attn_fwd(Q, K, V, ...) -> (O, LSE)``
* ``attn_fwd_varlen(Q, K, V, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, ...) -> (O, LSE)``
* ``attn_fwd_splitkv_decode(Q, Kcache, Vcache, k_lens, ...) -> (O, LSE)``
* ``attn_fwd_splitkv_decode_paged(Q, Kpages, Vpages, block_table, k_lens, ...) -> (O, LSE)``
* ``attn_bwd(Q, K, V, O, dO, LSE, ...) -> (dQ, dK, dV)``
* ``attn_fwd_sliding`` / ``attn_bwd_sliding``: the same with a sliding-window causal mask
* ``attn_fwd_fp8(Q8, K8, V8, q_scale, k_scale, v_scale, ...) -> (O, LSE)``: E4M3 inputs with
  one scale per 128-row tile
* the ``*_workspace_size`` queries and the device-status helpers.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

(ATTN_OK, ATTN_ERR_INVALID, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT,
 ATTN_ERR_CAPACITY) = range(6)
#: size of the fixed device scratch used by attn_fwd_splitkv_decode_noalloc
ATTN_NOALLOC_SCRATCH_BYTES = 16 << 20
ATTN_MASK_NONE, ATTN_MASK_CAUSAL = 0, 1
ATTN_DEV_BAD_KLEN, ATTN_DEV_TIMEOUT, ATTN_DEV_BAD_PAGE, ATTN_DEV_BAD_SCALE = 1, 2, 4, 8

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_f = ctypes.c_float

#: exported symbol -> (restype, argtypes); mirrors include/attn.h
SIGNATURES = {
    "attn_status_string": (ctypes.c_char_p, [_i]),
    "attn_num_sms": (_i, []),
    "attn_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _sz,
                      _vp]),
    "attn_fwd_sliding": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp,
                              _sz, _vp]),
    "attn_fwd_merge": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp,
                            _vp, _sz, _vp]),
    "attn_accumulate": (_i, [_vp, _vp, _vp, ctypes.c_longlong, _i, _vp]),
    "attn_merge_partial": (_i, [_vp, _vp, _vp, _vp, _vp, ctypes.c_longlong, _i, _i, _vp]),
    "attn_fwd_fp8": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i,
                          _vp, _vp, _sz, _vp]),
    "attn_bwd_sliding": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                              _f, _i, _vp, _vp, _sz, _vp]),
    "attn_fwd_varlen_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_fwd_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                             _f, _i, _vp, _sz, _vp]),
    "attn_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "attn_fwd_splitkv_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp,
                                     _sz, _vp]),
    "attn_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f,
                      _i, _vp, _vp, _sz, _vp]),
    "attn_fwd_splitkv_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f,
                                             _vp, _vp]),
    "attn_fwd_splitkv_decode_paged": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _i, _i,
                                           _i, _f, _vp, _vp, _sz, _vp]),
    "attn_read_device_status": (_i, [_vp, _vp, ctypes.POINTER(ctypes.c_int32)]),
    "attn_clear_device_status": (_i, [_vp, _vp]),
}


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"CUDA library not built: {LIB_PATH} is missing "
                    "(run `python -m exact_io_aware_46_b200.build`); there is no fallback")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().attn_status_string(int(code)).decode()
    except RuntimeError:
        return "library not loaded"


def _check(code: int, where: str) -> None:
    if code != ATTN_OK:
        raise AttnError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bf16(t, name):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor")


def _workspace(nbytes: int, device, stream):
    ws = torch.empty(max(256, int(nbytes)), dtype=torch.uint8, device=device)
    _check(lib().attn_clear_device_status(_ptr(ws), _stream(stream)), "attn_clear_device_status")
    return ws


def attn_num_sms() -> int:
    return int(lib().attn_num_sms())


def attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d) -> int:
    return int(lib().attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d))


def attn_fwd_varlen_workspace_size(B, Hq, Hkv, max_seqlen_q, max_seqlen_k, d) -> int:
    return int(lib().attn_fwd_varlen_workspace_size(B, Hq, Hkv, max_seqlen_q, max_seqlen_k, d))


def attn_decode_workspace_size(B, Hq, Hkv, Lmax, d) -> int:
    return int(lib().attn_decode_workspace_size(B, Hq, Hkv, Lmax, d))


def attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d) -> int:
    return int(lib().attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d))


def attn_read_device_status(workspace, stream=None) -> tuple[int, int]:
    bits = ctypes.c_int32(0)
    code = lib().attn_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(bits))
    return int(code), int(bits.value)


def attn_clear_device_status(workspace, stream=None) -> None:
    _check(lib().attn_clear_device_status(_ptr(workspace), _stream(stream)),
           "attn_clear_device_status")


def attn_fwd(Q, K, V, scale=None, causal=False, k_lens=None, O=None, lse=None, workspace=None,
             stream=None, want_lse=True):
    """Forward attention.  Q [B,Hq,Lq,d], K/V [B,Hkv,Lk,d] bf16 on the GPU.

    Returns (O, LSE) with O bf16 [B,Hq,Lq,d] and LSE fp32 [B,Hq,Lq] (None if
    ``want_lse`` is False)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _bf16(t, n)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _workspace(attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), Q.device, stream)
    code = lib().attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), B, Hq, Hkv, Lq, Lk, d,
                          float(scale), ATTN_MASK_CAUSAL if causal else ATTN_MASK_NONE,
                          _ptr(k_lens), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_fwd")
    return O, lse


def _u8(t, name):
    if t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA uint8 tensor of E4M3 codes")


def _f32(t, name):
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA float32 tensor")


def attn_fwd_fp8(Q8, K8, V8, q_scale, k_scale, v_scale, scale=None, causal=False, k_lens=None,
                 O=None, lse=None, workspace=None, stream=None, want_lse=True):
    """Forward of E4M3 inputs.  Q8 [B,Hq,Lq,d], K8/V8 [B,Hkv,Lk,d] uint8 codes;
    q_scale [B,Hq,ceil(Lq/128)], k_scale/v_scale [B,Hkv,ceil(Lk/128)] fp32 (one
    scale per 128-row tile).  Returns (O bf16 [B,Hq,Lq,d], LSE fp32 [B,Hq,Lq])."""
    for t, n in ((Q8, "Q8"), (K8, "K8"), (V8, "V8")):
        _u8(t, n)
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        _f32(t, n)
    B, Hq, Lq, d = Q8.shape
    Hkv, Lk = K8.shape[1], K8.shape[2]
    if tuple(q_scale.shape) != (B, Hq, (Lq + 127) // 128) or \
            tuple(k_scale.shape) != (B, Hkv, (Lk + 127) // 128) or \
            tuple(v_scale.shape) != (B, Hkv, (Lk + 127) // 128):
        raise ValueError("one scale per 128-row tile of each head expected")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty((B, Hq, Lq, d), dtype=torch.bfloat16, device=Q8.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=Q8.device)
    if workspace is None:
        workspace = _workspace(attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), Q8.device, stream)
    code = lib().attn_fwd_fp8(_ptr(Q8), _ptr(K8), _ptr(V8), _ptr(q_scale), _ptr(k_scale),
                              _ptr(v_scale), _ptr(O), _ptr(lse), B, Hq, Hkv, Lq, Lk, d,
                              float(scale), ATTN_MASK_CAUSAL if causal else ATTN_MASK_NONE,
                              _ptr(k_lens), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_fp8")
    return O, lse


def attn_fwd_merge(Q, K, V, O_acc, lse_acc, init, O_out=None, scale=None, causal=False,
                   k_lens=None, workspace=None, stream=None):
    """attn_fwd over K/V (a subset of the keys), folded into the fp32 accumulator
    (O_acc [B,Hq,Lq,d], lse_acc [B,Hq,Lq]) in place with the normalised merge
    rule (``init``: overwrite it instead); ``O_out`` (bf16, optional) receives
    the merged O."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _bf16(t, n)
    for t, n in ((O_acc, "O_acc"), (lse_acc, "lse_acc")):
        _f32(t, n)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    if tuple(O_acc.shape) != (B, Hq, Lq, d) or tuple(lse_acc.shape) != (B, Hq, Lq) or \
            (O_out is not None and tuple(O_out.shape) != (B, Hq, Lq, d)):
        raise ValueError("accumulator shapes must match Q")
    if O_out is not None:
        _bf16(O_out, "O_out")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        workspace = _workspace(attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), Q.device, stream)
    code = lib().attn_fwd_merge(_ptr(Q), _ptr(K), _ptr(V), _ptr(O_acc), _ptr(lse_acc),
                                _ptr(O_out), 1 if init else 0, B, Hq, Hkv, Lq, Lk, d,
                                float(scale), ATTN_MASK_CAUSAL if causal else ATTN_MASK_NONE,
                                _ptr(k_lens), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_merge")


def attn_accumulate(part, acc, init, out=None, stream=None):
    """acc (fp32) += part (bf16), or acc = part with ``init``; ``part`` None adds
    nothing; ``out`` (bf16, optional) receives the sum."""
    _f32(acc, "acc")
    if part is not None:
        _bf16(part, "part")
        if part.shape != acc.shape:
            raise ValueError("partial and accumulator shapes differ")
    if out is not None:
        _bf16(out, "out")
        if out.shape != acc.shape:
            raise ValueError("output and accumulator shapes differ")
    code = lib().attn_accumulate(_ptr(part), _ptr(acc), _ptr(out), acc.numel(),
                                 1 if init else 0, _stream(stream))
    _check(code, "attn_accumulate")


def attn_merge_partial(O_part, lse_part, O_acc, lse_acc, init, O_out=None, stream=None):
    """Fold a partial result (O_part bf16 [..., d], lse_part fp32 [...]) into the
    fp32 accumulator (O_acc, lse_acc) in place (``init``: overwrite it instead);
    ``O_out`` (bf16, optional) also receives the merged O."""
    _bf16(O_part, "O_part")
    for t, n in ((lse_part, "lse_part"), (O_acc, "O_acc"), (lse_acc, "lse_acc")):
        _f32(t, n)
    if O_out is not None:
        _bf16(O_out, "O_out")
    d = O_part.shape[-1]
    rows = O_part.numel() // d if d else 0
    if O_acc.shape != O_part.shape or lse_part.numel() != rows or lse_acc.numel() != rows or \
            (O_out is not None and O_out.shape != O_part.shape):
        raise ValueError("partial, accumulator and output shapes differ")
    code = lib().attn_merge_partial(_ptr(O_part), _ptr(lse_part), _ptr(O_acc), _ptr(lse_acc),
                                    _ptr(O_out), rows, d, 1 if init else 0, _stream(stream))
    _check(code, "attn_merge_partial")


def attn_fwd_sliding(Q, K, V, window, scale=None, k_lens=None, O=None, lse=None, workspace=None,
                     stream=None, want_lse=True):
    """Sliding-window causal forward: row i sees its ``window`` latest keys."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _bf16(t, n)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _workspace(attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), Q.device, stream)
    code = lib().attn_fwd_sliding(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), B, Hq, Hkv, Lq,
                                  Lk, d, float(scale), int(window), _ptr(k_lens), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_sliding")
    return O, lse


def attn_bwd_sliding(Q, K, V, O, dO, lse, window, scale=None, k_lens=None, dQ=None, dK=None,
                     dV=None, workspace=None, stream=None):
    """Backward of attn_fwd_sliding.  Returns (dQ, dK, dV) bf16."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O"), (dO, "dO")):
        _bf16(t, n)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    if workspace is None:
        workspace = _workspace(attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), Q.device, stream)
    code = lib().attn_bwd_sliding(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), B, Hq, Hkv, Lq, Lk, d,
                                  float(scale), int(window), _ptr(k_lens), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _check(code, "attn_bwd_sliding")
    return dQ, dK, dV


def attn_fwd_varlen(Q, K, V, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                    scale=None, causal=False, O=None, lse=None, workspace=None, stream=None,
                    want_lse=True):
    """Forward over packed sequences.  Q [total_q,Hq,d], K/V [total_k,Hkv,d] bf16;
    cu_seqlens_q / cu_seqlens_k int32 [B+1] on the device.  LSE is [Hq, total_q]."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _bf16(t, n)
    total_q, Hq, d = Q.shape
    total_k, Hkv = K.shape[0], K.shape[1]
    B = cu_seqlens_q.numel() - 1
    if cu_seqlens_k.numel() != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _workspace(attn_fwd_varlen_workspace_size(B, Hq, Hkv, max_seqlen_q,
                                                              max_seqlen_k, d), Q.device, stream)
    code = lib().attn_fwd_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                 _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, Hq, Hkv,
                                 int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, d,
                                 float(scale), ATTN_MASK_CAUSAL if causal else ATTN_MASK_NONE,
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_varlen")
    return O, lse


def attn_fwd_splitkv_decode(Q, Kc, Vc, k_lens, scale=None, O=None, lse=None, workspace=None,
                            stream=None, want_lse=True):
    """Split-KV decode.  Q [B,Hq,1,d]; Kc/Vc [B,Hkv,Lmax,d] bf16; k_lens int32 [B] (device)."""
    for t, n in ((Q, "Q"), (Kc, "Kcache"), (Vc, "Vcache")):
        _bf16(t, n)
    B, Hq, _, d = Q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _workspace(attn_decode_workspace_size(B, Hq, Hkv, Lmax, d), Q.device, stream)
    code = lib().attn_fwd_splitkv_decode(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(O), _ptr(lse), B, Hq,
                                         Hkv, Lmax, d, float(scale), _ptr(k_lens),
                                         _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_splitkv_decode")
    return O, lse


def attn_fwd_splitkv_decode_paged(Q, Kp, Vp, block_table, k_lens, scale=None, O=None, lse=None,
                                  workspace=None, stream=None, want_lse=True):
    """Split-KV decode over a paged cache.  Q [B,Hq,1,d]; Kp/Vp [n_pages,Hkv,page,d] bf16;
    block_table int32 [B,max_blocks] and k_lens int32 [B] on the device."""
    for t, n in ((Q, "Q"), (Kp, "Kpages"), (Vp, "Vpages")):
        _bf16(t, n)
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 [B, max_blocks] tensor")
    B, Hq, _, d = Q.shape
    n_pages, Hkv, page = Kp.shape[0], Kp.shape[1], Kp.shape[2]
    max_blocks = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _workspace(attn_decode_workspace_size(B, Hq, Hkv, max_blocks * page, d),
                               Q.device, stream)
    code = lib().attn_fwd_splitkv_decode_paged(_ptr(Q), _ptr(Kp), _ptr(Vp), _ptr(block_table),
                                               max_blocks, page, n_pages, _ptr(O), _ptr(lse), B,
                                               Hq, Hkv, d, float(scale), _ptr(k_lens),
                                               _ptr(workspace), workspace.numel(),
                                               _stream(stream))
    _check(code, "attn_fwd_splitkv_decode_paged")
    return O, lse


def attn_fwd_splitkv_decode_noalloc(Q, Kc, Vc, k_lens, scale=None, O=None, lse=None,
                                    stream=None, want_lse=True):
    """Split-KV decode without a workspace, for callers that cannot allocate
    device memory (the library call itself allocates nothing; this wrapper only
    creates O / LSE when they are not passed in).  Calls that overlap on the
    GPU share one fixed scratch array and race: serialise them."""
    for t, n in ((Q, "Q"), (Kc, "Kcache"), (Vc, "Vcache")):
        _bf16(t, n)
    B, Hq, _, d = Q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=Q.device)
    code = lib().attn_fwd_splitkv_decode_noalloc(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(O), _ptr(lse),
                                                 B, Hq, Hkv, Lmax, d, float(scale),
                                                 _ptr(k_lens), _stream(stream))
    _check(code, "attn_fwd_splitkv_decode_noalloc")
    return O, lse


def attn_bwd(Q, K, V, O, dO, lse, scale=None, causal=False, k_lens=None, dQ=None, dK=None,
             dV=None, workspace=None, stream=None):
    """Backward.  Returns (dQ, dK, dV) bf16."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O"), (dO, "dO")):
        _bf16(t, n)
    B, Hq, Lq, d = Q.shape
    Hkv, Lk = K.shape[1], K.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    if workspace is None:
        workspace = _workspace(attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), Q.device, stream)
    code = lib().attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse), _ptr(dQ),
                          _ptr(dK), _ptr(dV), B, Hq, Hkv, Lq, Lk, d, float(scale),
                          ATTN_MASK_CAUSAL if causal else ATTN_MASK_NONE, _ptr(k_lens),
                          _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_bwd")
    return dQ, dK, dV
