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
* ``attn_fwd_splitkv_decode_noalloc``: the split decode without a workspace (a fixed
  device array of ``ATTN_NOALLOC_SCRATCH_BYTES``)
* ``attn_fwd_merge``, ``attn_merge_partial``, ``attn_accumulate``: the folds of ring
  attention's partial results (``exact_io_aware_46_b200.ring`` drives them)
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


# ------------------------------------------------------------------ argument validation
# Every tensor handed to the library is checked here first: a host tensor, a
# tensor on another GPU, a wrong dtype or a shape smaller than the one the
# library derives from Q and K would otherwise reach the kernels as a raw
# pointer (an illegal address, or reads and writes past an allocation).  The
# checks use only shape, dtype, device and contiguity.

_DTYPE_NAMES = {torch.bfloat16: "bfloat16", torch.float32: "float32", torch.int32: "int32",
                torch.uint8: "uint8"}


def _need(t, name, dtype, shape=None, device=None):
    """``t`` must be a contiguous CUDA tensor of ``dtype`` (and ``shape`` and
    ``device`` when given)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor (host memory is not accepted; "
                         f"there is no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {_DTYPE_NAMES.get(dtype, dtype)}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other tensors on {device}")
    return t


def _opt(t, name, dtype, shape, device):
    """An optional tensor: None, or as ``_need``."""
    return None if t is None else _need(t, name, dtype, shape, device)


def _heads(Hq, Hkv):
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError(f"query heads ({Hq}) must be a multiple of key/value heads ({Hkv})")


def _qkv(Q, K, V, dtype=torch.bfloat16, names=("Q", "K", "V")):
    """Q [B,Hq,Lq,d], K and V [B,Hkv,Lk,d] of one dtype on one device.
    Returns (B, Hq, Hkv, Lq, Lk, d, device)."""
    _need(Q, names[0], dtype)
    if Q.dim() != 4:
        raise ValueError(f"{names[0]} must be [B, H, L, d], got {tuple(Q.shape)}")
    B, Hq, Lq, d = (int(x) for x in Q.shape)
    dev = Q.device
    _need(K, names[1], dtype, device=dev)
    if K.dim() != 4 or int(K.shape[0]) != B or int(K.shape[3]) != d:
        raise ValueError(f"{names[1]} must be [{B}, Hkv, Lk, {d}], got {tuple(K.shape)}")
    _need(V, names[2], dtype, tuple(K.shape), dev)
    Hkv, Lk = int(K.shape[1]), int(K.shape[2])
    _heads(Hq, Hkv)
    return B, Hq, Hkv, Lq, Lk, d, dev


def _klens(k_lens, B, dev, required=False):
    if k_lens is None:
        if required:
            raise ValueError("k_lens is required")
        return None
    return _need(k_lens, "k_lens", torch.int32, (B,), dev)


def _ws_check(ws, nbytes, dev):
    _need(ws, "workspace", torch.uint8, device=dev)
    if ws.numel() < nbytes:
        raise ValueError(f"workspace holds {ws.numel()} bytes, the call needs {nbytes}")
    return ws


def _bf16(t, name):
    _need(t, name, torch.bfloat16)


def _u8(t, name):
    _need(t, name, torch.uint8)


def _f32(t, name):
    _need(t, name, torch.float32)


def _workspace(nbytes: int, device, stream):
    ws = torch.empty(max(256, int(nbytes)), dtype=torch.uint8, device=device)
    _check(lib().attn_clear_device_status(_ptr(ws), _stream(stream)), "attn_clear_device_status")
    return ws


def _ws_or_new(workspace, nbytes, dev, stream):
    if workspace is None:
        return _workspace(nbytes, dev, stream)
    return _ws_check(workspace, nbytes, dev)


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


def _mask(causal):
    return ATTN_MASK_CAUSAL if causal else ATTN_MASK_NONE


def attn_fwd(Q, K, V, scale=None, causal=False, k_lens=None, O=None, lse=None, workspace=None,
             stream=None, want_lse=True):
    """Forward attention.  Q [B,Hq,Lq,d], K/V [B,Hkv,Lk,d] bf16 on the GPU.

    Returns (O, LSE) with O bf16 [B,Hq,Lq,d] and LSE fp32 [B,Hq,Lq] (None if
    ``want_lse`` is False)."""
    B, Hq, Hkv, Lq, Lk, d, dev = _qkv(Q, K, V)
    _klens(k_lens, B, dev)
    _opt(O, "O", torch.bfloat16, (B, Hq, Lq, d), dev)
    _opt(lse, "lse", torch.float32, (B, Hq, Lq), dev)
    workspace = _ws_or_new(workspace, attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=dev)
    code = lib().attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), B, Hq, Hkv, Lq, Lk, d,
                          float(scale), _mask(causal), _ptr(k_lens), _ptr(workspace),
                          workspace.numel(), _stream(stream))
    _check(code, "attn_fwd")
    return O, lse


def attn_fwd_fp8(Q8, K8, V8, q_scale, k_scale, v_scale, scale=None, causal=False, k_lens=None,
                 O=None, lse=None, workspace=None, stream=None, want_lse=True):
    """Forward of E4M3 inputs.  Q8 [B,Hq,Lq,d], K8/V8 [B,Hkv,Lk,d] uint8 codes;
    q_scale [B,Hq,ceil(Lq/128)], k_scale/v_scale [B,Hkv,ceil(Lk/128)] fp32 (one
    scale per 128-row tile).  Returns (O bf16 [B,Hq,Lq,d], LSE fp32 [B,Hq,Lq])."""
    B, Hq, Hkv, Lq, Lk, d, dev = _qkv(Q8, K8, V8, torch.uint8, ("Q8", "K8", "V8"))
    _need(q_scale, "q_scale", torch.float32, (B, Hq, (Lq + 127) // 128), dev)
    _need(k_scale, "k_scale", torch.float32, (B, Hkv, (Lk + 127) // 128), dev)
    _need(v_scale, "v_scale", torch.float32, (B, Hkv, (Lk + 127) // 128), dev)
    _klens(k_lens, B, dev)
    _opt(O, "O", torch.bfloat16, (B, Hq, Lq, d), dev)
    _opt(lse, "lse", torch.float32, (B, Hq, Lq), dev)
    workspace = _ws_or_new(workspace, attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty((B, Hq, Lq, d), dtype=torch.bfloat16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=dev)
    code = lib().attn_fwd_fp8(_ptr(Q8), _ptr(K8), _ptr(V8), _ptr(q_scale), _ptr(k_scale),
                              _ptr(v_scale), _ptr(O), _ptr(lse), B, Hq, Hkv, Lq, Lk, d,
                              float(scale), _mask(causal), _ptr(k_lens), _ptr(workspace),
                              workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_fp8")
    return O, lse


def attn_fwd_merge(Q, K, V, O_acc, lse_acc, init, O_out=None, scale=None, causal=False,
                   k_lens=None, workspace=None, stream=None):
    """attn_fwd over K/V (a subset of the keys), folded into the fp32 accumulator
    (O_acc [B,Hq,Lq,d], lse_acc [B,Hq,Lq]) in place with the normalised merge
    rule (``init``: overwrite it instead); ``O_out`` (bf16, optional) receives
    the merged O."""
    B, Hq, Hkv, Lq, Lk, d, dev = _qkv(Q, K, V)
    _need(O_acc, "O_acc", torch.float32, (B, Hq, Lq, d), dev)
    _need(lse_acc, "lse_acc", torch.float32, (B, Hq, Lq), dev)
    _opt(O_out, "O_out", torch.bfloat16, (B, Hq, Lq, d), dev)
    _klens(k_lens, B, dev)
    workspace = _ws_or_new(workspace, attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    code = lib().attn_fwd_merge(_ptr(Q), _ptr(K), _ptr(V), _ptr(O_acc), _ptr(lse_acc),
                                _ptr(O_out), 1 if init else 0, B, Hq, Hkv, Lq, Lk, d,
                                float(scale), _mask(causal), _ptr(k_lens), _ptr(workspace),
                                workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_merge")


def attn_accumulate(part, acc, init, out=None, stream=None):
    """acc (fp32) += part (bf16), or acc = part with ``init``; ``part`` None adds
    nothing; ``out`` (bf16, optional) receives the sum."""
    _need(acc, "acc", torch.float32)
    _opt(part, "part", torch.bfloat16, tuple(acc.shape), acc.device)
    _opt(out, "out", torch.bfloat16, tuple(acc.shape), acc.device)
    code = lib().attn_accumulate(_ptr(part), _ptr(acc), _ptr(out), acc.numel(),
                                 1 if init else 0, _stream(stream))
    _check(code, "attn_accumulate")


def attn_merge_partial(O_part, lse_part, O_acc, lse_acc, init, O_out=None, stream=None):
    """Fold a partial result (O_part bf16 [..., d], lse_part fp32 [...]) into the
    fp32 accumulator (O_acc, lse_acc) in place (``init``: overwrite it instead);
    ``O_out`` (bf16, optional) also receives the merged O."""
    _need(O_part, "O_part", torch.bfloat16)
    if O_part.dim() < 1:
        raise ValueError("O_part must have a trailing head dimension")
    dev = O_part.device
    rows_shape = tuple(O_part.shape[:-1])
    _need(lse_part, "lse_part", torch.float32, rows_shape, dev)
    _need(O_acc, "O_acc", torch.float32, tuple(O_part.shape), dev)
    _need(lse_acc, "lse_acc", torch.float32, rows_shape, dev)
    _opt(O_out, "O_out", torch.bfloat16, tuple(O_part.shape), dev)
    d = int(O_part.shape[-1])
    rows = O_part.numel() // d if d else 0
    code = lib().attn_merge_partial(_ptr(O_part), _ptr(lse_part), _ptr(O_acc), _ptr(lse_acc),
                                    _ptr(O_out), rows, d, 1 if init else 0, _stream(stream))
    _check(code, "attn_merge_partial")


def attn_fwd_sliding(Q, K, V, window, scale=None, k_lens=None, O=None, lse=None, workspace=None,
                     stream=None, want_lse=True):
    """Sliding-window causal forward: row i sees its ``window`` latest keys."""
    B, Hq, Hkv, Lq, Lk, d, dev = _qkv(Q, K, V)
    _klens(k_lens, B, dev)
    _opt(O, "O", torch.bfloat16, (B, Hq, Lq, d), dev)
    _opt(lse, "lse", torch.float32, (B, Hq, Lq), dev)
    workspace = _ws_or_new(workspace, attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=dev)
    code = lib().attn_fwd_sliding(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), B, Hq, Hkv, Lq,
                                  Lk, d, float(scale), int(window), _ptr(k_lens), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_sliding")
    return O, lse


def _bwd_args(Q, K, V, O, dO, lse, k_lens, dQ, dK, dV):
    """Validation shared by the backward entry points."""
    B, Hq, Hkv, Lq, Lk, d, dev = _qkv(Q, K, V)
    _need(O, "O", torch.bfloat16, (B, Hq, Lq, d), dev)
    _need(dO, "dO", torch.bfloat16, (B, Hq, Lq, d), dev)
    _need(lse, "lse", torch.float32, (B, Hq, Lq), dev)
    _klens(k_lens, B, dev)
    _opt(dQ, "dQ", torch.bfloat16, (B, Hq, Lq, d), dev)
    _opt(dK, "dK", torch.bfloat16, (B, Hkv, Lk, d), dev)
    _opt(dV, "dV", torch.bfloat16, (B, Hkv, Lk, d), dev)
    return B, Hq, Hkv, Lq, Lk, d, dev


def attn_bwd_sliding(Q, K, V, O, dO, lse, window, scale=None, k_lens=None, dQ=None, dK=None,
                     dV=None, workspace=None, stream=None):
    """Backward of attn_fwd_sliding.  Returns (dQ, dK, dV) bf16."""
    B, Hq, Hkv, Lq, Lk, d, dev = _bwd_args(Q, K, V, O, dO, lse, k_lens, dQ, dK, dV)
    workspace = _ws_or_new(workspace, attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
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
    _need(Q, "Q", torch.bfloat16)
    if Q.dim() != 3:
        raise ValueError(f"Q must be [total_q, Hq, d], got {tuple(Q.shape)}")
    total_q, Hq, d = (int(x) for x in Q.shape)
    dev = Q.device
    _need(K, "K", torch.bfloat16, device=dev)
    if K.dim() != 3 or int(K.shape[2]) != d:
        raise ValueError(f"K must be [total_k, Hkv, {d}], got {tuple(K.shape)}")
    _need(V, "V", torch.bfloat16, tuple(K.shape), dev)
    total_k, Hkv = int(K.shape[0]), int(K.shape[1])
    _heads(Hq, Hkv)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, device=dev)
    if cu_seqlens_q.dim() != 1 or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q must be a 1-D int32 tensor of B + 1 offsets")
    B = cu_seqlens_q.numel() - 1
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, (B + 1,), dev)
    _opt(O, "O", torch.bfloat16, (total_q, Hq, d), dev)
    _opt(lse, "lse", torch.float32, (Hq, total_q), dev)
    workspace = _ws_or_new(workspace, attn_fwd_varlen_workspace_size(
        B, Hq, Hkv, max_seqlen_q, max_seqlen_k, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=dev)
    code = lib().attn_fwd_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                 _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, Hq, Hkv,
                                 int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, d,
                                 float(scale), _mask(causal), _ptr(workspace), workspace.numel(),
                                 _stream(stream))
    _check(code, "attn_fwd_varlen")
    return O, lse


def _decode_args(Q, Kc, Vc, k_lens, O, lse, kv_names=("Kcache", "Vcache")):
    """Validation shared by the decode entry points: Q [B,Hq,1,d], the cache
    [X,Hkv,Y,d] (contiguous [B,Hkv,Lmax,d] or pages [n_pages,Hkv,page,d])."""
    _need(Q, "Q", torch.bfloat16)
    if Q.dim() != 4 or int(Q.shape[2]) != 1:
        raise ValueError(f"Q must be [B, Hq, 1, d], got {tuple(Q.shape)}")
    B, Hq, _, d = (int(x) for x in Q.shape)
    dev = Q.device
    _need(Kc, kv_names[0], torch.bfloat16, device=dev)
    if Kc.dim() != 4 or int(Kc.shape[3]) != d:
        raise ValueError(f"{kv_names[0]} must be [*, Hkv, *, {d}], got {tuple(Kc.shape)}")
    _need(Vc, kv_names[1], torch.bfloat16, tuple(Kc.shape), dev)
    Hkv = int(Kc.shape[1])
    _heads(Hq, Hkv)
    _klens(k_lens, B, dev, required=True)
    _opt(O, "O", torch.bfloat16, (B, Hq, 1, d), dev)
    _opt(lse, "lse", torch.float32, (B, Hq), dev)
    return B, Hq, Hkv, d, dev


def attn_fwd_splitkv_decode(Q, Kc, Vc, k_lens, scale=None, O=None, lse=None, workspace=None,
                            stream=None, want_lse=True):
    """Split-KV decode.  Q [B,Hq,1,d]; Kc/Vc [B,Hkv,Lmax,d] bf16; k_lens int32 [B] (device)."""
    B, Hq, Hkv, d, dev = _decode_args(Q, Kc, Vc, k_lens, O, lse)
    if int(Kc.shape[0]) != B:
        raise ValueError(f"Kcache must be [{B}, Hkv, Lmax, {d}], got {tuple(Kc.shape)}")
    Lmax = int(Kc.shape[2])
    workspace = _ws_or_new(workspace, attn_decode_workspace_size(B, Hq, Hkv, Lmax, d), dev,
                           stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    code = lib().attn_fwd_splitkv_decode(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(O), _ptr(lse), B, Hq,
                                         Hkv, Lmax, d, float(scale), _ptr(k_lens),
                                         _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "attn_fwd_splitkv_decode")
    return O, lse


def attn_fwd_splitkv_decode_paged(Q, Kp, Vp, block_table, k_lens, scale=None, O=None, lse=None,
                                  workspace=None, stream=None, want_lse=True):
    """Split-KV decode over a paged cache.  Q [B,Hq,1,d]; Kp/Vp [n_pages,Hkv,page,d] bf16;
    block_table int32 [B,max_blocks] and k_lens int32 [B] on the device."""
    B, Hq, Hkv, d, dev = _decode_args(Q, Kp, Vp, k_lens, O, lse, ("Kpages", "Vpages"))
    _need(block_table, "block_table", torch.int32, device=dev)
    if block_table.dim() != 2 or int(block_table.shape[0]) != B:
        raise ValueError(f"block_table must be [{B}, max_blocks], got {tuple(block_table.shape)}")
    n_pages, page = int(Kp.shape[0]), int(Kp.shape[2])
    max_blocks = int(block_table.shape[1])
    workspace = _ws_or_new(workspace, attn_decode_workspace_size(B, Hq, Hkv, max_blocks * page, d),
                           dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
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
    B, Hq, Hkv, d, dev = _decode_args(Q, Kc, Vc, k_lens, O, lse)
    if int(Kc.shape[0]) != B:
        raise ValueError(f"Kcache must be [{B}, Hkv, Lmax, {d}], got {tuple(Kc.shape)}")
    Lmax = int(Kc.shape[2])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    code = lib().attn_fwd_splitkv_decode_noalloc(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(O), _ptr(lse),
                                                 B, Hq, Hkv, Lmax, d, float(scale),
                                                 _ptr(k_lens), _stream(stream))
    _check(code, "attn_fwd_splitkv_decode_noalloc")
    return O, lse


def attn_bwd(Q, K, V, O, dO, lse, scale=None, causal=False, k_lens=None, dQ=None, dK=None,
             dV=None, workspace=None, stream=None):
    """Backward.  Returns (dQ, dK, dV) bf16."""
    B, Hq, Hkv, Lq, Lk, d, dev = _bwd_args(Q, K, V, O, dO, lse, k_lens, dQ, dK, dV)
    workspace = _ws_or_new(workspace, attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dev, stream)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    code = lib().attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse), _ptr(dQ),
                          _ptr(dK), _ptr(dV), B, Hq, Hkv, Lq, Lk, d, float(scale),
                          _mask(causal), _ptr(k_lens), _ptr(workspace), workspace.numel(),
                          _stream(stream))
    _check(code, "attn_bwd")
    return dQ, dK, dV
