"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
leg may import this package.  The CUDA library never calls it and shares no
code with it; there is no CPU fallback anywhere in the product path.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only compiles it with gcc and marshals numpy arrays.

Parity status of each function (what pins it, see ``tests/test_oracle_pins.py``):

* ``fwd`` / ``probs`` -- pinned: the worked example [2, 5, 1, 4] of the
  FlashAttention-2 tutorial (2.1.9), row sums, constant V, key permutation,
  causal row 0, closed forms (one key, Q = 0), the fully masked row, and an
  independent library witness (torch fp64 softmax) on small shapes.
* the sliding-window mask (``window`` > 0 with ``causal``) -- pinned: a window
  wider than the sequence equals the causal mask (forward exactly, backward to
  rounding), W = 1 closed forms (O_i = V_{i+off}, LSE_i = scale q_i.k_{i+off},
  dQ = dK = 0, dV = the routed dO), W = 2 as a two-term softmax, and brute force
  over each row's visible key set.
* ``bwd`` / ``bwd_sampled`` -- pinned: central finite differences of the
  forward's loss on tiny shapes, gradient invariants (columns of dS sum to
  zero, sum_j dV_j = sum_i dO_i), grouped-query equality to the sum of
  per-head gradients, and a torch fp64 autograd witness.
* ``e4m3_to_f64`` / ``dequant_tiles`` / ``fwd_fp8`` -- pinned: all 256 codes
  against torch's float8_e4m3fn widening (an independent library witness) and
  the format's landmark values (448, 2^-6, 2^-9, NaN), the row-to-tile scale
  assignment on constant codes with ragged tails, and invariances of the
  scales (a factor on v_scale scales O, a factor on q_scale traded against the
  softmax scale, a per-tile factor moved between codes and scales); the
  forward itself is ``fwd`` on the dequantised values.
* ``online_row`` / ``merge`` -- pinned: the worked example's block statistics
  (block A: m = 5, S = 1.0498; ratio 0.7312; block C = [10] rescale e^-5) and
  brute-force equality with the one-pass softmax over every block split.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libattn_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (fp64, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            lib.oracle_get_threads.restype = ctypes.c_int
            _c = ctypes.c_int
            lib.oracle_fwd_head.argtypes = [_dp, _dp, _dp, _c, _c, _c, ctypes.c_double, _c, _c, _c,
                                            _ip, _c, _dp, _dp]
            lib.oracle_probs_head.argtypes = [_dp, _dp, _c, _c, _c, ctypes.c_double, _c, _c, _c,
                                              _dp, _dp]
            lib.oracle_bwd_head.argtypes = [_dp, _dp, _dp, _dp, _c, _c, _c, ctypes.c_double, _c, _c,
                                            _c, _dp, _dp, _dp]
            lib.oracle_bwd_head_sampled.argtypes = [_dp, _dp, _dp, _dp, _c, _c, _c,
                                                    ctypes.c_double, _c, _c, _c, _ip, _c, _ip, _c,
                                                    _dp, _dp, _dp]
            lib.oracle_online_row.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, _ip, ctypes.c_int,
                                              _dp, _dp, _dp, _dp, _dp]
            lib.oracle_merge.argtypes = [ctypes.c_double, ctypes.c_double, _dp, ctypes.c_double,
                                         ctypes.c_double, _dp, ctypes.c_int, _dp, _dp, _dp]
            _lib = lib
    return _lib


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def threads() -> int:
    return int(_load().oracle_get_threads())


def _f64(x) -> np.ndarray:
    """fp64 C-contiguous copy; uint16 inputs are read as bf16 bit patterns."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        u = np.ascontiguousarray(x).astype(np.uint32) << np.uint32(16)
        return u.view(np.float32).astype(np.float64)
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _pi(a):
    if a is None:
        return None
    return a.ctypes.data_as(_ip)


def _kv_len(k_lens, b, Lk):
    return int(Lk if k_lens is None else k_lens[b])


def _window(causal, window):
    w = int(window or 0)
    if w > 0 and not causal:
        raise ValueError("a sliding window needs the causal mask")
    return w


def fwd(Q, K, V, scale: float, causal: bool = False, k_lens=None, rows=None, heads=None,
        window: int = 0):
    """Forward of every (b, h) head, or of the listed ``heads`` [(b, h), ...].
    ``window`` > 0 (with ``causal``): each query row sees only its ``window`` latest keys.

    Q [B,Hq,Lq,d]; K, V [B,Hkv,Lk,d] (fp64 or bf16 bits); query head h reads
    key/value head h // (Hq // Hkv).  ``rows`` restricts the query rows.
    Returns (O, LSE): O [B,Hq,R,d] fp64 and LSE [B,Hq,R] fp64 (R = len(rows) or
    Lq); heads not listed are left at zero.
    """
    lib = _load()
    B, Hq, Lq, d = np.shape(Q)
    _, Hkv, Lk, _ = np.shape(K)
    G = Hq // Hkv
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    R = Lq if rows_a is None else len(rows_a)
    O = np.zeros((B, Hq, R, d))
    L = np.zeros((B, Hq, R))
    todo = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    for b, h in todo:
        q = _f64(Q[b, h])
        k = _f64(K[b, h // G])
        v = _f64(V[b, h // G])
        o = np.zeros((R, d))
        lse = np.zeros(R)
        lib.oracle_fwd_head(_p(q), _p(k), _p(v), Lq, Lk, d, float(scale), int(bool(causal)),
                            _window(causal, window), _kv_len(k_lens, b, Lk), _pi(rows_a), R,
                            _p(o), _p(lse))
        O[b, h] = o
        L[b, h] = lse
    return O, L


def probs(Q, K, scale: float, causal: bool = False, kv_len=None, window: int = 0):
    """Full probability matrix P [Lq,Lk] and LSE [Lq] of one head (Q [Lq,d], K [Lk,d])."""
    lib = _load()
    q = _f64(Q)
    k = _f64(K)
    Lq, d = q.shape
    Lk = k.shape[0]
    P = np.zeros((Lq, Lk))
    lse = np.zeros(Lq)
    lib.oracle_probs_head(_p(q), _p(k), Lq, Lk, d, float(scale), int(bool(causal)),
                          _window(causal, window), int(Lk if kv_len is None else kv_len), _p(P),
                          _p(lse))
    return P, lse


def bwd(Q, K, V, dO, scale: float, causal: bool = False, k_lens=None, window: int = 0):
    """Full backward: returns (dQ [B,Hq,Lq,d], dK [B,Hkv,Lk,d], dV [B,Hkv,Lk,d]) in fp64.

    Grouped query heads accumulate into their shared key/value head."""
    lib = _load()
    B, Hq, Lq, d = np.shape(Q)
    _, Hkv, Lk, _ = np.shape(K)
    G = Hq // Hkv
    dQ = np.zeros((B, Hq, Lq, d))
    dK = np.zeros((B, Hkv, Lk, d))
    dV = np.zeros((B, Hkv, Lk, d))
    for b in range(B):
        for hk in range(Hkv):
            k = _f64(K[b, hk])
            v = _f64(V[b, hk])
            dk = np.zeros((Lk, d))
            dv = np.zeros((Lk, d))
            for h in range(hk * G, hk * G + G):
                q = _f64(Q[b, h])
                g = _f64(dO[b, h])
                dq = np.zeros((Lq, d))
                lib.oracle_bwd_head(_p(q), _p(k), _p(v), _p(g), Lq, Lk, d, float(scale),
                                    int(bool(causal)), _window(causal, window),
                                    _kv_len(k_lens, b, Lk), _p(dq), _p(dk), _p(dv))
                dQ[b, h] = dq
            dK[b, hk] = dk
            dV[b, hk] = dv
    return dQ, dK, dV


def bwd_sampled(Q, K, V, dO, scale: float, causal: bool, k_lens, b: int, hk: int, qrows, kcols,
                window: int = 0):
    """Backward of key/value head (b, hk) at sampled outputs.

    Returns (dQ [G,nq,d] for the G query heads of hk at rows ``qrows``,
    dK [nk,d] and dV [nk,d] at key rows ``kcols``), all fp64."""
    lib = _load()
    B, Hq, Lq, d = np.shape(Q)
    _, Hkv, Lk, _ = np.shape(K)
    G = Hq // Hkv
    qa = np.ascontiguousarray(qrows, dtype=np.int32)
    ka = np.ascontiguousarray(kcols, dtype=np.int32)
    k = _f64(K[b, hk])
    v = _f64(V[b, hk])
    dQs = np.zeros((G, len(qa), d))
    dKs = np.zeros((len(ka), d))
    dVs = np.zeros((len(ka), d))
    for gi, h in enumerate(range(hk * G, hk * G + G)):
        q = _f64(Q[b, h])
        g = _f64(dO[b, h])
        dq = np.zeros((len(qa), d))
        lib.oracle_bwd_head_sampled(_p(q), _p(k), _p(v), _p(g), Lq, Lk, d, float(scale),
                                    int(bool(causal)), _window(causal, window),
                                    _kv_len(k_lens, b, Lk), _pi(qa), len(qa), _pi(ka), len(ka),
                                    _p(dq), _p(dKs), _p(dVs))
        dQs[gi] = dq
    return dQs, dKs, dVs


def online_row(s, V, block_ends):
    """Unnormalised online softmax over one score row; returns (O, m, l, m_trace, l_trace)."""
    lib = _load()
    s = _f64(s)
    V = _f64(V)
    n, d = V.shape
    be = np.ascontiguousarray(block_ends, dtype=np.int32)
    O = np.zeros(d)
    m = np.zeros(1)
    l = np.zeros(1)
    mt = np.zeros(len(be))
    lt = np.zeros(len(be))
    lib.oracle_online_row(_p(s), _p(V), n, d, _pi(be), len(be), _p(O), _p(m), _p(l), _p(mt),
                          _p(lt))
    return O, float(m[0]), float(l[0]), mt, lt


def merge(m_a, l_a, O_a, m_b, l_b, O_b):
    """Normalised merge of two partial (m, l, O) results; returns (m, l, O)."""
    lib = _load()
    Oa = _f64(O_a)
    Ob = _f64(O_b)
    d = Oa.shape[0]
    O = np.zeros(d)
    m = np.zeros(1)
    l = np.zeros(1)
    lib.oracle_merge(float(m_a), float(l_a), _p(Oa), float(m_b), float(l_b), _p(Ob), d, _p(m),
                     _p(l), _p(O))
    return float(m[0]), float(l[0]), O


# ---------------------------------------------------------------- 8-bit (E4M3) inputs
# The low-precision forward of the FlashAttention line ("FlashAttention" blog,
# section 10 on FlashAttention-3: new-hardware features and low-precision
# execution) takes Q, K and V as 8-bit floats.  The oracle decodes them exactly
# and runs the fp64 forward above on the dequantised values: it is the exact
# attention of the inputs the low-precision path is given.


def e4m3_to_f64(codes) -> np.ndarray:
    """Exact values of E4M3 8-bit floats (the OCP 8-bit floating-point format):
    bit 7 sign, bits 6-3 exponent with bias 7, bits 2-0 mantissa.  Exponent
    field 0 holds zero and the subnormals (m / 8) * 2^-6; otherwise the value is
    (1 + m / 8) * 2^(e - 7).  There are no infinities: S.1111.111 is NaN, so the
    largest finite magnitude is S.1111.110 = 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def dequant_tiles(codes, scales, tile: int = 128) -> np.ndarray:
    """Dequantise [..., L, d] E4M3 codes with one scale per ``tile`` rows:
    row i of every head is multiplied by scales[..., i // tile]."""
    x = e4m3_to_f64(codes)
    L = x.shape[-2]
    sc = np.asarray(scales, dtype=np.float64)
    if sc.shape[-1] != (L + tile - 1) // tile:
        raise ValueError("one scale per row tile expected")
    return x * sc[..., np.arange(L) // tile][..., None]


def fwd_fp8(Q8, K8, V8, q_scale, k_scale, v_scale, scale: float, causal: bool = False,
            k_lens=None, rows=None, heads=None, tile: int = 128):
    """Forward of E4M3 inputs with per-tile scales: Q8 [B,Hq,Lq,d] with q_scale
    [B,Hq,ceil(Lq/tile)], K8/V8 [B,Hkv,Lk,d] with k_scale/v_scale
    [B,Hkv,ceil(Lk/tile)].  Exact attention (``fwd``) of the dequantised tensors;
    returns (O, LSE) like ``fwd``."""
    return fwd(dequant_tiles(Q8, q_scale, tile), dequant_tiles(K8, k_scale, tile),
               dequant_tiles(V8, v_scale, tile), scale, causal=causal, k_lens=k_lens, rows=rows,
               heads=heads)
