"""Float64 CPU oracle for attention with a KV cache and fused RoPE.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product path
(``rotary_embedding_b200``) never does, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, built with
gcc into ``liboracle.so`` beside it).  This module only builds that library
and marshals numpy arrays into it.  ``brute.py`` holds a second, pure-Python
statement of the same definitions for tiny shapes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FMT_NONE, FMT_FP16, FMT_BF16 = 0, 1, 2
_FMT = {None: FMT_NONE, "none": FMT_NONE, "fp16": FMT_FP16, "bf16": FMT_BF16,
        "float16": FMT_FP16, "bfloat16": FMT_BF16}


def build(force: bool = False, extra_flags: tuple = (), out_path: str | None = None) -> str:
    """Compile oracle.c with gcc (-O2, no fast-math) into a shared library."""
    out = out_path or _LIB_PATH
    if (not force and out_path is None and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", *extra_flags, _SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    d, i64, i32 = ctypes.c_double, ctypes.c_int64, ctypes.c_int
    P = ctypes.c_void_p
    lib.oracle_round_one.argtypes = [d, i32]
    lib.oracle_round_one.restype = d
    lib.oracle_round.argtypes = [P, i64, i32]
    lib.oracle_round.restype = None
    lib.oracle_rope.argtypes = [P, P, i64, i32, P, P, P, i64, i32, i32]
    lib.oracle_rope.restype = i32
    lib.oracle_rotary.argtypes = [P, P, i64, i32, P, P, P, i64, i32, i32, i32, i32]
    lib.oracle_rotary.restype = ctypes.c_int
    lib.oracle_kvcache_fwd.argtypes = [i64, i64, i64, i64, i64, i32, i32, i64,
                                       P, P, P, P, P, P, P, i64, i32, i32, P,
                                       i32, d, i32, P, P, i64, i64]
    lib.oracle_kvcache_fwd.restype = i32
    lib.oracle_fwd.argtypes = [i64, i64, i64, i64, i64, i32, i32, P, P, P, i32, d, P, P, i64, i64]
    lib.oracle_fwd.restype = i32
    lib.oracle_bwd.argtypes = [i64, i64, i64, i64, i64, i32, i32, P, P, P, P, i32, d, i64, i64, P, P, P]
    lib.oracle_bwd.restype = i32
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library; `path` loads a variant build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def round_to(x, fmt):
    """Round float64 values to the nearest fp16/bf16 value (ties to even)."""
    a = _f64(x).copy()
    load().oracle_round(_ptr(a), a.size, _FMT[fmt])
    return a


def rope(x, pos, cos_tab, sin_tab, rotary_dim, interleaved, lib=None):
    """RoPE of rows x[..., d] at table rows pos[...]; returns float64."""
    lib = lib or load()
    x = _f64(x)
    d = x.shape[-1]
    rows = x.size // d if d else 0
    pos = np.asarray(pos, dtype=np.int64)
    if x.ndim == 1:
        pos = pos.reshape(())
    pos = np.ascontiguousarray(np.broadcast_to(pos, x.shape[:-1]))
    cos_tab = _f64(cos_tab)
    sin_tab = _f64(sin_tab)
    y = np.empty_like(x)
    tab_rows = cos_tab.shape[0] if cos_tab.ndim == 2 else 0
    rc = lib.oracle_rope(_ptr(x), _ptr(y), rows, d, _ptr(pos), _ptr(cos_tab), _ptr(sin_tab),
                         tab_rows, int(rotary_dim), int(bool(interleaved)))
    if rc != 0:
        raise ValueError("position outside the rotary table")
    return y


def rotary_positions(batch, seqlen, seqlen_offsets, cu_seqlens=None):
    """Table row of every row of a rotary input ([P2] SEQLEN_OFFSET, an int or
    one value per batch entry; IS_VARLEN).  Batched input [b, s, ...]: row i
    of entry k is at offset_k + i, returned as [b, s].  Packed input [total,
    ...] with cu_seqlens [b + 1]: row t of entry k (cu[k] <= t < cu[k+1]) is
    at offset_k + t - cu[k], returned as [total]."""
    if cu_seqlens is None:
        off = np.broadcast_to(np.asarray(seqlen_offsets, dtype=np.int64).reshape(-1, 1)
                              if np.ndim(seqlen_offsets) else np.int64(seqlen_offsets), (batch, 1))
        return off + np.arange(seqlen, dtype=np.int64)[None, :]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nb = len(cu) - 1
    off = np.broadcast_to(np.asarray(seqlen_offsets, dtype=np.int64), (nb,))
    pos = np.empty(cu[-1], dtype=np.int64)
    for k in range(nb):
        for t in range(cu[k], cu[k + 1]):
            pos[t] = off[k] + t - cu[k]
    return pos


def rotary(x, cos_tab, sin_tab, seqlen_offsets=0, rotary_dim=0, interleaved=False, conjugate=False,
           cu_seqlens=None, fmt=None, lib=None):
    """Standalone rotary of x ([b, s, h, d], or packed [total, h, d] with
    cu_seqlens): every head of a row rotated at the row's table position,
    by the negated angle when `conjugate`, rounded to `fmt`.  float64."""
    lib = lib or load()
    x = _f64(x)
    d = x.shape[-1]
    if cu_seqlens is None:
        pos = rotary_positions(x.shape[0], x.shape[1], seqlen_offsets)
    else:
        pos = rotary_positions(None, None, seqlen_offsets, cu_seqlens)
    pos = np.ascontiguousarray(np.broadcast_to(pos[..., None], x.shape[:-1]))
    cos_tab = _f64(cos_tab)
    sin_tab = _f64(sin_tab)
    tab_rows = cos_tab.shape[0] if cos_tab.ndim == 2 else 0
    y = np.empty_like(x)
    rows = x.size // d if d else 0
    rc = lib.oracle_rotary(_ptr(x), _ptr(y), rows, d, _ptr(pos), _ptr(cos_tab), _ptr(sin_tab), tab_rows,
                           int(rotary_dim), int(bool(interleaved)), int(bool(conjugate)), _FMT[fmt])
    if rc != 0:
        raise ValueError("position outside the rotary table")
    return y


def kvcache_fwd(q, k_cache, v_cache, k_new, v_new, cos_tab, sin_tab, cache_seqlens,
                rotary_dim=0, interleaved=False, causal=False, scale=None, fmt=None,
                window=(-1, -1),
                lib=None):
    """The whole attn_with_kvcache path in float64.

    Arrays are [batch, seq, heads, dim] (any float dtype; upconverted exactly).
    `cache_seqlens` is an int or a per-batch int array.  Returns
    (out [b, s_q, h_q, d_v], lse [b, h_q, s_q], k_cache', v_cache') with the
    caches updated copies; the inputs are not modified.
    """
    lib = lib or load()
    q = _f64(q)
    kc = _f64(k_cache).copy()
    vc = _f64(v_cache).copy()
    b, s_q, h_q, d_qk = q.shape
    _, cap, h_kv, _ = kc.shape
    d_v = vc.shape[3]
    if k_new is None:
        kn = np.zeros((b, 0, h_kv, d_qk))
        vn = np.zeros((b, 0, h_kv, d_v))
    else:
        kn, vn = _f64(k_new), _f64(v_new)
    s_new = kn.shape[1]
    seql = np.ascontiguousarray(np.broadcast_to(np.asarray(cache_seqlens, dtype=np.int32), (b,)))
    r = int(rotary_dim)
    if r > 0:
        ct, st = _f64(cos_tab), _f64(sin_tab)
        tab_rows = ct.shape[0]
    else:
        ct = st = np.zeros((1, 1))
        tab_rows = 0
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d_qk)
    out = np.zeros((b, s_q, h_q, d_v))
    lse = np.zeros((b, h_q, s_q))
    rc = lib.oracle_kvcache_fwd(b, s_q, s_new, h_q, h_kv, d_qk, d_v, cap,
                                _ptr(q), _ptr(kc), _ptr(vc), _ptr(kn), _ptr(vn),
                                _ptr(ct), _ptr(st), tab_rows, r, int(bool(interleaved)),
                                _ptr(seql), int(bool(causal)), float(scale), _FMT[fmt],
                                _ptr(out), _ptr(lse), int(window[0]), int(window[1]))
    if rc != 0:
        raise ValueError(f"oracle_kvcache_fwd rejected its arguments (code {rc})")
    return out, lse, kc, vc


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, causal=False, scale=None, lib=None, window=(-1, -1)):
    """Attention over packed sequences ([P2] IS_VARLEN): q [total_q, h_q, d_qk],
    k/v [total_k, h_kv, d]; sequence s holds query rows cu_q[s] .. cu_q[s+1]-1
    and key rows cu_k[s] .. cu_k[s+1]-1, each attended exactly as a batch of
    one by fwd (bottom-right alignment inside the sequence).  Returns
    (out [total_q, h_q, d_v], lse [h_q, total_q])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    out = np.zeros((q.shape[0], q.shape[1], v.shape[2]))
    lse = np.full((q.shape[1], q.shape[0]), -np.inf)
    for sidx in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[sidx], cq[sidx + 1], ck[sidx], ck[sidx + 1]
        if q1 == q0:
            continue
        o, l = fwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], causal=causal, scale=scale, lib=lib,
                   window=window)
        out[q0:q1] = o[0]
        lse[:, q0:q1] = l[0]
    return out, lse


def fwd(q, k, v, causal=False, scale=None, lib=None, window=(-1, -1)):
    """Cache-less attention in float64: returns (out [b,s_q,h_q,d_v], lse [b,h_q,s_q]).
    window = (left, right): query i (at key position a = i + s_k - s_q) sees keys
    a - left .. a + right; -1 leaves that side unbounded."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, s_q, h_q, d_qk = q.shape
    s_k, h_kv = k.shape[1], k.shape[2]
    d_v = v.shape[3]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d_qk)
    out = np.zeros((b, s_q, h_q, d_v))
    lse = np.zeros((b, h_q, s_q))
    rc = lib.oracle_fwd(b, s_q, s_k, h_q, h_kv, d_qk, d_v, _ptr(q), _ptr(k), _ptr(v),
                        int(bool(causal)), float(scale), _ptr(out), _ptr(lse), int(window[0]),
                        int(window[1]))
    if rc != 0:
        raise ValueError(f"oracle_fwd rejected its arguments (code {rc})")
    return out, lse


def bwd(q, k, v, dout, causal=False, scale=None, lib=None, window=(-1, -1)):
    """Gradients of cache-less attention in float64 ([P4] d_qk != d_v
    backward): the gradient of sum(dout * fwd(q, k, v)) with respect to q, k
    and v, for the same mask, scale and GQA mapping.  Returns (dq, dk, dv)
    shaped like q, k, v."""
    lib = lib or load()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    b, s_q, h_q, d_qk = q.shape
    s_k, h_kv = k.shape[1], k.shape[2]
    d_v = v.shape[3]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d_qk)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = lib.oracle_bwd(b, s_q, s_k, h_q, h_kv, d_qk, d_v, _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                        int(bool(causal)), float(scale), int(window[0]), int(window[1]),
                        _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError(f"oracle_bwd rejected its arguments (code {rc})")
    return dq, dk, dv
