"""Attention with a KV cache and fused RoPE on NVIDIA B200 (sm_100a).

A thin Python binding over the C ABI of ``libfa.so`` (declared in
``include/fa.h``).  Functions carry the C names; they only marshal torch
tensors into ``fa_tensor`` descriptors, pick the current CUDA stream, let
torch allocate outputs and the workspace, and raise on a non-zero status.
Every step of the computation runs in the library's CUDA kernels; there is
no CPU or PyTorch fallback: if the library is missing, importing this
package raises.

Argument names follow flash_attn_with_kvcache as used on flash-attention
issue #1402 (rotary_cos, rotary_sin, cache_seqlens, rotary_interleaved,
causal, softmax_scale).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_LAYOUT = -3
FA_ERR_WORKSPACE = -4
FA_ERR_CUDA = -5
FA_ERR_DEVICE_PRECONDITION = -6
FA_ERR_DEVICE_TIMEOUT = -7
FA_DTYPE_F16 = 1
FA_DTYPE_BF16 = 2

_DTYPES = {torch.float16: FA_DTYPE_F16, torch.bfloat16: FA_DTYPE_BF16}


class FaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class FaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python rotary_embedding_b200/build.py`")
lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.POINTER(FaTensor)
_v = ctypes.c_void_p
_i32 = ctypes.c_int32
lib.fa_kvcache_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _v, _i32, _i32, _i32, ctypes.c_float,
                               _P, _v, _i32, _v, ctypes.c_size_t, _v]
lib.fa_kvcache_fwd.restype = ctypes.c_int
lib.fa_kvcache_workspace_size.argtypes = [_P, _P, _P, _P, _i32, ctypes.POINTER(ctypes.c_size_t)]
lib.fa_kvcache_workspace_size.restype = ctypes.c_int
lib.fa_fwd.argtypes = [_P, _P, _P, _i32, ctypes.c_float, _P, _v, _v, ctypes.c_size_t, _v]
lib.fa_fwd.restype = ctypes.c_int
lib.fa_fwd_window.argtypes = [_P, _P, _P, _i32, _i32, _i32, ctypes.c_float, _P, _v, _v, ctypes.c_size_t, _v]
lib.fa_fwd_window.restype = ctypes.c_int
lib.fa_kvcache_fwd_window.argtypes = [_P, _P, _P, _P, _P, _P, _P, _v, _i32, _i32, _i32, _i32, _i32,
                                      ctypes.c_float, _P, _v, _i32, _v, ctypes.c_size_t, _v]
lib.fa_kvcache_fwd_window.restype = ctypes.c_int
lib.fa_fwd_varlen.argtypes = [_P, _P, _P, _v, _v, _i32, _i32, _i32, _i32, _i32, ctypes.c_float, _P, _v, _v]
lib.fa_fwd_varlen.restype = ctypes.c_int
lib.fa_bwd.argtypes = [_P, _P, _P, _P, _P, _v, _i32, _i32, _i32, ctypes.c_float, _P, _P, _P, _v, ctypes.c_size_t,
                       _v]
lib.fa_bwd.restype = ctypes.c_int
lib.fa_bwd_workspace_size.argtypes = [_P, ctypes.POINTER(ctypes.c_size_t)]
lib.fa_bwd_workspace_size.restype = ctypes.c_int
lib.fa_fwd_workspace_size.argtypes = [_P, _P, _P, ctypes.POINTER(ctypes.c_size_t)]
lib.fa_fwd_workspace_size.restype = ctypes.c_int
lib.fa_device_status.argtypes = [_v, ctypes.POINTER(ctypes.c_int32)]
lib.fa_device_status.restype = ctypes.c_int
lib.fa_status_string.argtypes = [ctypes.c_int]
lib.fa_status_string.restype = ctypes.c_char_p
lib.fa_last_error.argtypes = []
lib.fa_last_error.restype = ctypes.c_char_p
lib.fa_version.argtypes = []
lib.fa_version.restype = ctypes.c_int
lib.fa_set_kernel_events.argtypes = [_v, _v]
lib.fa_set_kernel_events.restype = ctypes.c_int


_I64x4 = ctypes.c_int64 * 4
# Descriptors already built, keyed by everything a descriptor holds (address,
# dtype, shape, strides): a hit is the identical, read-only structure, so a
# call on the same tensors (a decode or serving loop) skips rebuilding it.
_desc_cache: dict = {}


def describe(t: torch.Tensor | None):
    """fa_tensor descriptor of a torch tensor (None -> NULL)."""
    if t is None:
        return None
    shape, stride = t.shape, t.stride()
    key = (t.data_ptr(), t.dtype, shape, stride)
    d = _desc_cache.get(key)
    if d is None:
        n = len(shape)
        pad = (0,) * max(0, 4 - n)
        d = FaTensor(key[0], _DTYPES.get(t.dtype, 0), n, _I64x4(*(tuple(shape[:4]) + pad)),
                     _I64x4(*(tuple(stride[:4]) + pad)))
        if len(_desc_cache) >= 512:
            _desc_cache.clear()
        _desc_cache[key] = d
    return d


def _ref(d):
    return ctypes.byref(d) if d is not None else None


def _lse_ptr(lse, shape):
    """Pointer to an fp32 lse buffer of exactly `shape`, contiguous (the C
    ABI takes lse as a plain float array in that layout), or None."""
    if lse is None:
        return None
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != tuple(shape):
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {tuple(shape)}")
    return ctypes.c_void_p(lse.data_ptr())


def _i32_ptr(t, name, min_len):
    """Pointer to a contiguous int32 tensor of at least `min_len` entries."""
    if t.dtype != torch.int32 or not t.is_contiguous() or t.numel() < min_len:
        raise ValueError(f"{name} must be a contiguous int32 tensor of at least {min_len} entries")
    return ctypes.c_void_p(t.data_ptr())


def _check(status: int):
    if status != FA_OK:
        msg = lib.fa_last_error().decode() or lib.fa_status_string(status).decode()
        raise FaError(status, msg)


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _require_device(device, **tensors):
    """Every tensor given (None entries are skipped) must live on `device`, a
    CUDA device.  The C ABI takes raw addresses and cannot tell a host
    pointer from a device one, so a CPU tensor, or one on another GPU, is
    rejected here with ValueError before any work is enqueued."""
    if device.type != "cuda":
        raise ValueError(f"tensors must be CUDA tensors (got {device})")
    for name, t in tensors.items():
        if t is not None and (not t.is_cuda or t.device != device):
            raise ValueError(f"{name} must be a CUDA tensor on {device} (got {t.device})")


def fa_kvcache_workspace_size(q, k_cache, v_cache, k_new=None, rotary_dim=0) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.fa_kvcache_workspace_size(_ref(describe(q)), _ref(describe(k_cache)),
                                         _ref(describe(v_cache)), _ref(describe(k_new)),
                                         int(rotary_dim), ctypes.byref(n)))
    return n.value


def fa_fwd_workspace_size(q, k, v) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.fa_fwd_workspace_size(_ref(describe(q)), _ref(describe(k)), _ref(describe(v)),
                                     ctypes.byref(n)))
    return n.value


def _kvcache_args(q, v_cache, rotary_cos, rotary_dim, cache_seqlens, out, lse, return_lse):
    """Shared argument marshalling of the two kvcache entry points."""
    b, s_q, h_q, _ = q.shape
    d_v = v_cache.shape[3]
    if rotary_cos is not None and rotary_dim is None:
        rotary_dim = 2 * rotary_cos.shape[1]
    rotary_dim = int(rotary_dim or 0) if rotary_cos is not None else 0
    if out is None:
        out = torch.empty((b, s_q, h_q, d_v), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=q.device)
    if isinstance(cache_seqlens, torch.Tensor):
        seq_ptr, seq_scalar = _i32_ptr(cache_seqlens, "cache_seqlens", b), 0
    else:
        seq_ptr, seq_scalar = None, int(cache_seqlens)
    return rotary_dim, out, lse, seq_ptr, seq_scalar, (b, h_q, s_q)


def fa_kvcache_fwd(q, k_cache, v_cache, k_new=None, v_new=None, rotary_cos=None, rotary_sin=None,
                   cache_seqlens=0, rotary_dim=None, rotary_interleaved=False, causal=False,
                   softmax_scale=None, out=None, lse=None, workspace=None, return_lse=True,
                   stream=None, window=(-1, -1)):
    """RoPE of q/k_new at positions cache_seqlens[b] + i, append of the rotated
    k and raw v into k_cache/v_cache (in place), then attention over cache and
    new rows.  Tensors are [batch, seq, heads, dim] CUDA tensors on one
    device; cache_seqlens is an int or an int32 CUDA tensor [batch]; window =
    (left, right) keys around the query's aligned position (-1 = unbounded).
    Returns (out, lse)."""
    _require_device(q.device, q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                    rotary_cos=rotary_cos, rotary_sin=rotary_sin, out=out, lse=lse, workspace=workspace,
                    cache_seqlens=cache_seqlens if isinstance(cache_seqlens, torch.Tensor) else None)
    rotary_dim, out, lse, seq_ptr, seq_scalar, lse_shape = _kvcache_args(
        q, v_cache, rotary_cos, rotary_dim, cache_seqlens, out, lse, return_lse)
    if workspace is None:
        ws_bytes = fa_kvcache_workspace_size(q, k_cache, v_cache, k_new, rotary_dim)
        if ws_bytes > 0:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib.fa_kvcache_fwd_window(
            _ref(describe(q)), _ref(describe(k_cache)), _ref(describe(v_cache)), _ref(describe(k_new)),
            _ref(describe(v_new)), _ref(describe(rotary_cos)), _ref(describe(rotary_sin)), seq_ptr,
            rotary_dim, int(bool(rotary_interleaved)), int(bool(causal)), int(window[0]), int(window[1]),
            float(softmax_scale or 0.0), _ref(describe(out)), _lse_ptr(lse, lse_shape), seq_scalar,
            ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None,
            workspace.numel() if workspace is not None else 0, _stream_handle(stream, q.device)))
    return out, lse


lib.fa_rotary.argtypes = [_P, _P, _P, _v, _i32, _v, _i32, _i32, _i32, _i32, _P, _v]
lib.fa_rotary.restype = ctypes.c_int


def fa_rotary(x, cos, sin, seqlen_offsets=0, rotary_dim=None, interleaved=False, conjugate=False,
              cu_seqlens=None, out=None, stream=None):
    """Standalone rotary embedding of x ([b, s, h, d], or [total, h, d] packed
    rows with cu_seqlens [n_seqs + 1]): every head of a row rotated at table
    row offset + i (per batch entry / packed sequence), by the negated angle
    when `conjugate`.  seqlen_offsets is an int or an int32 CUDA tensor.
    out may be x (in place); a new tensor is allocated when it is None."""
    _require_device(x.device, x=x, cos=cos, sin=sin, out=out, cu_seqlens=cu_seqlens,
                    seqlen_offsets=seqlen_offsets if isinstance(seqlen_offsets, torch.Tensor) else None)
    packed = cu_seqlens is not None
    xv = x.unsqueeze(0) if packed else x
    if out is None:
        out = torch.empty_like(x)
    ov = out.unsqueeze(0) if packed else out
    if rotary_dim is None:
        rotary_dim = 2 * cos.shape[1] if cos is not None else 0
    n_seqs = int(cu_seqlens.numel()) - 1 if packed else 0
    if isinstance(seqlen_offsets, torch.Tensor):
        off_ptr, off_scalar = _i32_ptr(seqlen_offsets, "seqlen_offsets", n_seqs if packed else x.shape[0]), 0
    else:
        off_ptr, off_scalar = None, int(seqlen_offsets)
    cu_ptr = _i32_ptr(cu_seqlens, "cu_seqlens", 1) if packed else None
    with torch.cuda.device(x.device):
        _check(lib.fa_rotary(_ref(describe(xv)), _ref(describe(cos)), _ref(describe(sin)), off_ptr, off_scalar,
                             cu_ptr, n_seqs, int(rotary_dim), int(bool(interleaved)), int(bool(conjugate)),
                             _ref(describe(ov)), _stream_handle(stream, x.device)))
    return out


lib.fa_kvcache_fwd_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _P, _v, _i32, _i32, _i32, ctypes.c_float,
                                        _P, _v, _i32, _v]
lib.fa_kvcache_fwd_noalloc.restype = ctypes.c_int
FA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def fa_kvcache_fwd_noalloc(q, k_cache, v_cache, k_new=None, v_new=None, rotary_cos=None,
                           rotary_sin=None, cache_seqlens=0, rotary_dim=None,
                           rotary_interleaved=False, causal=False, softmax_scale=None, out=None,
                           lse=None, return_lse=True, stream=None):
    """fa_kvcache_fwd whose scratch comes from the library's built-in array
    (FA_NOALLOC_SCRATCH_BYTES) instead of a workspace: for callers that must not
    allocate device memory when attention runs.  The library call itself
    allocates nothing; this Python wrapper only allocates `out`/`lse` when they
    are not passed.  The first call on a device loads the array's module and
    reserves its memory: make it once, outside the region that must not
    allocate.  Calls that overlap on the GPU share the scratch and race."""
    _require_device(q.device, q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                    rotary_cos=rotary_cos, rotary_sin=rotary_sin, out=out, lse=lse,
                    cache_seqlens=cache_seqlens if isinstance(cache_seqlens, torch.Tensor) else None)
    rotary_dim, out, lse, seq_ptr, seq_scalar, lse_shape = _kvcache_args(
        q, v_cache, rotary_cos, rotary_dim, cache_seqlens, out, lse, return_lse)
    with torch.cuda.device(q.device):
        _check(lib.fa_kvcache_fwd_noalloc(
            _ref(describe(q)), _ref(describe(k_cache)), _ref(describe(v_cache)), _ref(describe(k_new)),
            _ref(describe(v_new)), _ref(describe(rotary_cos)), _ref(describe(rotary_sin)), seq_ptr,
            rotary_dim, int(bool(rotary_interleaved)), int(bool(causal)), float(softmax_scale or 0.0),
            _ref(describe(out)), _lse_ptr(lse, lse_shape), seq_scalar, _stream_handle(stream, q.device)))
    return out, lse


def fa_fwd(q, k, v, causal=False, softmax_scale=None, out=None, lse=None, workspace=None,
           return_lse=True, stream=None, window=(-1, -1)):
    """Cache-less attention: q [b, s_q, h_q, d_qk], k/v [b, s_k, h_kv, d]; window =
    (left, right) keys around the query's aligned position (-1 = unbounded);
    returns (out, lse)."""
    _require_device(q.device, q=q, k=k, v=v, out=out, lse=lse, workspace=workspace)
    b, s_q, h_q, _ = q.shape
    d_v = v.shape[3]
    if out is None:
        out = torch.empty((b, s_q, h_q, d_v), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        ws_bytes = fa_fwd_workspace_size(q, k, v)
        if ws_bytes > 0:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib.fa_fwd_window(
            _ref(describe(q)), _ref(describe(k)), _ref(describe(v)), int(bool(causal)), int(window[0]),
            int(window[1]), float(softmax_scale or 0.0), _ref(describe(out)), _lse_ptr(lse, (b, h_q, s_q)),
            ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None,
            workspace.numel() if workspace is not None else 0, _stream_handle(stream, q.device)))
    return out, lse


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal=False, softmax_scale=None,
                  window=(-1, -1), out=None, lse=None, return_lse=True, stream=None):
    """Attention over packed sequences: q [total_q, h_q, d_qk], k/v [total_k,
    h_kv, d]; cu_seqlens_q/k int32 CUDA tensors [n_seqs + 1] of row starts.
    Returns (out [total_q, h_q, d_v], lse [h_q, total_q])."""
    _require_device(q.device, q=q, k=k, v=v, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, out=out,
                    lse=lse)
    total_q, h_q, _ = q.shape
    d_v = v.shape[2]
    if out is None:
        out = torch.empty((total_q, h_q, d_v), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((h_q, total_q), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib.fa_fwd_varlen(
            _ref(describe(q)), _ref(describe(k)), _ref(describe(v)),
            _i32_ptr(cu_seqlens_q, "cu_seqlens_q", 2),
            _i32_ptr(cu_seqlens_k, "cu_seqlens_k", cu_seqlens_q.numel()),
            int(cu_seqlens_q.numel()) - 1, int(max_seqlen_q), int(bool(causal)), int(window[0]),
            int(window[1]), float(softmax_scale or 0.0), _ref(describe(out)), _lse_ptr(lse, (h_q, total_q)),
            _stream_handle(stream, q.device)))
    return out, lse


def fa_bwd_workspace_size(q):
    n = ctypes.c_size_t(0)
    _check(lib.fa_bwd_workspace_size(_ref(describe(q)), ctypes.byref(n)))
    return n.value


def fa_bwd(q, k, v, out, dout, lse, causal=False, softmax_scale=None, window=(-1, -1), dq=None, dk=None,
           dv=None, workspace=None, stream=None):
    """Gradients of fa_fwd for an upstream gradient dout, given the forward's
    out and lse [b, h_q, s_q]: returns (dq, dk, dv) shaped like q, k, v."""
    _require_device(q.device, q=q, k=k, v=v, out=out, dout=dout, lse=lse, dq=dq, dk=dk, dv=dv,
                    workspace=workspace)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        ws_bytes = fa_bwd_workspace_size(q)
        if ws_bytes > 0:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib.fa_bwd(
            _ref(describe(q)), _ref(describe(k)), _ref(describe(v)), _ref(describe(out)), _ref(describe(dout)),
            _lse_ptr(lse, (q.shape[0], q.shape[2], q.shape[1])), int(bool(causal)), int(window[0]),
            int(window[1]), float(softmax_scale or 0.0), _ref(describe(dq)), _ref(describe(dk)),
            _ref(describe(dv)), ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None,
            workspace.numel() if workspace is not None else 0, _stream_handle(stream, q.device)))
    return dq, dk, dv


class FaPlan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("launches", ctypes.c_int32), ("n_splits", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("workspace_bytes", ctypes.c_size_t)]


FA_PATH_DECODE, FA_PATH_PREFILL, FA_PATH_DENSE = 1, 2, 3
lib.fa_kvcache_plan.argtypes = [_P, _P, _P, _P, _i32, ctypes.POINTER(FaPlan)]
lib.fa_kvcache_plan.restype = ctypes.c_int
lib.fa_fwd_plan.argtypes = [_P, _P, _P, ctypes.POINTER(FaPlan)]
lib.fa_fwd_plan.restype = ctypes.c_int


def fa_kvcache_plan(q, k_cache, v_cache, k_new=None, rotary_dim=0) -> dict:
    p = FaPlan()
    _check(lib.fa_kvcache_plan(_ref(describe(q)), _ref(describe(k_cache)), _ref(describe(v_cache)),
                               _ref(describe(k_new)), int(rotary_dim), ctypes.byref(p)))
    return {k: getattr(p, k) for k, _ in FaPlan._fields_}


def fa_fwd_plan(q, k, v) -> dict:
    p = FaPlan()
    _check(lib.fa_fwd_plan(_ref(describe(q)), _ref(describe(k)), _ref(describe(v)), ctypes.byref(p)))
    return {k: getattr(p, k) for k, _ in FaPlan._fields_}


def fa_device_status(stream=None) -> int:
    """Synchronise and read (then clear) the device status word."""
    s = ctypes.c_int32(0)
    h = ctypes.c_void_p(stream.cuda_stream) if stream is not None else None
    _check(lib.fa_device_status(h, ctypes.byref(s)))
    return s.value


def fa_version() -> int:
    return lib.fa_version()


lib.fa_testing_set_prefill_tiles.argtypes = [_i32]
lib.fa_testing_set_prefill_tiles.restype = ctypes.c_int


def fa_testing_set_prefill_tiles(tiles: int) -> None:
    """Test hook (include/fa_testing.h): pin the prefill kernel of later calls
    to one (1) or two (2) query tiles per CTA, to one tile with its key range
    split between the two softmax warpgroups (3), or give the choice back to
    the planner (0)."""
    _check(lib.fa_testing_set_prefill_tiles(int(tiles)))


def fa_set_kernel_events(start=None, stop=None) -> None:
    """Profiling hook: record `start` / `stop` (torch.cuda.Event, timing
    enabled) around the attention kernel of every following call, or switch
    it off with no arguments.  Both events are recorded once here on the
    current stream so that their CUDA handles exist."""
    if start is None and stop is None:
        _check(lib.fa_set_kernel_events(None, None))
        return
    if start is None or stop is None:
        raise ValueError("pass both events or neither")
    start.record()
    stop.record()
    _check(lib.fa_set_kernel_events(ctypes.c_void_p(start.cuda_event), ctypes.c_void_p(stop.cuda_event)))
