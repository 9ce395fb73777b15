"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/fa.h declares, validates arguments before touching
the device, and plans workspace sizes."""
import ctypes
import os
import re

import pytest
import torch

import rotary_embedding_b200 as fa
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(fa_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = _header_functions()
    for n in ("fa_kvcache_fwd", "fa_fwd", "fa_kvcache_workspace_size", "fa_fwd_workspace_size",
              "fa_status_string", "fa_last_error", "fa_device_status", "fa_version"):
        assert n in names


@pytest.mark.parametrize("name", _header_functions())
def test_library_exports(name):
    assert hasattr(fa.lib, name), f"libfa.so does not export {name}"


def test_version_and_strings():
    assert fa.fa_version() >= 100
    assert fa.lib.fa_status_string(fa.FA_ERR_LAYOUT).decode()
    assert fa.lib.fa_status_string(12345).decode() == "unknown status"


def _kv_tensors(b=2, s=3, hq=4, hkv=2, d=64, dv=64, cap=16, dtype=torch.float16):
    q = torch.zeros(b, s, hq, d, dtype=dtype)
    kc = torch.zeros(b, cap, hkv, d, dtype=dtype)
    vc = torch.zeros(b, cap, hkv, dv, dtype=dtype)
    kn = torch.zeros(b, s, hkv, d, dtype=dtype)
    vn = torch.zeros(b, s, hkv, dv, dtype=dtype)
    out = torch.zeros(b, s, hq, dv, dtype=dtype)
    return q, kc, vc, kn, vn, out


def _call(q, kc, vc, kn, vn, out, cos=None, sin=None, seq=0, rotary_dim=0, ws=None, ws_bytes=0):
    d = fa.describe
    r = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    return fa.lib.fa_kvcache_fwd(r(d(q)), r(d(kc)), r(d(vc)), r(d(kn)), r(d(vn)), r(d(cos)),
                                 r(d(sin)), None, rotary_dim, 0, 1, 0.0, r(d(out)), None, seq,
                                 ws, ws_bytes, None)


def test_rejects_null_q():
    q, kc, vc, kn, vn, out = _kv_tensors()
    assert _call(None, kc, vc, kn, vn, out) == fa.FA_ERR_INVALID_ARG
    assert "q is NULL" in fa.lib.fa_last_error().decode()


def test_rejects_fp32():
    q, kc, vc, kn, vn, out = _kv_tensors(dtype=torch.float32)
    assert _call(q, kc, vc, kn, vn, out) == fa.FA_ERR_UNSUPPORTED


def test_rejects_mixed_dtypes():
    q, kc, vc, kn, vn, out = _kv_tensors()
    assert _call(q, kc.bfloat16(), vc, kn, vn, out) == fa.FA_ERR_INVALID_ARG


def test_rejects_strided_head_dim():
    q, kc, vc, kn, vn, out = _kv_tensors(d=64)
    q2 = torch.zeros(2, 3, 4, 128, dtype=torch.float16)[..., ::2]
    assert _call(q2, kc, vc, kn, vn, out) == fa.FA_ERR_LAYOUT


def test_rejects_unaligned_row_stride():
    q, kc, vc, kn, vn, out = _kv_tensors(d=64)
    big = torch.zeros(2, 3, 4, 68, dtype=torch.float16)   # 136-byte rows
    assert _call(big[..., :64], kc, vc, kn, vn, out) == fa.FA_ERR_LAYOUT


def test_accepts_transposed_views_in_validation():
    # issue #1402 passes [b, h, s, d] tensors transposed to [b, s, h, d]: only the
    # head-dim stride must be 1; the call then fails later only for lack of a GPU
    q = torch.zeros(2, 4, 3, 64, dtype=torch.float16).transpose(1, 2)
    _, kc, vc, kn, vn, out = _kv_tensors()
    # a workspace of the planned size at a 256-byte boundary (never touched here)
    need = fa.fa_kvcache_workspace_size(q, kc, vc, kn)
    buf = torch.zeros(need + 256, dtype=torch.uint8)
    ws = (buf.data_ptr() + 255) // 256 * 256
    rc = _call(q, kc, vc, kn, vn, out, ws=ws, ws_bytes=need)
    assert rc in (fa.FA_OK, fa.FA_ERR_CUDA)


def test_rejects_bad_head_dims_and_groups():
    q, kc, vc, kn, vn, out = _kv_tensors(d=264, dv=264)
    assert _call(q, kc, vc, kn, vn, out) == fa.FA_ERR_UNSUPPORTED
    q, kc, vc, kn, vn, out = _kv_tensors(hq=3, hkv=2)
    assert _call(q, kc, vc, kn, vn, out) == fa.FA_ERR_INVALID_ARG


def test_rejects_half_new_rows_and_shape_mismatch():
    q, kc, vc, kn, vn, out = _kv_tensors()
    assert _call(q, kc, vc, kn, None, out) == fa.FA_ERR_INVALID_ARG
    assert _call(q, kc, vc, kn[:, :2], vn[:, :2], out) == fa.FA_ERR_INVALID_ARG
    assert _call(q, kc, vc, kn, vn, out[:, :, :, :32]) == fa.FA_ERR_INVALID_ARG


def test_rejects_bad_rotary():
    q, kc, vc, kn, vn, out = _kv_tensors()
    cos = torch.zeros(16, 32, dtype=torch.float16)
    sin = torch.zeros(16, 32, dtype=torch.float16)
    assert _call(q, kc, vc, kn, vn, out, cos, sin, rotary_dim=63) == fa.FA_ERR_INVALID_ARG
    assert _call(q, kc, vc, kn, vn, out, cos, sin, rotary_dim=66) == fa.FA_ERR_INVALID_ARG
    assert _call(q, kc, vc, kn, vn, out, cos, None, rotary_dim=64) == fa.FA_ERR_INVALID_ARG
    short = torch.zeros(4, 32, dtype=torch.float16)
    # scalar cache_seqlens: positions 2..4 exceed a 4-row table
    assert _call(q, kc, vc, kn, vn, out, short, short, seq=2, rotary_dim=64) == fa.FA_ERR_INVALID_ARG


def test_rejects_scalar_seqlens_past_capacity():
    q, kc, vc, kn, vn, out = _kv_tensors(cap=16)
    assert _call(q, kc, vc, kn, vn, out, seq=14) == fa.FA_ERR_INVALID_ARG
    assert _call(q, kc, vc, kn, vn, out, seq=-1) == fa.FA_ERR_INVALID_ARG


def test_workspace_checked_before_launch():
    # a decode-shaped call (one new row, GQA 4) over a cache large enough to split
    kc = torch.zeros(2, 4096, 2, 128, dtype=torch.bfloat16)
    vc = torch.zeros(2, 4096, 2, 128, dtype=torch.bfloat16)
    q = torch.zeros(2, 1, 8, 128, dtype=torch.bfloat16)
    kn = torch.zeros(2, 1, 2, 128, dtype=torch.bfloat16)
    vn = torch.zeros(2, 1, 2, 128, dtype=torch.bfloat16)
    out = torch.zeros(2, 1, 8, 128, dtype=torch.bfloat16)
    need = fa.fa_kvcache_workspace_size(q, kc, vc, kn, 0)
    assert need > 0
    assert _call(q, kc, vc, kn, vn, out, seq=5) == fa.FA_ERR_WORKSPACE


def test_workspace_plans():
    # decode: split partials (fp32 out rows + lse) for every split of every row
    kc = torch.zeros(2, 4096, 2, 128, dtype=torch.bfloat16)
    q = torch.zeros(2, 1, 8, 128, dtype=torch.bfloat16)
    kn = torch.zeros(2, 1, 2, 128, dtype=torch.bfloat16)
    n = fa.fa_kvcache_workspace_size(q, kc, kc, kn, 64)
    rows_per_split = 2 * 8 * 1
    assert n % 256 == 0 and n >= rows_per_split * 129 * 4 * 2
    # prefill with RoPE: one rotated copy of q
    q = torch.zeros(2, 100, 4, 128, dtype=torch.float16)
    kc = torch.zeros(2, 512, 4, 128, dtype=torch.float16)
    kn = torch.zeros(2, 100, 4, 128, dtype=torch.float16)
    n = fa.fa_kvcache_workspace_size(q, kc, kc, kn, 128)
    assert n >= 2 * 100 * 4 * 128 * 2
    assert fa.fa_kvcache_workspace_size(q, kc, kc, kn, 0) == 0


def test_fa_fwd_validation():
    q = torch.zeros(1, 8, 2, 64, dtype=torch.float16)
    k = torch.zeros(1, 8, 2, 64, dtype=torch.float16)
    v = torch.zeros(1, 8, 2, 32, dtype=torch.float16)
    out = torch.zeros(1, 8, 2, 64, dtype=torch.float16)   # wrong: d_v is 32
    d = fa.describe
    rc = fa.lib.fa_fwd(ctypes.byref(d(q)), ctypes.byref(d(k)), ctypes.byref(d(v)), 1, 0.0,
                       ctypes.byref(d(out)), None, None, 0, None)
    assert rc == fa.FA_ERR_INVALID_ARG


def test_kernel_events_hook_arguments():
    # both or neither: a lone event is rejected, clearing is always allowed
    assert fa.lib.fa_set_kernel_events(ctypes.c_void_p(16), None) == fa.FA_ERR_INVALID_ARG
    assert fa.lib.fa_set_kernel_events(None, ctypes.c_void_p(16)) == fa.FA_ERR_INVALID_ARG
    assert fa.lib.fa_set_kernel_events(None, None) == fa.FA_OK


def test_binding_rejects_host_tensors():
    """The C ABI takes raw device addresses and cannot tell a host pointer from
    a device one, so the binding refuses CPU tensors (and tensors on another
    device than q) before anything is enqueued."""
    q, kc, vc, kn, vn, out = _kv_tensors()
    seq = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_kvcache_fwd(q, kc, vc, kn, vn, cache_seqlens=seq, causal=True)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_kvcache_fwd_noalloc(q, kc, vc, kn, vn, cache_seqlens=3, causal=True)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_fwd(q, kc, vc, causal=True)
    cos = torch.zeros(16, 32, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_rotary(q, cos, cos.clone(), 0)
    cu = torch.tensor([0, 3], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_fwd_varlen(q[0], kc[0], vc[0], cu, cu, 3)
    lse = torch.zeros(2, 4, 3)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_bwd(q, kc[:, :3], vc[:, :3], out, out, lse)


def test_descriptor_cache_keys_on_every_field():
    # the binding reuses a descriptor only for the same address, dtype, shape and strides
    base = torch.zeros(4, 6, 2, 64, dtype=torch.float16)
    d1 = fa.describe(base)
    assert fa.describe(base) is d1
    assert (d1.data, d1.ndim, list(d1.shape), list(d1.stride)) == (base.data_ptr(), 4, [4, 6, 2, 64],
                                                                    [768, 128, 64, 1])
    view = base[:, :3]                                   # same address, other shape
    d2 = fa.describe(view)
    assert d2 is not d1 and list(d2.shape) == [4, 3, 2, 64] and d2.data == d1.data
    t = base.transpose(1, 2)                             # same address, other strides
    d3 = fa.describe(t)
    assert list(d3.stride) == [768, 64, 128, 1] and list(d3.shape) == [4, 2, 6, 64]
    other = base.view(torch.bfloat16)                    # same address and layout, other dtype
    assert fa.describe(other).dtype != d1.dtype
    small = torch.zeros(5, 3, dtype=torch.float16)       # rank below 4 pads with zeros
    d4 = fa.describe(small)
    assert d4.ndim == 2 and list(d4.shape) == [5, 3, 0, 0] and list(d4.stride) == [3, 1, 0, 0]
