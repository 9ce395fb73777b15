"""Standalone rotary (fa_rotary): host validation on the CPU, and the CUDA path
against the float64 oracle on the GPU.  The rotary kernel rounds fp32 pair
arithmetic to the element type; the oracle rounds the float64 result, so the
two may differ by one unit in the last place (the contract for rotated rows)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import rotary_embedding_b200 as fa
import workloads as W
from parity_util import ulp_distance

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _raw_call(x, cos, sin, rotary_dim, out, cu=None, n_seqs=0, offsets=0):
    d = fa.describe
    r = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    return fa.lib.fa_rotary(r(d(x)), r(d(cos)), r(d(sin)), None, offsets, cu, n_seqs, rotary_dim, 0, 0,
                            r(d(out)), None)


def test_rotary_host_validation():
    x = torch.zeros(2, 3, 4, 64, dtype=torch.float16)
    cos = torch.zeros(16, 32, dtype=torch.float16)
    sin = torch.zeros(16, 32, dtype=torch.float16)
    out = torch.zeros_like(x)
    assert _raw_call(x, cos, sin, 63, out) == fa.FA_ERR_INVALID_ARG          # odd rotary_dim
    assert _raw_call(x, cos, sin, 66, out) == fa.FA_ERR_INVALID_ARG          # rotary_dim > d
    assert _raw_call(x, cos[:, :8], sin[:, :8], 32, out) == fa.FA_ERR_INVALID_ARG   # too few columns
    assert _raw_call(x, cos, sin, 64, out[:, :2]) == fa.FA_ERR_INVALID_ARG   # out shape
    assert _raw_call(x, None, None, 64, out) == fa.FA_ERR_INVALID_ARG        # tables missing
    assert _raw_call(x, cos, sin, 64, out, cu=ctypes.c_void_p(16), n_seqs=1) == fa.FA_ERR_INVALID_ARG  # b != 1
    big = torch.zeros(1, 2, 2, 264, dtype=torch.float16)
    assert _raw_call(big, None, None, 0, torch.zeros_like(big)) == fa.FA_ERR_UNSUPPORTED


def _inputs(shape, dtype, r, s_ro, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32).to(DT[dtype])
    if r > 0:
        cos, sin = W.rotary_tables(s_ro, r, 10000.0, DT[dtype])
    else:
        cos = sin = None
    return x, cos, sin


def _expect(x, cos, sin, offsets, r, inter, conj, dtype, cu=None):
    c = cos.double().numpy() if cos is not None else np.zeros((0, 0))
    s = sin.double().numpy() if sin is not None else np.zeros((0, 0))
    y = oracle.rotary(x.double().numpy(), c, s, offsets, r, inter, conj, cu_seqlens=cu, fmt=dtype)
    return torch.from_numpy(y).to(DT[dtype])


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("d,r", [(64, 64), (128, 64), (128, 128), (192, 128), (256, 256), (64, 8), (128, 0)])
@pytest.mark.parametrize("inter", [False, True])
@pytest.mark.parametrize("conj", [False, True])
def test_rotary_batched(cuda_device, dtype, d, r, inter, conj):
    b, s, h = 3, 37, 5
    x, cos, sin = _inputs((b, s, h, d), dtype, r, 200, seed=d + r)
    offs = torch.tensor([0, 41, 150], dtype=torch.int32)
    xd = x.to(cuda_device)
    out = fa.fa_rotary(xd, cos.to(cuda_device) if cos is not None else None,
                       sin.to(cuda_device) if sin is not None else None, offs.to(cuda_device), r, inter, conj)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    ref = _expect(x, cos, sin, offs.numpy(), r, inter, conj, dtype)
    dist = ulp_distance(out.cpu(), ref)
    assert dist.max() <= 1, f"{dist.max()} ulp"
    if r < d:   # dims past rotary_dim are bit copies
        assert torch.equal(out.cpu()[..., r:], x[..., r:])


@pytest.mark.gpu
@pytest.mark.parametrize("h", [2, 6, 12])
@pytest.mark.parametrize("inter", [False, True])
@pytest.mark.parametrize("in_place", [False, True])
def test_rotary_head_groups(cuda_device, h, inter, in_place):
    # heads are taken in groups of 4, 2 or 1 per thread; partial rotary_dim
    # exercises the copied chunks of every group
    b, s, d, r = 2, 23, 128, 64
    x, cos, sin = _inputs((b, s, h, d), "bf16", r, 80, seed=100 + h)
    offs = torch.tensor([3, 40], dtype=torch.int32)
    xd = x.to(cuda_device)
    out = fa.fa_rotary(xd, cos.to(cuda_device), sin.to(cuda_device), offs.to(cuda_device), r, inter, False,
                       out=xd if in_place else None)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    ref = _expect(x, cos, sin, offs.numpy(), r, inter, False, "bf16")
    assert ulp_distance(out.cpu(), ref).max() <= 1
    assert torch.equal(out.cpu()[..., r:], x[..., r:])


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_rotary_scalar_offset_in_place_and_transposed(cuda_device, dtype):
    b, s, h, d, r = 2, 19, 4, 128, 96
    x, cos, sin = _inputs((b, h, s, d), dtype, r, 64, seed=7)
    xt = x.transpose(1, 2)                       # [b, s, h, d] view with head stride d*s... as in issue #1402
    ref = _expect(xt.contiguous(), cos, sin, 5, r, False, False, dtype)
    xd = x.to(cuda_device).transpose(1, 2).contiguous()
    out = fa.fa_rotary(xd, cos.to(cuda_device), sin.to(cuda_device), 5, r, False, False, out=xd)
    torch.cuda.synchronize()
    assert out.data_ptr() == xd.data_ptr()
    assert ulp_distance(out.cpu(), ref).max() <= 1
    # a non-contiguous (transposed) input view, separate output
    xv = x.to(cuda_device).transpose(1, 2)
    out2 = fa.fa_rotary(xv, cos.to(cuda_device), sin.to(cuda_device), 5, r, False, False,
                        out=torch.empty(xv.shape, dtype=xv.dtype, device=cuda_device))
    torch.cuda.synchronize()
    assert ulp_distance(out2.cpu(), ref).max() <= 1


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("inter", [False, True])
def test_rotary_packed_varlen(cuda_device, dtype, inter):
    lens = [5, 1, 0, 33, 12]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total, h, d, r = int(cu[-1]), 3, 128, 128
    x, cos, sin = _inputs((total, h, d), dtype, r, 100, seed=11)
    offs = np.array([0, 7, 3, 50, 60], dtype=np.int32)
    out = fa.fa_rotary(x.to(cuda_device), cos.to(cuda_device), sin.to(cuda_device),
                       torch.from_numpy(offs).to(cuda_device), r, inter, True,
                       cu_seqlens=torch.from_numpy(cu).to(cuda_device))
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    ref = _expect(x, cos, sin, offs, r, inter, True, dtype, cu=cu)
    assert ulp_distance(out.cpu(), ref).max() <= 1


@pytest.mark.gpu
def test_rotary_packed_rows_outside_sequences_are_copied(cuda_device):
    cu = np.array([2, 6, 9], dtype=np.int32)     # rows 0-1 and 9-10 belong to no sequence
    x, cos, sin = _inputs((11, 2, 64), "bf16", 64, 32, seed=12)
    out = fa.fa_rotary(x.to(cuda_device), cos.to(cuda_device), sin.to(cuda_device), 4, 64, False, False,
                       cu_seqlens=torch.from_numpy(cu).to(cuda_device))
    torch.cuda.synchronize()
    o = out.cpu()
    assert torch.equal(o[:2], x[:2]) and torch.equal(o[9:], x[9:])
    ref = _expect(x[2:9], cos, sin, 4, 64, False, False, "bf16", cu=cu - 2)
    assert ulp_distance(o[2:9], ref).max() <= 1


@pytest.mark.gpu
def test_rotary_conjugate_undoes_rotation_on_gpu(cuda_device):
    # the GPU's own round trip: rotate, then conjugate, returns x within rounding
    x, cos, sin = _inputs((2, 64, 8, 128), "fp16", 128, 128, seed=13)
    xd, c, s = x.to(cuda_device), cos.to(cuda_device), sin.to(cuda_device)
    back = fa.fa_rotary(fa.fa_rotary(xd, c, s, 0, 128, False, False), c, s, 0, 128, False, True)
    torch.cuda.synchronize()
    assert (back.float() - xd.float()).abs().max().item() <= 4e-3


@pytest.mark.gpu
def test_rotary_position_outside_table_is_reported(cuda_device):
    x, cos, sin = _inputs((1, 4, 2, 64), "fp16", 64, 8, seed=14)
    xd = x.to(cuda_device)
    fa.fa_device_status()
    out = fa.fa_rotary(xd, cos.to(cuda_device), sin.to(cuda_device), 6, 64, False, False)   # rows 6..9 vs 8 rows
    assert fa.fa_device_status() == fa.FA_ERR_DEVICE_PRECONDITION
    o = out.cpu()
    ref = _expect(x[:, :2], cos, sin, 6, 64, False, False, "fp16")
    assert ulp_distance(o[:, :2], ref).max() <= 1     # rows 6, 7 are inside the table


@pytest.mark.gpu
def test_rotary_full_size_workload_sampled(cuda_device):
    # the benchmarked workload at full size, in the bench's call; sampled rows against the oracle
    w = W.CONFIGS["rotary-q"]
    inp = W.make_inputs(w, seed=0)
    dev = {k: v.to(cuda_device) for k, v in inp.items()}
    out = fa.fa_rotary(dev["q"], dev["cos"], dev["sin"], dev["cache_seqlens"], w.rotary_dim, w.interleaved,
                       w.conjugate)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    o = out.cpu()
    for b in range(w.batch):
        for i0 in (0, 1777, w.s_q - 40):
            x = inp["q"][b:b + 1, i0:i0 + 40]
            ref = _expect(x, inp["cos"], inp["sin"], int(inp["cache_seqlens"][b]) + i0, w.rotary_dim,
                          w.interleaved, w.conjugate, w.dtype)
            assert ulp_distance(o[b:b + 1, i0:i0 + 40], ref).max() <= 1
