"""Attention over packed sequences (fa_fwd_varlen): host validation on the CPU,
and the CUDA path against the float64 oracle (the pinned dense attention per
sequence) on the GPU, on both tcgen05 prefill kernels."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import rotary_embedding_b200 as fa
import workloads as W
from parity_util import LSE_TOL, OUT_TOL

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def test_varlen_host_validation():
    q = torch.zeros(10, 4, 64, dtype=torch.float16)
    d = fa.describe
    r = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    call = lambda qq, kk, vv, oo, cu=ctypes.c_void_p(16): fa.lib.fa_fwd_varlen(  # noqa: E731
        r(d(qq)), r(d(kk)), r(d(vv)), cu, cu, 1, 10, 1, -1, -1, 0.0, r(d(oo)), None, None)
    assert call(q, q, q, q, cu=None) == fa.FA_ERR_INVALID_ARG                  # cu_seqlens missing
    assert call(q, q[:, :3], q[:, :3], q) == fa.FA_ERR_INVALID_ARG             # h_q not a multiple
    q32 = torch.zeros(10, 4, 32, dtype=torch.float16)
    assert call(q32, q32, q32, q32) == fa.FA_ERR_UNSUPPORTED                   # head dim
    assert call(q, q, q, q[:, :, :32]) == fa.FA_ERR_INVALID_ARG                # out shape


def _case(seed, lens_q, lens_k, h_q, h_kv, d_qk, d_v, dtype):
    g = torch.Generator().manual_seed(seed)
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q = torch.randn((int(cq[-1]), h_q, d_qk), generator=g).to(DT[dtype])
    k = torch.randn((int(ck[-1]), h_kv, d_qk), generator=g).to(DT[dtype])
    v = torch.randn((int(ck[-1]), h_kv, d_v), generator=g).to(DT[dtype])
    return q, k, v, cq, ck


def _check(out, lse, r_out, r_lse, dtype):
    err = (out.float().cpu().double() - torch.from_numpy(r_out)).abs().max().item()
    assert err <= OUT_TOL[dtype], f"out max|err| {err}"
    l = lse.cpu().double().numpy()
    fin = np.isfinite(r_lse)
    assert np.array_equal(np.isfinite(l), fin)
    if fin.any():
        assert np.abs(l[fin] - r_lse[fin]).max() <= LSE_TOL


@pytest.mark.gpu
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (192, 128)])
@pytest.mark.parametrize("causal,window", [(True, (-1, -1)), (False, (-1, -1)), (True, (90, -1))])
def test_varlen_parity(cuda_device, prefill_tiles, dims, causal, window):
    lens_q = [130, 1, 0, 300, 64, 257]
    lens_k = [200, 77, 5, 300, 64, 257]      # s_k >= s_q (bottom-right), a key-only sequence
    q, k, v, cq, ck = _case(7, lens_q, lens_k, 8, 2, dims[0], dims[1], "bf16")
    dev = cuda_device
    out, lse = fa.fa_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(cq).to(dev),
                                torch.from_numpy(ck).to(dev), max(lens_q), causal=causal, window=window)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    r_out, r_lse = oracle.fwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), cq, ck,
                                     causal=causal, window=window)
    _check(out, lse, r_out, r_lse, "bf16")


@pytest.mark.gpu
def test_varlen_bad_offsets_are_reported(cuda_device):
    q, k, v, cq, ck = _case(8, [16, 16], [16, 16], 2, 2, 64, 64, "fp16")
    bad = ck.copy()
    bad[2] = 1000                                   # past the packed key rows
    dev = cuda_device
    fa.fa_device_status()
    out, _ = fa.fa_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(cq).to(dev),
                              torch.from_numpy(bad).to(dev), 16, causal=True)
    assert fa.fa_device_status() == fa.FA_ERR_DEVICE_PRECONDITION
    r_out, _ = oracle.fwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), cq[:2], ck[:2],
                                 causal=True)
    assert (out[:16].float().cpu().double() - torch.from_numpy(r_out[:16])).abs().max().item() <= 2e-3


@pytest.mark.gpu
def test_varlen_full_size_workload_sampled(cuda_device):
    w = W.CONFIGS["varlen-prefill"]
    inp = W.make_inputs(w, seed=0)
    dev = {n: t.to(cuda_device) for n, t in inp.items()}
    out, lse = fa.fa_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["cu_seqlens"], dev["cu_seqlens"], w.s_q,
                                causal=w.causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    cu = inp["cu_seqlens"].numpy()
    for s_idx, h in ((0, 0), (3, 9), (7, 15)):
        q0, q1 = cu[s_idx], cu[s_idx + 1]
        r_out, r_lse = oracle.fwd(inp["q"][None, q0:q1, h:h + 1].double().numpy(),
                                  inp["k"][None, q0:q1, h:h + 1].double().numpy(),
                                  inp["v"][None, q0:q1, h:h + 1].double().numpy(), causal=True)
        _check(out[q0:q1, h:h + 1], lse[h:h + 1, q0:q1], r_out[0], r_lse[0], w.dtype)
