"""Sliding-window attention (fa_fwd_window / fa_kvcache_fwd_window) against the
float64 oracle on the GPU, on the decode, one-tile, two-tile and generic
kernels.  Tolerances are those of the attention contract."""
import numpy as np
import pytest
import torch

import oracle
import rotary_embedding_b200 as fa
import workloads as W
from parity_util import LSE_TOL, OUT_TOL, ulp_distance

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _draw(g, shape, dtype):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(DT[dtype])


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
@pytest.mark.parametrize("causal,window", [(True, (100, -1)), (True, (0, -1)), (False, (40, 40)),
                                           (False, (0, 0)), (False, (-1, 60)), (True, (5000, -1)),
                                           (False, (300, -1))])
def test_dense_window(cuda_device, prefill_tiles, dims, causal, window):
    d_qk, d_v = dims
    dtype = "bf16"
    g = torch.Generator().manual_seed(hash((prefill_tiles, dims, causal, window)) % 1000)
    b, s_q, s_k, h_q, h_kv = 2, 300, 700, 4, 2
    q = _draw(g, (b, s_q, h_q, d_qk), dtype)
    k = _draw(g, (b, s_k, h_kv, d_qk), dtype)
    v = _draw(g, (b, s_k, h_kv, d_v), dtype)
    out, lse = fa.fa_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=causal,
                         window=window)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    r_out, r_lse = oracle.fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                              window=window)
    _check(out, lse, r_out, r_lse, dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [32, 96])
def test_dense_window_generic_kernel(cuda_device, d):
    g = torch.Generator().manual_seed(d)
    q = _draw(g, (1, 50, 2, d), "fp16")
    k = _draw(g, (1, 90, 2, d), "fp16")
    v = _draw(g, (1, 90, 2, d), "fp16")
    for causal, window in ((True, (7, -1)), (False, (3, 11))):
        out, lse = fa.fa_fwd(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=causal,
                             window=window)
        torch.cuda.synchronize()
        r_out, r_lse = oracle.fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                                  window=window)
        _check(out, lse, r_out, r_lse, "fp16")


def _kv_case(seed, b, s_q, h_q, h_kv, d, cap, lens, r, dtype):
    g = torch.Generator().manual_seed(seed)
    q = _draw(g, (b, s_q, h_q, d), dtype)
    kn = _draw(g, (b, s_q, h_kv, d), dtype)
    vn = _draw(g, (b, s_q, h_kv, d), dtype)
    kc = _draw(g, (b, cap, h_kv, d), dtype)
    vc = _draw(g, (b, cap, h_kv, d), dtype)
    seq = torch.tensor(lens, dtype=torch.int32)
    cos, sin = W.rotary_tables(cap, r, 10000.0, DT[dtype]) if r else (None, None)
    return q, kn, vn, kc, vc, seq, cos, sin


@pytest.mark.gpu
@pytest.mark.parametrize("s_q,h_q,h_kv", [(1, 8, 2), (2, 4, 4), (64, 8, 2)])
@pytest.mark.parametrize("window", [(64, -1), (5, -1), (1000, -1), (130, -1)])
def test_kvcache_window(cuda_device, s_q, h_q, h_kv, window):
    dtype, d, cap, r = "bf16", 128, 1024, 64
    lens = [900, 37, 600]
    q, kn, vn, kc, vc, seq, cos, sin = _kv_case(11 + s_q + window[0], 3, s_q, h_q, h_kv, d, cap, lens, r, dtype)
    dev = lambda t: t.to(cuda_device) if t is not None else None  # noqa: E731
    kcd, vcd = dev(kc), dev(vc)
    out, lse = fa.fa_kvcache_fwd(dev(q), kcd, vcd, dev(kn), dev(vn), dev(cos), dev(sin), dev(seq), r,
                                 False, True, window=window)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    r_out, r_lse, r_kc, r_vc = oracle.kvcache_fwd(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                                  kn.double().numpy(), vn.double().numpy(), cos.double().numpy(),
                                                  sin.double().numpy(), lens, rotary_dim=r, causal=True,
                                                  fmt=dtype, window=window)
    _check(out, lse, r_out, r_lse, dtype)
    assert torch.equal(vcd.cpu(), torch.from_numpy(r_vc).to(DT[dtype]))
    assert ulp_distance(kcd.cpu(), torch.from_numpy(r_kc).to(DT[dtype])).max() <= 1


@pytest.mark.gpu
def test_window_rejects_bad_bounds(cuda_device):
    q = torch.zeros(1, 4, 2, 64, dtype=torch.float16, device=cuda_device)
    with pytest.raises(fa.FaError):
        fa.fa_fwd(q, q, q, window=(-2, 0))


@pytest.mark.gpu
def test_window_prefill_full_size_sampled(cuda_device):
    # the benchmarked workload at full size; sampled (batch, head) rows against the oracle
    w = W.CONFIGS["window-prefill"]
    inp = W.make_inputs(w, seed=0)
    q, k, v = (inp[n].to(cuda_device) for n in ("q", "k", "v"))
    out, lse = fa.fa_fwd(q, k, v, causal=w.causal, window=w.window)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    for bi, h, i0 in ((0, 0, 0), (1, 7, 3000), (0, 15, 8192 - 256)):
        qs = inp["q"][bi:bi + 1, i0:i0 + 256, h:h + 1].double().numpy()
        # rows i0 .. i0 + 255 see keys up to i0 + 255 and down to i0 - 1024
        k0 = max(0, i0 - 1024)
        ks = inp["k"][bi:bi + 1, k0:i0 + 256, h:h + 1].double().numpy()
        vs = inp["v"][bi:bi + 1, k0:i0 + 256, h:h + 1].double().numpy()
        r_out, r_lse = oracle.fwd(qs, ks, vs, causal=True, window=w.window)
        _check(out[bi:bi + 1, i0:i0 + 256, h:h + 1], lse[bi:bi + 1, h:h + 1, i0:i0 + 256], r_out, r_lse, w.dtype)
