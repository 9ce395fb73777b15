"""Attention backward (fa_bwd: dq, dk, dv with d_qk != d_v, GQA, causal and
window masks) against the float64 oracle's gradient.

Tolerance (normwise, per tensor): max|got - ref| <= TOL * max|ref|.  The
kernels round P and dS to the element type as MMA operands, read D_i from
the rounded out, and round dq, dk, dv; a numpy model of exactly those
roundings (_rounding_model) differs from the float64 gradient by at most
5.1e-3 (bf16) and 6.9e-4 (fp16) of max|ref| on these shapes.  TOL is four
times that; test_bwd_tolerance_covers_the_rounding_model keeps the margin.
Gradients that no visible (query, key) pair reaches (a query row that sees no
key, a key no query sees) must be exactly zero.  Gradients that are zero only
by cancellation (a row with one visible key has P = 1, so dP - D = 0) are
held to TOL like every other element: the kernel's P = exp2(s - lse) and
its D from the rounded out leave residues of a few ulps there."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import rotary_embedding_b200 as fa
import workloads as W

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}
TOL = {"bf16": 2e-2, "fp16": 3e-3}


def test_bwd_host_validation():
    d = fa.describe
    r = lambda t: ctypes.byref(d(t))  # noqa: E731
    q = torch.zeros(1, 8, 2, 64, dtype=torch.float16)
    lse = torch.zeros(1, 2, 8, dtype=torch.float32)
    ws = torch.zeros(4096, dtype=torch.uint8)

    def call(qq=q, kk=q, vv=q, oo=q, dd=q, ll=lse, dq=q, dk=q, dv=q, wl=-1, wsb=4096):
        return fa.lib.fa_bwd(r(qq), r(kk), r(vv), r(oo), r(dd),
                             ctypes.c_void_p(ll.data_ptr()) if ll is not None else None, 1, wl, -1, 0.0,
                             r(dq), r(dk), r(dv), ctypes.c_void_p(ws.data_ptr()), wsb, None)
    q32 = torch.zeros(1, 8, 2, 32, dtype=torch.float16)
    assert call(q32, q32, q32, q32, q32, dq=q32, dk=q32, dv=q32) == fa.FA_ERR_UNSUPPORTED   # head dim
    assert call(oo=q[:, :4]) == fa.FA_ERR_INVALID_ARG                                        # out shape
    assert call(dd=q[:, :, :1]) == fa.FA_ERR_INVALID_ARG                                     # dout shape
    assert call(dk=q[:, :4]) == fa.FA_ERR_INVALID_ARG                                        # dk shape
    assert call(ll=None) == fa.FA_ERR_INVALID_ARG                                            # lse missing
    assert call(wl=-2) == fa.FA_ERR_INVALID_ARG                                              # window bound
    assert call(wsb=16) == fa.FA_ERR_WORKSPACE                                               # workspace
    assert call(kk=q.to(torch.bfloat16)) == fa.FA_ERR_INVALID_ARG                            # dtype mix
    # lse * log2(e) and D_i, each fp32 [b, h_q, s_q rounded up to 64 rows], 256-byte aligned
    assert fa.fa_bwd_workspace_size(q) == 2 * 1 * 2 * 64 * 4


def _case(seed, b, s_q, s_k, h_q, h_kv, d_qk, d_v, dtype):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *sh: torch.randn(sh, generator=g, dtype=torch.float32).to(DT[dtype])  # noqa: E731
    return mk(b, s_q, h_q, d_qk), mk(b, s_k, h_kv, d_qk), mk(b, s_k, h_kv, d_v), mk(b, s_q, h_q, d_v)


def _forward_inputs(q, k, v, causal, window, dtype):
    """out (rounded to the element type) and lse of the oracle's forward."""
    out, lse = oracle.fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal=causal,
                          window=window)
    return torch.from_numpy(out).to(DT[dtype]), torch.from_numpy(lse).float()


def _unreached(q, k, v, causal, window):
    """Masks of the gradient rows no visible pair reaches: query rows with no
    visible key (the oracle forward's lse is -inf) and keys no query sees (the
    oracle's dv for dout = 1 is zero: it sums P > 0 over the rows seeing them)."""
    q, k, v = (t.double().numpy() for t in (q, k, v))
    _, lse = oracle.fwd(q, k, v, causal=causal, window=window)
    ones = np.ones(q.shape[:3] + (v.shape[3],))
    _, _, dv1 = oracle.bwd(q, k, v, ones, causal=causal, window=window)
    row_none = np.isneginf(lse).transpose(0, 2, 1)[..., None]     # [b, s_q, h_q, 1]
    key_none = (dv1 == 0.0).all(axis=-1, keepdims=True)          # [b, s_k, h_kv, 1]
    return row_none, key_none


def _check(got, ref, dtype, unreached=None):
    for x, (name, a, r) in enumerate(zip(("dq", "dk", "dv"), got, ref)):
        a = a.float().cpu().double().numpy()
        scale = max(np.abs(r).max(), 1e-30)
        err = np.abs(a - r).max()
        assert err <= TOL[dtype] * scale, f"{name}: max|err| {err:.3e} vs max|ref| {scale:.3e}"
        if unreached is not None:
            mask = np.broadcast_to(unreached[0] if x == 0 else unreached[1], a.shape)
            assert np.all(a[mask] == 0.0), f"{name}: nonzero where no visible pair reaches"


def _rounding_model(q, k, v, do, out, lse, causal, window, dtype):
    """The kernels' arithmetic with their roundings and nothing else: P from
    the forward's lse in fp32, P and dS rounded to the element type as MMA
    operands, D from the rounded out, dq/dk/dv rounded; products otherwise
    exact.  Used only to derive TOL."""
    def rnd(x):
        return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(DT[dtype]).double().numpy()
    b, s_q, h_q, d = q.shape
    s_k, h_kv = k.shape[1], k.shape[2]
    g = h_q // h_kv
    sc = 1.0 / np.sqrt(d)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    i = np.arange(s_q)[:, None]
    j = np.arange(s_k)[None, :]
    dist = i + s_k - s_q - j
    vis = np.ones((s_q, s_k), bool)
    if causal:
        vis &= dist >= 0
    if window[0] >= 0:
        vis &= dist <= window[0]
    if window[1] >= 0:
        vis &= -dist <= window[1]
    for bi in range(b):
        for h in range(h_q):
            hk = h // g
            s = (q[bi, :, h] @ k[bi, :, hk].T).astype(np.float32)
            L = lse[bi, h][:, None].astype(np.float32)
            p = np.where(vis, np.exp2(s * np.float32(sc * np.log2(np.e)) - L * np.float32(np.log2(np.e))), 0)
            dp = (do[bi, :, h] @ v[bi, :, hk].T).astype(np.float32)
            dsum = (do[bi, :, h] * out[bi, :, h]).sum(-1).astype(np.float32)[:, None]
            ds = (p * (dp - dsum)).astype(np.float32)
            dv[bi, :, hk] += rnd(p).T @ do[bi, :, h]
            dk[bi, :, hk] += sc * (rnd(ds).T @ q[bi, :, h])
            dq[bi, :, h] = sc * (rnd(ds) @ k[bi, :, hk])
    return rnd(dq), rnd(dk), rnd(dv)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_bwd_tolerance_covers_the_rounding_model(dtype):
    """TOL stays at least three times the normwise error that the kernels'
    roundings alone cause, on shapes of the GPU parity cases."""
    worst = 0.0
    for (d_qk, d_v), (causal, window), shape in (((192, 128), (True, (-1, -1)), (2, 100, 170, 4, 1)),
                                                ((64, 64), (False, (30, 20)), (1, 200, 64, 2, 1)),
                                                ((128, 128), (True, (40, -1)), (1, 130, 130, 2, 2))):
        b, s_q, s_k, h_q, h_kv = shape
        q, k, v, do = (t.double().numpy() for t in _case(d_qk + s_q + s_k, b, s_q, s_k, h_q, h_kv, d_qk, d_v, dtype))
        out, lse = oracle.fwd(q, k, v, causal=causal, window=window)
        out = torch.from_numpy(out).to(DT[dtype]).double().numpy()
        ref = oracle.bwd(q, k, v, do, causal=causal, window=window)
        got = _rounding_model(q, k, v, do, out, lse, causal, window, dtype)
        for a, r in zip(got, ref):
            worst = max(worst, np.abs(a - r).max() / np.abs(r).max())
    assert 3.0 * worst <= TOL[dtype], (worst, TOL[dtype])


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (192, 128)])
@pytest.mark.parametrize("causal,window", [(True, (-1, -1)), (False, (-1, -1)), (True, (40, -1)),
                                           (False, (30, 20))])
@pytest.mark.parametrize("shape", [(2, 100, 170, 4, 1), (1, 130, 130, 2, 2), (1, 200, 64, 2, 1)])
def test_bwd_parity(cuda_device, dtype, dims, causal, window, shape):
    b, s_q, s_k, h_q, h_kv = shape
    d_qk, d_v = dims
    q, k, v, do = _case(d_qk + s_q + s_k, b, s_q, s_k, h_q, h_kv, d_qk, d_v, dtype)
    out, lse = _forward_inputs(q, k, v, causal, window, dtype)
    dev = cuda_device
    got = fa.fa_bwd(q.to(dev), k.to(dev), v.to(dev), out.to(dev), do.to(dev), lse.to(dev), causal=causal,
                    window=window)
    torch.cuda.synchronize()
    ref = oracle.bwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                     causal=causal, window=window)
    _check(got, ref, dtype, _unreached(q, k, v, causal, window))


@pytest.mark.gpu
def test_bwd_after_gpu_forward_and_deterministic(cuda_device):
    # the chain a training step runs: forward on the GPU, then its out and lse into the backward
    dtype, dev = "bf16", cuda_device
    q, k, v, do = _case(5, 2, 257, 257, 8, 2, 192, 128, dtype)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    out, lse = fa.fa_fwd(qd, kd, vd, causal=True)
    g1 = fa.fa_bwd(qd, kd, vd, out, dod, lse, causal=True)
    g2 = fa.fa_bwd(qd, kd, vd, out, dod, lse, causal=True)
    torch.cuda.synchronize()
    for a, b_ in zip(g1, g2):
        assert torch.equal(a, b_)          # no atomics: bit-identical
    ref = oracle.bwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                     causal=True)
    _check(g1, ref, dtype)


@pytest.mark.gpu
def test_bwd_empty_sides(cuda_device):
    dev = cuda_device
    q, k, v, do = _case(6, 1, 0, 40, 2, 1, 64, 64, "fp16")
    dq, dk, dv = fa.fa_bwd(q.to(dev), k.to(dev), v.to(dev), do.to(dev), do.to(dev),
                           torch.empty(1, 2, 0, device=dev), causal=True)
    torch.cuda.synchronize()
    assert dk.abs().max().item() == 0 and dv.abs().max().item() == 0     # no queries: no gradient
    q, k, v, do = _case(7, 1, 16, 0, 2, 1, 64, 64, "fp16")
    out = torch.zeros(1, 16, 2, 64, dtype=torch.float16)
    lse = torch.full((1, 2, 16), float("-inf"))
    dq, dk, dv = fa.fa_bwd(q.to(dev), k.to(dev), v.to(dev), out.to(dev), do.to(dev), lse.to(dev), causal=True)
    torch.cuda.synchronize()
    assert dq.abs().max().item() == 0                                    # no keys: no gradient


@pytest.mark.gpu
def test_bwd_full_size_workload_sampled(cuda_device):
    # the benchmarked backward workload at full size, in the bench's call; dq on
    # sampled query rows and dk, dv on sampled key rows against the oracle
    w = W.CONFIGS["mla-backward"]
    inp = W.make_inputs(w, seed=0)
    dev = {n: t.to(cuda_device) for n, t in inp.items()}
    out, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=w.causal)
    dq, dk, dv = fa.fa_bwd(dev["q"], dev["k"], dev["v"], out, dev["dout"], lse, causal=w.causal)
    torch.cuda.synchronize()
    f64 = lambda t: t.double().numpy()  # noqa: E731
    S = w.s_q
    for bi, h, i0 in ((0, 0, 0), (1, 5, 2000), (3, 15, S - 64)):
        # rows i0 .. i0+63 see keys 0 .. i0+63 (causal, s_q = s_k)
        sl = slice(i0, i0 + 64)
        ref = oracle.bwd(f64(inp["q"][bi:bi + 1, sl, h:h + 1]), f64(inp["k"][bi:bi + 1, :i0 + 64, h:h + 1]),
                         f64(inp["v"][bi:bi + 1, :i0 + 64, h:h + 1]), f64(inp["dout"][bi:bi + 1, sl, h:h + 1]),
                         causal=True)
        a = dq[bi:bi + 1, sl, h:h + 1].float().cpu().double().numpy()
        assert np.abs(a - ref[0]).max() <= TOL[w.dtype] * np.abs(ref[0]).max()
    for bi, h, j0 in ((2, 3, S - 64), (0, 9, S - 256)):
        # keys j0 .. j0+63 are seen by queries j0 .. S-1, which see keys 0 .. S-1
        ref = oracle.bwd(f64(inp["q"][bi:bi + 1, j0:, h:h + 1]), f64(inp["k"][bi:bi + 1, :, h:h + 1]),
                         f64(inp["v"][bi:bi + 1, :, h:h + 1]), f64(inp["dout"][bi:bi + 1, j0:, h:h + 1]),
                         causal=True)
        for got, r in ((dk, ref[1]), (dv, ref[2])):
            a = got[bi:bi + 1, j0:j0 + 64, h:h + 1].float().cpu().double().numpy()
            rr = r[:, j0:j0 + 64]
            assert np.abs(a - rr).max() <= TOL[w.dtype] * np.abs(rr).max()
