"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.  Small cases are compared element by element; the
full-size configurations are run in the launch configuration the bench times
and compared on sampled batch entries / heads / query rows that the oracle
can evaluate on its own."""
import numpy as np
import pytest
import torch

import oracle
import rotary_embedding_b200 as fa
import workloads as W
from parity_util import (LSE_TOL, OUT_TOL, check_dense, check_kvcache, run_gpu_dense,
                         run_gpu_kvcache, run_oracle_kvcache, to_dtype_cpu, ulp_distance)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ issue #1402 reproducer
def test_issue_repro_config(cuda_device):
    """fp16 b4 h16 d16, q ~ U[0,1), k_new = v_new = q, zero cache of capacity 2,
    cache_seqlens = 0 (int), non-causal, no rotary, scale 1/4."""
    w = W.ISSUE_REPRO
    inp = W.make_inputs(w)
    gpu = run_gpu_kvcache(w, inp, cuda_device, transpose_views=True)
    check_kvcache(w, inp, gpu, run_oracle_kvcache(w, inp))


def test_issue_repro_seqlen1_is_v(cuda_device):
    """Seqlen 1: the single visible key gives out = v exactly (every backend
    agreed to 1e-5 on the issue)."""
    w = W.ISSUE_REPRO.scaled(s_q=1, cap=1)
    inp = W.make_inputs(w)
    out, lse, kc, vc = run_gpu_kvcache(w, inp, cuda_device)
    assert torch.equal(out, inp["v_new"])


def test_issue_1402_double_rotation(cuda_device):
    """The RoPE reproducer passes already-rotated q/k plus rotary_cos/sin, so
    the kernel rotates them a second time: invisible at seqlen 1, visible at
    seqlen 2.  Rotating once through the kernel matches attention on the
    rotated tensors."""
    for seqlen, should_match in ((1, True), (2, False)):
        w = W.Workload(name="issue-1402-rope", mode="kvcache", dtype="fp16", batch=2, h_q=16, h_kv=16,
                       d_qk=16, d_v=16, s_q=seqlen, cap=seqlen, seqlens_scalar=True, causal=False,
                       rotary_dim=16, dist="rand", kv_is_q=True, zero_cache=True)
        inp = W.make_inputs(w)
        inp["cos"], inp["sin"] = W.rotary_tables(512, 16, 10000.0, torch.float16)
        # rotate once on the host with the oracle (as the page's apply_rotary_emb does)
        pos = np.broadcast_to(np.arange(seqlen)[None, :, None], inp["q"].shape[:3])
        xr = to_dtype_cpu(oracle.round_to(oracle.rope(inp["q"].double().numpy(), pos,
                                                      inp["cos"].double().numpy(),
                                                      inp["sin"].double().numpy(), 16, False),
                                          "fp16"), torch.float16)
        sdpa = oracle.kvcache_fwd(xr.double().numpy(), np.zeros((2, seqlen, 16, 16)),
                                  np.zeros((2, seqlen, 16, 16)), xr.double().numpy(),
                                  inp["q"].double().numpy(), None, None, 0, causal=False,
                                  fmt="fp16")[0]
        once = run_gpu_kvcache(w, inp, cuda_device)[0].double().numpy()
        assert np.abs(once - sdpa).max() <= 1e-3
        twice_inp = dict(inp, q=xr, k_new=xr.clone())
        twice = run_gpu_kvcache(w, twice_inp, cuda_device)[0].double().numpy()
        assert (np.abs(twice - sdpa).max() <= 1e-3) == should_match


# ------------------------------------------------------------------ kvcache sweeps (element-wise)
DECODE_SMALL = W.GQA_DECODE.scaled(name="gqa-decode small", batch=3, cap=700, seqlens=(60, 690))
PREFILL_SMALL = W.CHUNKED_PREFILL.scaled(name="chunked-prefill small", batch=2, h_q=4, h_kv=4,
                                         s_q=70, cap=400, seqlens=(0, 300))
MLA_DECODE_SMALL = W.MLA_DECODE.scaled(name="mla-decode small", batch=2, h_q=4, h_kv=4, cap=1000,
                                       seqlens=(999, 999))


@pytest.mark.parametrize("w", [DECODE_SMALL, PREFILL_SMALL, MLA_DECODE_SMALL], ids=lambda w: w.name)
def test_kvcache_small_configs(w, prefill_tiles, cuda_device):
    inp = W.make_inputs(w)
    check_kvcache(w, inp, run_gpu_kvcache(w, inp, cuda_device), run_oracle_kvcache(w, inp))


def _sweep_cases():
    cases = []
    for d_qk, d_v in ((16, 16), (64, 64), (128, 128), (192, 128)):
        for frac in (0.0, 0.5, 1.0):
            r = int(d_qk * frac) // 2 * 2
            for inter in (False, True):
                if r == 0 and inter:
                    continue
                for s_new in (1, 2, 3, 8):
                    for hq, hkv in ((4, 4), (8, 2), (8, 1)):
                        cases.append((d_qk, d_v, r, inter, s_new, hq, hkv))
    # thin the full product to keep the suite quick, but keep every value of every axis
    rng = np.random.default_rng(0)
    keep = rng.choice(len(cases), size=40, replace=False)
    return [cases[i] for i in sorted(keep)]


@pytest.mark.parametrize("case", _sweep_cases(), ids=lambda c: "d%d-%d_r%d_%s_s%d_g%d-%d" % (
    c[0], c[1], c[2], "int" if c[3] else "half", c[4], c[5], c[6]))
def test_kvcache_sweep(case, cuda_device):
    d_qk, d_v, r, inter, s_new, hq, hkv = case
    for batch, dtype in ((2, "bf16"), (4, "fp16")):
        w = W.Workload(name="sweep", mode="kvcache", dtype=dtype, batch=batch, h_q=hq, h_kv=hkv,
                       d_qk=d_qk, d_v=d_v, s_q=s_new, cap=200, seqlens=(0, 200 - s_new),
                       causal=True, rotary_dim=r, interleaved=inter)
        inp = W.make_inputs(w, seed=d_qk + r + s_new)
        check_kvcache(w, inp, run_gpu_kvcache(w, inp, cuda_device), run_oracle_kvcache(w, inp))


@pytest.mark.parametrize("s_new", [1, 4, 70])
def test_kvcache_int_seqlens_and_noncausal(s_new, cuda_device):
    w = W.Workload(name="int-seqlens", mode="kvcache", dtype="fp16", batch=3, h_q=8, h_kv=2, d_qk=64,
                   d_v=64, s_q=s_new, cap=300, seqlens=(117, 117), seqlens_scalar=True, causal=False,
                   rotary_dim=32, interleaved=False)
    inp = W.make_inputs(w, seed=3)
    check_kvcache(w, inp, run_gpu_kvcache(w, inp, cuda_device), run_oracle_kvcache(w, inp))


def test_kvcache_transposed_views(cuda_device):
    w = DECODE_SMALL
    inp = W.make_inputs(w, seed=5)
    check_kvcache(w, inp, run_gpu_kvcache(w, inp, cuda_device, transpose_views=True),
                  run_oracle_kvcache(w, inp))


def test_kvcache_edges_empty_and_full(cuda_device):
    # L = 0 (only the new rows), L = cap - s_new (cache filled to the last row)
    for lo, hi in ((0, 0), (193, 193)):
        w = W.Workload(name="edges", mode="kvcache", dtype="bf16", batch=2, h_q=4, h_kv=4, d_qk=128,
                       d_v=128, s_q=7, cap=200, seqlens=(lo, hi), causal=True, rotary_dim=128)
        inp = W.make_inputs(w, seed=9)
        check_kvcache(w, inp, run_gpu_kvcache(w, inp, cuda_device), run_oracle_kvcache(w, inp))


def test_kvcache_without_new_rows(cuda_device):
    """k_new = v_new = NULL: attention over the cache rows only."""
    w = W.Workload(name="no-new", mode="kvcache", dtype="fp16", batch=2, h_q=4, h_kv=2, d_qk=64,
                   d_v=64, s_q=2, cap=150, seqlens=(40, 140), causal=True)
    inp = W.make_inputs(w, seed=2)
    dev = {k: v.to(cuda_device) for k, v in inp.items()}
    out, lse = fa.fa_kvcache_fwd(dev["q"], dev["k_cache"], dev["v_cache"],
                                 cache_seqlens=dev["cache_seqlens"], causal=True)
    torch.cuda.synchronize()
    r_out, r_lse, _, _ = oracle.kvcache_fwd(inp["q"].double().numpy(), inp["k_cache"].double().numpy(),
                                            inp["v_cache"].double().numpy(), None, None, None, None,
                                            inp["cache_seqlens"].numpy(), causal=True)
    assert np.abs(out.cpu().double().numpy() - r_out).max() <= OUT_TOL["fp16"]
    assert np.abs(lse.cpu().double().numpy() - r_lse).max() <= LSE_TOL


def test_device_precondition_is_reported(cuda_device):
    """cache_seqlens past the capacity on the device: the batch entry is
    skipped and the status word reports it; no fault."""
    w = W.Workload(name="bad-seqlens", mode="kvcache", dtype="fp16", batch=2, h_q=4, h_kv=4, d_qk=64,
                   d_v=64, s_q=1, cap=64, seqlens=(10, 10), causal=True)
    inp = W.make_inputs(w)
    dev = {k: v.to(cuda_device) for k, v in inp.items()}
    dev["cache_seqlens"][1] = 64   # 64 + 1 > capacity 64
    fa.fa_kvcache_fwd(dev["q"], dev["k_cache"], dev["v_cache"], dev["k_new"], dev["v_new"],
                      cache_seqlens=dev["cache_seqlens"], causal=True)
    assert fa.fa_device_status() == fa.FA_ERR_DEVICE_PRECONDITION
    assert fa.fa_device_status() == 0     # cleared by the read


def test_empty_batch(cuda_device):
    q = torch.zeros(0, 1, 4, 64, dtype=torch.float16, device=cuda_device)
    kc = torch.zeros(0, 16, 4, 64, dtype=torch.float16, device=cuda_device)
    out, lse = fa.fa_kvcache_fwd(q, kc, kc.clone(), cache_seqlens=0)
    assert out.shape == (0, 1, 4, 64)


# ------------------------------------------------------------------ dense (fa_fwd)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dims", [(64, 64, "fp16"), (192, 128, "bf16"), (128, 128, "bf16"), (16, 16, "fp16")])
def test_dense_small(dims, causal, prefill_tiles, cuda_device):
    d_qk, d_v, dt = dims
    for s_q, s_k in ((200, 200), (77, 300), (300, 77)):
        w = W.Workload(name="dense-small", mode="dense", dtype=dt, batch=2, h_q=4, h_kv=2, d_qk=d_qk,
                       d_v=d_v, s_q=s_q, s_k=s_k, causal=causal)
        inp = W.make_inputs(w, seed=s_q)
        ref = oracle.fwd(inp["q"].double().numpy(), inp["k"].double().numpy(), inp["v"].double().numpy(),
                         causal=causal, scale=w.softmax_scale())
        check_dense(w, run_gpu_dense(w, inp, cuda_device), ref)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dims", [(128, 128, "bf16", 6, 2), (192, 128, "bf16", 4, 4), (64, 64, "fp16", 8, 1),
                                  (128, 64, "fp16", 3, 3), (64, 128, "bf16", 2, 2)])
def test_dense_multi_tile(dims, causal, prefill_tiles, cuda_device):
    """Several 128-row query and key tiles with ragged tails; g = 3 takes the
    unpacked path, g = 8 and g = 1 the packed one; the K/V ring wraps."""
    d_qk, d_v, dt, hq, hkv = dims
    w = W.Workload(name="dense-multi", mode="dense", dtype=dt, batch=2, h_q=hq, h_kv=hkv, d_qk=d_qk,
                   d_v=d_v, s_q=1000, s_k=1000, causal=causal)
    inp = W.make_inputs(w, seed=11)
    ref = oracle.fwd(inp["q"].double().numpy(), inp["k"].double().numpy(), inp["v"].double().numpy(),
                     causal=causal, scale=w.softmax_scale())
    check_dense(w, run_gpu_dense(w, inp, cuda_device), ref)


@pytest.mark.parametrize("s_new", [1, 300])
def test_kvcache_garbage_past_sequence(s_new, prefill_tiles, cuda_device):
    """Cache rows at and past N_b hold NaN: they must not reach the result (the
    rows are masked in the scores and zeroed before the PV product)."""
    w = W.Workload(name="nan-tail", mode="kvcache", dtype="bf16", batch=2, h_q=8, h_kv=2, d_qk=128,
                   d_v=128, s_q=s_new, cap=900, seqlens=(100, 500), causal=True, rotary_dim=64)
    inp = W.make_inputs(w, seed=4)
    for b, L in enumerate(inp["cache_seqlens"].tolist()):
        inp["k_cache"][b, L:] = float("nan")
        inp["v_cache"][b, L:] = float("nan")
    gpu = run_gpu_kvcache(w, inp, cuda_device)
    ref_inp = dict(inp)
    ref_inp["k_cache"] = torch.nan_to_num(inp["k_cache"])
    ref_inp["v_cache"] = torch.nan_to_num(inp["v_cache"])
    ref = run_oracle_kvcache(w, ref_inp)
    out, lse, kc, vc = gpu
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    assert np.abs(out.double().numpy() - ref[0]).max() <= OUT_TOL["bf16"]
    assert np.abs(lse.double().numpy() - ref[1]).max() <= LSE_TOL
    # the appended rows replaced the NaN rows at L_b .. L_b + s_new - 1
    for b, L in enumerate(inp["cache_seqlens"].tolist()):
        assert torch.isfinite(vc[b, L:L + s_new]).all()
        assert torch.equal(vc[b, L:L + s_new], inp["v_new"][b])


@pytest.mark.parametrize("lens", [(0, 40, 300, 700, 700, 1500), (1500, 700, 700, 300, 40, 0)],
                         ids=["ascending", "descending"])
def test_kvcache_prefill_unequal_entries(lens, prefill_tiles, cuda_device):
    """Cached prefill over entries of very different lengths, two of them
    equal: one-tile grids take their (entry, query tile) items heaviest first
    by visible keys, ranked on the device, with ties broken by index; every
    row must land where it belongs whatever the rank order."""
    w = W.Workload(name="unequal", mode="kvcache", dtype="fp16", batch=len(lens), h_q=4, h_kv=2, d_qk=128,
                   d_v=128, s_q=200, cap=1800, seqlens=(0, 1), causal=True, rotary_dim=128, interleaved=True)
    inp = W.make_inputs(w, seed=31)
    inp["cache_seqlens"] = torch.tensor(lens, dtype=torch.int32)
    check_kvcache(w, inp, run_gpu_kvcache(w, inp, cuda_device), run_oracle_kvcache(w, inp))


# ------------------------------------------------------------------ full-size configurations
def _slice_kv_inputs(inp, batches, heads=None):
    out = {}
    for k, v in inp.items():
        if k in ("cos", "sin"):
            out[k] = v
        elif k == "cache_seqlens":
            out[k] = v[batches]
        else:
            t = v[batches]
            if heads is not None:
                t = t[:, :, heads]
            out[k] = t
    return out


@pytest.mark.parametrize("name", ["gqa-decode", "mla-decode", "issue-repro"])
def test_full_size_decode_configs(name, cuda_device):
    w = W.CONFIGS[name]
    inp = W.make_inputs(w)
    out, lse, kc, vc = run_gpu_kvcache(w, inp, cuda_device)
    batches = [0, w.batch - 1]
    sub = _slice_kv_inputs(inp, batches)
    ws = w.scaled(batch=len(batches))
    check_kvcache(ws, sub, (out[batches], lse[batches], kc[batches], vc[batches]),
                  run_oracle_kvcache(ws, sub))


def test_full_size_chunked_prefill(cuda_device):
    w = W.CHUNKED_PREFILL
    inp = W.make_inputs(w)
    out, lse, kc, vc = run_gpu_kvcache(w, inp, cuda_device)
    batches, heads = [1, 3], [0, 13]
    sub = _slice_kv_inputs(inp, batches, heads)
    ws = w.scaled(batch=2, h_q=2, h_kv=2)
    g = (out[batches][:, :, heads], lse[batches][:, heads], kc[batches][:, :, heads],
         vc[batches][:, :, heads])
    check_kvcache(ws, sub, g, run_oracle_kvcache(ws, sub))


@pytest.mark.parametrize("name", ["dense-causal", "dense-noncausal", "mla-prefill"])
def test_full_size_dense_configs(name, cuda_device):
    w = W.CONFIGS[name]
    inp = W.make_inputs(w)
    out, lse = run_gpu_dense(w, inp, cuda_device)
    # sampled (batch, head, query-row block) triples against the oracle on the keys they see:
    # the first and last rows, a block across a tile boundary, and one block inside every
    # 128-row query tile (so every tile of every CTA, whichever tiles a CTA pairs, is
    # checked), with the batch entry, head and offset inside the tile varying
    blocks = [(0, 0, 0, 64), (w.batch - 1, w.h_q - 1, w.s_q - 128, w.s_q), (0, 3, 1000, 1100)]
    n_tiles = (w.s_q + 127) // 128
    for t in range(n_tiles):
        r0 = t * 128 + (37 * t) % 112
        blocks.append((t % w.batch, (5 * t + 1) % w.h_q, r0, min(r0 + 16, w.s_q)))
    for b, h, r0, r1 in blocks:
        k1 = r1 if w.causal else w.s_k
        q = inp["q"][b:b + 1, r0:r1, h:h + 1].double().numpy()
        k = inp["k"][b:b + 1, :k1, h:h + 1].double().numpy()
        v = inp["v"][b:b + 1, :k1, h:h + 1].double().numpy()
        r_out, r_lse = oracle.fwd(q, k, v, causal=w.causal, scale=w.softmax_scale())
        err = np.abs(out[b:b + 1, r0:r1, h:h + 1].double().numpy() - r_out).max()
        assert err <= OUT_TOL[w.dtype], (b, h, r0, err)
        lerr = np.abs(lse[b:b + 1, h:h + 1, r0:r1].double().numpy() - r_lse).max()
        assert lerr <= LSE_TOL, (b, h, r0, lerr)
