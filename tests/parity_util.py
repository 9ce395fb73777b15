"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the float64 oracle on the same seeded inputs, and compare with the
tolerances the attention-with-KV-cache contract states:

* v cache rows: bit-exact;
* rotated k cache rows: within 1 ulp of the element type;
* out: max |err| <= 2e-3 (fp16) or 1.6e-2 (bf16);
* lse: |err| <= 1e-3 (fp32).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import rotary_embedding_b200 as fa
import workloads as W

OUT_TOL = {"fp16": 2e-3, "bf16": 1.6e-2}
LSE_TOL = 1e-3


def ordinal16(t: torch.Tensor) -> np.ndarray:
    """Monotonic integer order of 16-bit float bit patterns (sign-magnitude)."""
    bits = t.contiguous().view(torch.int16).numpy().astype(np.int32)
    return np.where(bits >= 0, bits, -(bits & 0x7FFF))


def ulp_distance(a: torch.Tensor, b: torch.Tensor) -> np.ndarray:
    return np.abs(ordinal16(a) - ordinal16(b))


def to_dtype_cpu(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def run_gpu_kvcache(w: W.Workload, inp: dict, device, seqlens_as_tensor=None, causal=None,
                    transpose_views=False):
    """fa_kvcache_fwd on copies of the inputs; returns CPU (out, lse, k_cache, v_cache)."""
    dev = {k: v.to(device) for k, v in inp.items()}
    q, kc, vc, kn, vn = dev["q"], dev["k_cache"], dev["v_cache"], dev["k_new"], dev["v_new"]
    if transpose_views:
        # issue #1402 passes [b, h, s, d] tensors as transposed [b, s, h, d] views
        q = q.transpose(1, 2).contiguous().transpose(1, 2)
        kn = kn.transpose(1, 2).contiguous().transpose(1, 2)
        vn = vn.transpose(1, 2).contiguous().transpose(1, 2)
        kc = kc.transpose(1, 2).contiguous().transpose(1, 2)
        vc = vc.transpose(1, 2).contiguous().transpose(1, 2)
    as_tensor = (not w.seqlens_scalar) if seqlens_as_tensor is None else seqlens_as_tensor
    if as_tensor:
        seq = dev["cache_seqlens"]
    else:
        vals = inp["cache_seqlens"].tolist()
        assert len(set(vals)) == 1, "the int form needs one offset for every batch entry"
        seq = int(vals[0])
    out, lse = fa.fa_kvcache_fwd(
        q, kc, vc, kn, vn, dev.get("cos"), dev.get("sin"), cache_seqlens=seq,
        rotary_dim=w.rotary_dim if w.rotary_dim else None,
        rotary_interleaved=w.interleaved, causal=w.causal if causal is None else causal,
        softmax_scale=w.scale if w.scale > 0 else None)
    torch.cuda.synchronize(device)
    status = fa.fa_device_status()
    assert status == 0, f"device status {status}"
    return out.cpu(), lse.cpu(), kc.cpu(), vc.cpu()


def run_oracle_kvcache(w: W.Workload, inp: dict, causal=None):
    return oracle.kvcache_fwd(
        inp["q"].double().numpy(), inp["k_cache"].double().numpy(), inp["v_cache"].double().numpy(),
        inp["k_new"].double().numpy(), inp["v_new"].double().numpy(),
        inp["cos"].double().numpy() if "cos" in inp else None,
        inp["sin"].double().numpy() if "sin" in inp else None,
        inp["cache_seqlens"].numpy(), rotary_dim=w.rotary_dim, interleaved=w.interleaved,
        causal=w.causal if causal is None else causal, scale=w.softmax_scale(), fmt=w.dtype)


def check_kvcache(w: W.Workload, inp: dict, gpu, ref):
    """Element-by-element comparison of the whole result."""
    out, lse, kc, vc = gpu
    r_out, r_lse, r_kc, r_vc = ref
    dt = w.torch_dtype
    # v cache: bit-exact everywhere (appended rows = v_new, others untouched)
    assert torch.equal(vc.view(torch.int16), to_dtype_cpu(r_vc, dt).view(torch.int16)), "v cache differs"
    # k cache: appended rows within 1 ulp; other rows bit-identical
    dist = ulp_distance(kc, to_dtype_cpu(r_kc, dt))
    assert dist.max() <= 1, f"k cache differs by {dist.max()} ulp"
    untouched = np.ones(kc.shape[:2], bool)
    for b, L in enumerate(inp["cache_seqlens"].tolist()):
        untouched[b, L:L + inp["k_new"].shape[1]] = False
    assert dist[untouched].max(initial=0) == 0, "k cache rows outside the append changed"
    err = np.abs(out.double().numpy() - r_out)
    assert err.max() <= OUT_TOL[w.dtype], f"out max err {err.max():.3e}"
    fin = np.isfinite(r_lse)
    assert np.array_equal(np.isfinite(lse.numpy()), fin)
    lerr = np.abs(lse.double().numpy()[fin] - r_lse[fin])
    assert lerr.max(initial=0) <= LSE_TOL, f"lse max err {lerr.max():.3e}"
    return float(err.max()), float(lerr.max(initial=0))


def run_gpu_dense(w: W.Workload, inp: dict, device, causal=None):
    q, k, v = (inp[n].to(device) for n in ("q", "k", "v"))
    out, lse = fa.fa_fwd(q, k, v, causal=w.causal if causal is None else causal,
                         softmax_scale=w.scale if w.scale > 0 else None)
    torch.cuda.synchronize(device)
    assert fa.fa_device_status() == 0
    return out.cpu(), lse.cpu()


def check_dense(w: W.Workload, gpu, ref):
    out, lse = gpu
    r_out, r_lse = ref
    err = np.abs(out.double().numpy() - r_out)
    assert err.max() <= OUT_TOL[w.dtype], f"out max err {err.max():.3e}"
    fin = np.isfinite(r_lse)
    assert np.array_equal(np.isfinite(lse.numpy()), fin)
    lerr = np.abs(lse.double().numpy()[fin] - r_lse[fin])
    assert lerr.max(initial=0) <= LSE_TOL, f"lse max err {lerr.max():.3e}"
    return float(err.max()), float(lerr.max(initial=0))
