"""The no-allocation entry point, fa_kvcache_fwd_noalloc.

Some callers cannot allocate device memory when they run attention (a
plug-in whose host application owns every allocation, or a loop that must
never enter the CUDA allocator).  For them the library offers a variant of
fa_kvcache_fwd whose scratch lives in a fixed array inside the library.
These checks call it through the C ABI and compare it with the workspace
entry point and with the float64 oracle, on two calls in a row (the second
call finds the first call's data in the shared scratch).  The file name
sorts last so that a run that stops at the first failure has already run
every other test.
"""
import numpy as np
import pytest
import torch

import rotary_embedding_b200 as fa
import workloads as W
from parity_util import LSE_TOL, OUT_TOL, check_kvcache, run_oracle_kvcache

pytestmark = pytest.mark.gpu

CASES = [
    # decode: split-KV partials live in the scratch
    W.GQA_DECODE.scaled(name="noalloc decode", batch=4, cap=2048, seqlens=(300, 2000)),
    # chunked prefill with RoPE: the rotated copy of q lives in the scratch
    W.CHUNKED_PREFILL.scaled(name="noalloc prefill", batch=2, h_q=4, h_kv=4, s_q=96, cap=600,
                             seqlens=(0, 400)),
]


def _call(fn, w, inp, dev):
    d = {k: v.to(dev) for k, v in inp.items()}
    out, lse = fn(d["q"], d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d.get("cos"), d.get("sin"),
                  cache_seqlens=d["cache_seqlens"], rotary_interleaved=w.interleaved, causal=w.causal)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), d["k_cache"].cpu(), d["v_cache"].cpu()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point(w, cuda_device):
    inp = W.make_inputs(w, seed=21)
    ws = fa.fa_kvcache_plan(inp["q"], inp["k_cache"], inp["v_cache"], inp["k_new"], w.rotary_dim)
    assert 0 < ws["workspace_bytes"] <= fa.FA_NOALLOC_SCRATCH_BYTES
    ref = _call(fa.fa_kvcache_fwd, w, inp, cuda_device)
    oracle_ref = run_oracle_kvcache(w, inp)
    for _ in range(2):
        got = _call(fa.fa_kvcache_fwd_noalloc, w, inp, cuda_device)
        assert fa.fa_device_status() == 0
        check_kvcache(w, inp, got, oracle_ref)
        assert np.abs(got[0].double().numpy() - ref[0].double().numpy()).max() <= OUT_TOL[w.dtype]
        assert np.abs(got[1].double().numpy() - ref[1].double().numpy()).max() <= LSE_TOL
        assert torch.equal(got[2].view(torch.int16), ref[2].view(torch.int16))
        assert torch.equal(got[3].view(torch.int16), ref[3].view(torch.int16))


def test_noalloc_rejects_shapes_beyond_the_scratch(cuda_device):
    # decode over a 32768-row cache: 512 split slots x 4 x 32 rows x 129 floats > 32 MiB
    q = torch.zeros(4, 1, 32, 128, dtype=torch.bfloat16, device=cuda_device)
    kc = torch.zeros(4, 32768, 8, 128, dtype=torch.bfloat16, device=cuda_device)
    need = fa.fa_kvcache_workspace_size(q, kc, kc, None, 0)
    assert need > fa.FA_NOALLOC_SCRATCH_BYTES
    with pytest.raises(fa.FaError) as e:
        fa.fa_kvcache_fwd_noalloc(q, kc, kc, cache_seqlens=100, causal=True)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    assert "scratch" in str(e.value)
