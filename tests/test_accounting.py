"""The algorithmic amounts behind every roofline figure (workloads.py):
visible (query, key) pairs, FLOPs and bytes, checked on small shapes against
brute-force enumeration of the mask's definition (CPU only)."""
import pytest

import workloads as W


def _brute_pairs(s_q, N, causal, window):
    """Count pairs (i, j) with query i aligned bottom-right at a = i + N - s_q,
    j <= a when causal, a - left <= j <= a + right for the bounds given."""
    left, right = window
    n = 0
    for i in range(s_q):
        a = i + N - s_q
        for j in range(N):
            if causal and j > a:
                continue
            if right >= 0 and j > a + right:
                continue
            if left >= 0 and j < a - left:
                continue
            n += 1
    return n


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("window", [(-1, -1), (3, -1), (2, 4), (0, 0), (-1, 5)])
@pytest.mark.parametrize("s_q,s_k", [(7, 7), (5, 11), (9, 4), (1, 13)])
def test_dense_pairs_match_enumeration(causal, window, s_q, s_k):
    w = W.Workload(name="t", mode="dense", dtype="fp16", batch=3, h_q=4, h_kv=2, d_qk=64, d_v=32,
                   s_q=s_q, s_k=s_k, causal=causal, window=window)
    assert W.visible_pairs(w) == 3 * 4 * _brute_pairs(s_q, s_k, causal, window)
    assert W.flops(w) == 2.0 * (64 + 32) * W.visible_pairs(w)


def test_backward_flops_per_pair():
    # q.k, dout.v, p*dout (dv), ds*q (dk), ds*k (dq): 2*(3*d_qk + 2*d_v) per pair
    w = W.CONFIGS["mla-backward"]
    pairs = w.batch * w.h_q * w.s_q * (w.s_q + 1) // 2          # causal, s_q = s_k
    assert W.visible_pairs(w) == pairs
    assert W.flops(w) == 2.0 * (3 * 192 + 2 * 128) * pairs


@pytest.mark.parametrize("causal", [True, False])
def test_kvcache_pairs_match_enumeration(causal):
    w = W.Workload(name="t", mode="kvcache", dtype="bf16", batch=3, h_q=4, h_kv=2, d_qk=32, d_v=32,
                   s_q=3, cap=40, seqlens=(0, 30), causal=causal)
    seqlens = [0, 17, 30]
    want = sum(_brute_pairs(3, L + 3, causal, (-1, -1)) for L in seqlens) * 4
    assert W.visible_pairs(w, seqlens) == want


def test_varlen_pairs_match_enumeration():
    w = W.CONFIGS["varlen-prefill"].scaled(batch=3, h_q=2, h_kv=2)
    lens = [5, 1, 9]
    assert W.visible_pairs(w, lens) == 2 * sum(_brute_pairs(n, n, True, (-1, -1)) for n in lens)


def test_kvcache_bytes_by_hand():
    # b2, h_q 4, h_kv 2, d_qk 16, d_v 8, s_new 3, rotary 8, cache lengths 5 and 0
    w = W.Workload(name="t", mode="kvcache", dtype="fp16", batch=2, h_q=4, h_kv=2, d_qk=16, d_v=8,
                   s_q=3, cap=16, seqlens=(0, 5), causal=True, rotary_dim=8)
    cache_read = (5 + 0) * 2 * (16 + 8) * 2
    new_rows = 2 * 3 * 2 * (16 + 8) * 2 * 2          # read and written
    q_out = 2 * 3 * 4 * (16 + 8) * 2
    lse = 2 * 4 * 3 * 4
    cos_sin = 2 * 3 * 8 * 2                          # r/2 cos + r/2 sin per row
    assert W.kvcache_bytes(w, [5, 0]) == cache_read + new_rows + q_out + lse + cos_sin


def test_rotary_bytes_by_hand():
    w = W.CONFIGS["rotary-q"].scaled(batch=2, s_q=3, h_q=5, d_qk=64, rotary_dim=32)
    assert W.rotary_bytes(w) == 2 * (2 * 3 * 5 * 64 * 2) + 2 * 3 * 32 * 2
