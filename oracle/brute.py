"""Pure-Python brute force for tiny shapes (test infrastructure only).

A second statement of the definitions in oracle.c, written differently on
purpose so that the two do not share mistakes:

* RoPE is the RoFormer complex form named in ROCm/flash-attention PR #99
  ("Added Support for Rotary Positional Embeddings", Motivation): each
  rotated pair is read as a complex number a + ib and multiplied by
  e^{i theta}.  Half-split pairs are (j, j + r/2), interleaved pairs
  (2j, 2j + 1).
* Attention enumerates every (query, key) pair, decides visibility with an
  explicit predicate, and normalises with sum(exp(s)) directly (no max
  shift; fine for the tiny magnitudes used here).

Only for inputs of a few hundred elements: nested Python loops.
"""
from __future__ import annotations

import cmath
import math


def rope_row(x, theta, rotary_dim, interleaved):
    """Rotate one row (list of floats) by the per-pair angles theta[j]."""
    y = list(x)
    half = rotary_dim // 2
    for j in range(half):
        ia, ib = (2 * j, 2 * j + 1) if interleaved else (j, j + half)
        z = complex(x[ia], x[ib]) * cmath.exp(1j * theta[j])
        y[ia], y[ib] = z.real, z.imag
    return y


def visible(i, j, s_q, n_keys, causal, window=(-1, -1)):
    """Visibility of key j to query i, stated through the signed distance
    dist = (i + n_keys - s_q) - j from the query's bottom-right aligned key:
    causal keeps dist >= 0; a sliding window ("optimizing-attention-flash",
    window_size=(left, right), -1 = unbounded) keeps dist <= left and
    -dist <= right."""
    if j >= n_keys:
        return False
    dist = (i + n_keys - s_q) - j
    if causal and dist < 0:
        return False
    left, right = window
    if left >= 0 and dist > left:
        return False
    if right >= 0 and -dist > right:
        return False
    return True


def attention(q, keys, vals, s_q, causal, scale, window=(-1, -1)):
    """q: [s_q][d_qk], keys: [N][d_qk], vals: [N][d_v] -> (out [s_q][d_v], lse [s_q])."""
    n = len(keys)
    d_v = len(vals[0]) if vals else 0
    out, lse = [], []
    for i in range(s_q):
        weights = []
        for j in range(n):
            if visible(i, j, s_q, n, causal, window):
                s = scale * sum(a * b for a, b in zip(q[i], keys[j]))
                weights.append((j, math.exp(s)))
        if not weights:
            out.append([0.0] * d_v)
            lse.append(-math.inf)
            continue
        z = sum(w for _, w in weights)
        out.append([sum(w * vals[j][t] for j, w in weights) / z for t in range(d_v)])
        lse.append(math.log(z))
    return out, lse


def kvcache_fwd(q, k_cache, v_cache, k_new, v_new, angles, seqlens, rotary_dim,
                interleaved, causal, scale, round_fn=lambda x: x):
    """Nested-list version of the whole path.

    q [b][s_q][h_q][d_qk], caches [b][cap][h_kv][d], new rows [b][s_new][h_kv][d],
    angles(pos) -> list of rotary_dim/2 angles, round_fn rounds one float.
    Returns out [b][s_q][h_q][d_v], lse [b][h_q][s_q], and updated caches.
    """
    b = len(q)
    s_q = len(q[0])
    h_q = len(q[0][0])
    h_kv = len(k_cache[0][0])
    group = h_q // h_kv
    s_new = len(k_new[0]) if k_new else 0
    kc = [[[list(r) for r in row] for row in kb] for kb in k_cache]
    vc = [[[list(r) for r in row] for row in vb] for vb in v_cache]
    out = [[[None] * h_q for _ in range(s_q)] for _ in range(b)]
    lse = [[[None] * s_q for _ in range(h_q)] for _ in range(b)]
    for bi in range(b):
        L = seqlens[bi]
        for i in range(s_new):
            for h in range(h_kv):
                k = k_new[bi][i][h]
                if rotary_dim:
                    k = rope_row(k, angles(L + i), rotary_dim, interleaved)
                kc[bi][L + i][h] = [round_fn(t) for t in k]
                vc[bi][L + i][h] = list(v_new[bi][i][h])
        n_keys = L + s_new
        for h in range(h_q):
            hk = h // group
            qs = []
            for i in range(s_q):
                qi = q[bi][i][h]
                if rotary_dim:
                    qi = rope_row(qi, angles(L + i), rotary_dim, interleaved)
                qs.append([round_fn(t) for t in qi])
            keys = [kc[bi][j][hk] for j in range(n_keys)]
            vals = [vc[bi][j][hk] for j in range(n_keys)]
            o, l = attention(qs, keys, vals, s_q, causal, scale)
            for i in range(s_q):
                out[bi][i][h] = o[i]
                lse[bi][h][i] = l[i]
    return out, lse, kc, vc
