"""Pins for the float64 oracle: facts fixed by the pages or by mathematics.

Each ``pin_*`` function takes a loaded oracle library and raises
AssertionError if the oracle disagrees with the fact.  test_oracle.py runs
them against the real oracle (all must hold) and against builds with a
planted mistake (each mistake must break at least one pin).

Nothing here restates the oracle's formulas: the expected values come from
closed forms (rotation by a right angle, rotation by zero), invariants
(norms, relative position, softmax rows summing to one), special cases that
reduce to a library routine (scipy softmax / logsumexp, numpy float16
rounding), the pure-Python brute force in oracle/brute.py, and the printed
outcomes of the flash-attention issue #1402 reproducers.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
from scipy.special import logsumexp, softmax

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _tables(rows, r, base=10000.0):
    j = np.arange(r // 2, dtype=np.float64)
    ang = np.outer(np.arange(rows, dtype=np.float64), base ** (-2.0 * j / r))
    return np.cos(ang), np.sin(ang), ang


def _const_tables(rows, r, angle):
    shape = (rows, r // 2)
    return np.full(shape, math.cos(angle)), np.full(shape, math.sin(angle))


# ---------------------------------------------------------------- rounding
def pin_round_fp16_matches_numpy(lib):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-8, 5, 4000),
        np.array([65504.0, 65519.99, 65520.0, 1e-8, 2.0 ** -24, 3 * 2.0 ** -25,
                  1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, -0.0, 5.9604644775390625e-08]),
    ])
    got = oracle.round_to(x, "fp16")
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).astype(np.float64)
    assert np.array_equal(got, want), "fp16 rounding differs from numpy's correctly rounded cast"


def pin_round_bf16_matches_torch(lib):
    """bf16 rounding equals torch's round-to-nearest-even cast from float32 on
    4000 random float32 bit patterns (normals of every exponent, subnormals
    down to 2^-149, values past the largest finite bf16) and on the edges:
    the smallest bf16 subnormal 2^-133 and the ties around it, the largest
    finite bf16 (2 - 2^-7) 2^127, and the midpoint above it, which rounds to
    infinity.  Every value is a float32, so the float64 the oracle takes and
    the float32 torch takes are the same number."""
    import torch
    rng = np.random.default_rng(7)
    x32 = rng.integers(0, 2 ** 32, 4000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    x32 = x32[np.isfinite(x32)]
    top = (2.0 - 2.0 ** -7) * 2.0 ** 127
    edges = np.array([2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -134, 1.5 * 2.0 ** -133, 2.0 ** -126,
                      2.0 ** -126 - 2.0 ** -134, 2.0 ** -127 + 2.0 ** -134, top, -top,
                      (2.0 - 2.0 ** -8) * 2.0 ** 127, (2.0 - 2.0 ** -9) * 2.0 ** 127,
                      -(2.0 - 2.0 ** -8) * 2.0 ** 127, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    x = np.concatenate([x32, edges]).astype(np.float64)
    got = oracle.round_to(x, "bf16")
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"bf16 rounding differs from torch at {x[bad[:5]]}: {got[bad[:5]]} vs {want[bad[:5]]}"
    assert np.isinf(oracle.round_to(np.array([(2.0 - 2.0 ** -8) * 2.0 ** 127]), "bf16")[0])


def pin_round_bf16_ties_to_even(lib):
    # exact bf16 neighbours of 1.0 are 1.0 and 1 + 2^-7; the midpoint ties to the even one
    cases = {1.0 + 2.0 ** -8: 1.0, 1.0 + 3 * 2.0 ** -8: 1.0 + 2.0 ** -6,
             1.0 + 2.0 ** -8 + 2.0 ** -30: 1.0 + 2.0 ** -7, -3.0: -3.0,
             2.0 ** -130: 2.0 ** -130, 3.3895313892515355e38: 3.3895313892515355e38}
    for x, want in cases.items():
        assert oracle.round_to(np.array([x]), "bf16")[0] == want, x


# ---------------------------------------------------------------- RoPE
def pin_rope_right_angle_is_rotate_half(lib):
    """Angle pi/2 (cos 0, sin 1): the RoPE reproducer of issue #1402 gives
    q*cos + rotate_half(q)*sin = rotate_half(q) = cat(-x2, x1) (half-split);
    interleaved pairs (a, b) -> (-b, a)."""
    x = np.arange(1.0, 9.0)[None, :]
    c, s = _const_tables(1, 8, math.pi / 2)
    c[:] = 0.0
    s[:] = 1.0
    y = oracle.rope(x, [0], c, s, 8, False, lib=lib)
    assert np.array_equal(y[0], [-5.0, -6.0, -7.0, -8.0, 1.0, 2.0, 3.0, 4.0]), y
    y = oracle.rope(x, [0], c, s, 8, True, lib=lib)
    assert np.array_equal(y[0], [-2.0, 1.0, -4.0, 3.0, -6.0, 5.0, -8.0, 7.0]), y


def pin_rope_partial_right_angle(lib):
    """rotary_dim 4 of head_dim 8 (rotary_fraction 0.5 of PR #99): half-split
    pairs (0,2),(1,3); dims 4..7 unchanged."""
    x = np.arange(1.0, 9.0)[None, :]
    c = np.zeros((1, 2))
    s = np.ones((1, 2))
    y = oracle.rope(x, [0], c, s, 4, False, lib=lib)
    assert np.array_equal(y[0], [-3.0, -4.0, 1.0, 2.0, 5.0, 6.0, 7.0, 8.0]), y
    y = oracle.rope(x, [0], c, s, 4, True, lib=lib)
    assert np.array_equal(y[0], [-2.0, 1.0, -4.0, 3.0, 5.0, 6.0, 7.0, 8.0]), y


def pin_rope_position_zero_and_r_zero_identity(lib):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 16))
    c, s, _ = _tables(8, 16)
    for inter in (False, True):
        y = oracle.rope(x, [0] * 5, c, s, 16, inter, lib=lib)
        assert np.array_equal(y, x)
    y = oracle.rope(x, [3] * 5, c, s, 0, False, lib=lib)
    assert np.array_equal(y, x)


def pin_rope_norm_and_relative_position(lib):
    """Rotation preserves norms; (R_m q).(R_n k) depends only on m - n."""
    rng = np.random.default_rng(3)
    d = r = 32
    c, s, _ = _tables(64, r)
    q = rng.standard_normal((1, d))
    k = rng.standard_normal((1, d))
    for inter in (False, True):
        for m in (0, 5, 17, 40):
            y = oracle.rope(q, [m], c, s, r, inter, lib=lib)
            assert abs(np.linalg.norm(y) - np.linalg.norm(q)) < 1e-12
        dots = []
        for m, n in ((7, 3), (11, 7), (50, 46), (4, 0)):
            dots.append(float(oracle.rope(q, [m], c, s, r, inter, lib=lib)[0]
                              @ oracle.rope(k, [n], c, s, r, inter, lib=lib)[0]))
        assert max(dots) - min(dots) < 1e-10, dots
        # and it does change with the distance
        far = float(oracle.rope(q, [20], c, s, r, inter, lib=lib)[0]
                    @ oracle.rope(k, [0], c, s, r, inter, lib=lib)[0])
        assert abs(far - dots[0]) > 1e-3


def pin_rope_angle_sign(lib):
    """Counter-clockwise rotation: e_a at angle t maps to (cos t, sin t) on the
    (a, b) plane, matching the page's q*cos + rotate_half(q)*sin."""
    t = 0.3
    c = np.full((1, 1), math.cos(t))
    s = np.full((1, 1), math.sin(t))
    y = oracle.rope(np.array([[1.0, 0.0]]), [0], c, s, 2, False, lib=lib)
    assert np.allclose(y[0], [math.cos(t), math.sin(t)], atol=1e-15)
    y = oracle.rope(np.array([[0.0, 1.0]]), [0], c, s, 2, True, lib=lib)
    assert np.allclose(y[0], [-math.sin(t), math.cos(t)], atol=1e-15)


def pin_rope_pairings_are_permutations(lib):
    """Half-split and interleaved differ only by the pairing: permuting dims
    (j, j+r/2) <-> (2j, 2j+1) maps one onto the other."""
    rng = np.random.default_rng(4)
    d, r = 24, 16
    c, s, _ = _tables(20, r)
    x = rng.standard_normal((6, d))
    pos = [0, 1, 5, 9, 13, 19]
    perm = np.arange(d)
    for j in range(r // 2):
        perm[2 * j] = j
        perm[2 * j + 1] = j + r // 2
    y_half = oracle.rope(x, pos, c, s, r, False, lib=lib)
    y_int = oracle.rope(x[:, perm], pos, c, s, r, True, lib=lib)
    assert np.allclose(y_int, y_half[:, perm], atol=0, rtol=0)


def pin_rope_matches_complex_form(lib):
    rng = np.random.default_rng(5)
    d, r = 12, 8
    c, s, ang = _tables(30, r)
    x = rng.standard_normal((4, d))
    pos = [0, 3, 17, 29]
    for inter in (False, True):
        y = oracle.rope(x, pos, c, s, r, inter, lib=lib)
        for i, p in enumerate(pos):
            want = brute.rope_row(list(x[i]), list(ang[p]), r, inter)
            assert np.allclose(y[i], want, atol=1e-13), (inter, i)


# ---------------------------------------------------------------- attention
def pin_single_key_gives_v(lib):
    """One key: softmax weight 1, out = v exactly, lse = scale*q.k (issue
    #1402: every backend agrees at seqlen 1)."""
    rng = np.random.default_rng(6)
    q = rng.standard_normal((2, 1, 3, 8))
    k = rng.standard_normal((2, 1, 3, 8))
    v = rng.standard_normal((2, 1, 3, 5))
    for causal in (False, True):
        out, lse = oracle.fwd(q, k, v, causal=causal, scale=0.7, lib=lib)
        assert np.array_equal(out, v)
        want = 0.7 * np.einsum("bshd,bshd->bhs", q, k)
        assert np.allclose(lse, want, atol=1e-14)


def pin_equal_keys_average_values(lib):
    rng = np.random.default_rng(7)
    n = 6
    q = rng.standard_normal((1, 1, 1, 4))
    k = np.repeat(rng.standard_normal((1, 1, 1, 4)), n, axis=1)
    v = rng.standard_normal((1, n, 1, 3))
    out, lse = oracle.fwd(q, k, v, causal=False, scale=1.0, lib=lib)
    assert np.allclose(out[0, 0, 0], v[0, :, 0].mean(axis=0), atol=1e-14)
    assert abs(lse[0, 0, 0] - (float(q[0, 0, 0] @ k[0, 0, 0]) + math.log(n))) < 1e-13


def pin_probabilities_rows_and_bottom_right_mask(lib):
    """With V = identity the output rows are the attention weights: each row
    is a probability vector, zero exactly on the masked keys.  Causal is
    aligned bottom-right: query i of s_q sees keys j <= i + N - s_q."""
    rng = np.random.default_rng(8)
    for s_q, n in ((3, 7), (7, 7), (1, 5), (4, 4)):
        q = rng.standard_normal((1, s_q, 1, 4))
        k = rng.standard_normal((1, n, 1, 4))
        v = np.eye(n)[None, :, None, :]
        out, _ = oracle.fwd(q, k, v, causal=True, scale=0.5, lib=lib)
        p = out[0, :, 0, :]
        assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14)
        for i in range(s_q):
            for j in range(n):
                if j <= i + n - s_q:
                    assert p[i, j] > 0.0
                else:
                    assert p[i, j] == 0.0


def pin_matches_textbook_softmax(lib):
    """scipy softmax(scale q k^T + mask) v and logsumexp, causal and not, with
    s_q == N (lower-triangular mask) and s_q < N (bottom-right)."""
    rng = np.random.default_rng(9)
    for s_q, n, causal in ((5, 5, True), (5, 5, False), (3, 9, True), (2, 6, False)):
        q = rng.standard_normal((1, s_q, 1, 6))
        k = rng.standard_normal((1, n, 1, 6))
        v = rng.standard_normal((1, n, 1, 4))
        out, lse = oracle.fwd(q, k, v, causal=causal, scale=0.3, lib=lib)
        sc = 0.3 * q[0, :, 0] @ k[0, :, 0].T
        if causal:
            sc = np.where(np.triu(np.ones((s_q, n), bool), k=n - s_q + 1), -np.inf, sc)
        assert np.allclose(out[0, :, 0], softmax(sc, axis=1) @ v[0, :, 0], atol=1e-13)
        assert np.allclose(lse[0, 0], logsumexp(sc, axis=1), atol=1e-13)


def pin_default_scale(lib):
    """softmax_scale=None means 1/sqrt(d) ("optimizing-attention-flash", Workflow 2)."""
    rng = np.random.default_rng(10)
    q = rng.standard_normal((1, 2, 1, 16))
    k = rng.standard_normal((1, 3, 1, 16))
    v = rng.standard_normal((1, 3, 1, 2))
    a = oracle.fwd(q, k, v, scale=None, lib=lib)
    b = oracle.fwd(q, k, v, scale=0.25, lib=lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def pin_gqa_equals_repeated_heads(lib):
    """Fewer KV heads ("optimizing-attention-flash", Workflow 2 Step 3): query
    head h uses kv head h // (h_q/h_kv); equal to MHA with each kv head
    repeated for its group."""
    rng = np.random.default_rng(11)
    h_q, h_kv = 6, 2
    q = rng.standard_normal((2, 3, h_q, 4))
    k = rng.standard_normal((2, 5, h_kv, 4))
    v = rng.standard_normal((2, 5, h_kv, 3))
    a = oracle.fwd(q, k, v, causal=True, lib=lib)
    b = oracle.fwd(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), causal=True, lib=lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # through the cache path as well
    kc = rng.standard_normal((2, 8, h_kv, 4))
    vc = rng.standard_normal((2, 8, h_kv, 3))
    a = oracle.kvcache_fwd(q, kc, vc, k[:, :3], v[:, :3], None, None, [2, 4], causal=True, lib=lib)
    b = oracle.kvcache_fwd(q, np.repeat(kc, 3, axis=2), np.repeat(vc, 3, axis=2),
                           np.repeat(k[:, :3], 3, axis=2), np.repeat(v[:, :3], 3, axis=2),
                           None, None, [2, 4], causal=True, lib=lib)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------- whole path
def _tiny_case(rng, b, s_new, h_q, h_kv, d_qk, d_v, cap, seqlens, r):
    q = rng.standard_normal((b, s_new, h_q, d_qk))
    kc = rng.standard_normal((b, cap, h_kv, d_qk))
    vc = rng.standard_normal((b, cap, h_kv, d_v))
    kn = rng.standard_normal((b, s_new, h_kv, d_qk))
    vn = rng.standard_normal((b, s_new, h_kv, d_v))
    return q, kc, vc, kn, vn


def pin_brute_force_whole_path(lib):
    """The pure-Python enumeration agrees on tiny shapes: RoPE (both pairings,
    partial), append at per-batch offsets, GQA, bottom-right causal, fp16
    rounding of the rotated rows (numpy's cast as the rounding routine)."""
    rng = np.random.default_rng(12)
    for (b, s_new, h_q, h_kv, d, dv, cap, seql, r, inter, causal) in (
            (2, 3, 4, 2, 8, 6, 8, [1, 4], 8, False, True),
            (2, 2, 2, 1, 8, 4, 6, [0, 3], 4, True, True),
            (1, 1, 3, 3, 6, 6, 5, [4], 6, False, False),
            (2, 4, 2, 2, 4, 4, 9, [5, 0], 0, False, True)):
        q, kc, vc, kn, vn = _tiny_case(rng, b, s_new, h_q, h_kv, d, dv, cap, seql, r)
        c, s, ang = _tables(cap, max(r, 2))
        out, lse, kc2, vc2 = oracle.kvcache_fwd(q, kc, vc, kn, vn, c, s, seql, rotary_dim=r,
                                                interleaved=inter, causal=causal, scale=0.4,
                                                fmt="fp16", lib=lib)
        bo, bl, bkc, bvc = brute.kvcache_fwd(
            q.tolist(), kc.tolist(), vc.tolist(), kn.tolist(), vn.tolist(),
            lambda p: list(ang[p]), seql, r, inter, causal, 0.4,
            round_fn=lambda t: float(np.float16(t)))
        assert np.allclose(out, np.array(bo), atol=1e-12)
        assert np.allclose(lse, np.array(bl), atol=1e-12)
        assert np.array_equal(kc2, np.array(bkc)) and np.array_equal(vc2, np.array(bvc))


def pin_append_rows_and_canaries(lib):
    """Cache append: rows L_b .. L_b+s_new-1 get rope(k_new) rounded and the raw
    v_new bits; every other row is untouched (flash_attn_with_kvcache usage of
    issue #1402, cache_seqlens offsets)."""
    rng = np.random.default_rng(13)
    b, s_new, h, d, cap, r = 3, 2, 2, 8, 10, 8
    q, kc, vc, kn, vn = _tiny_case(rng, b, s_new, h, h, d, d, cap, None, r)
    kc = oracle.round_to(kc, "bf16")
    vc = oracle.round_to(vc, "bf16")
    c, s, _ = _tables(cap, r)
    seql = [0, 3, 8]
    _, _, kc2, vc2 = oracle.kvcache_fwd(q, kc, vc, kn, vn, c, s, seql, rotary_dim=r,
                                        causal=True, fmt="bf16", lib=lib)
    for bi, L in enumerate(seql):
        for row in range(cap):
            if L <= row < L + s_new:
                i = row - L
                want_k = oracle.round_to(oracle.rope(kn[bi, i], [row] * h, c, s, r, False,
                                                     lib=lib), "bf16")
                assert np.array_equal(kc2[bi, row], want_k)
                assert np.array_equal(vc2[bi, row], vn[bi, i])
            else:
                assert np.array_equal(kc2[bi, row], kc[bi, row])
                assert np.array_equal(vc2[bi, row], vc[bi, row])


def pin_query_rotation_positions(lib):
    """The rotated query used by attention is q rotated at row L_b + i: with a
    single cached key at position p and its own rotation built in, the score
    of query i equals (R_{L+i} q_i).(R_p k)."""
    rng = np.random.default_rng(15)
    d = 8
    c, s, _ = _tables(32, d)
    L, s_new = 5, 3
    q = rng.standard_normal((1, s_new, 1, d))
    kc = np.zeros((1, 12, 1, d))
    vc = np.zeros((1, 12, 1, 1))
    kn = rng.standard_normal((1, s_new, 1, d))
    vn = np.zeros((1, s_new, 1, 1))
    # v = 1 on key 0 only, so out = weight of key 0
    vc[0, 0, 0, 0] = 1.0
    kc[0, 0, 0] = rng.standard_normal(d)
    out, lse, kc2, _ = oracle.kvcache_fwd(q, kc, vc, kn, vn, c, s, [L], rotary_dim=d,
                                          causal=True, scale=1.0, lib=lib)
    for i in range(s_new):
        qi = oracle.rope(q[0, i, 0], [L + i], c, s, d, False, lib=lib)
        scores = np.array([qi @ kc2[0, j, 0] for j in range(L + i + 1)])
        assert abs(out[0, i, 0, 0] - softmax(scores)[0]) < 1e-12
        assert abs(lse[0, 0, i] - logsumexp(scores)) < 1e-12


def pin_issue_1402_no_rope(lib):
    """The no-RoPE reproducer of issue #1402: q = k = v ~ U[0,1) fp16, zero
    cache, cache_seqlens=0, non-causal.  Seqlen 1: the output is v exactly
    (all backends agree to 1e-5).  Seqlen 2: the textbook softmax."""
    rng = np.random.default_rng(16)
    for seqlen in (1, 2):
        x = oracle.round_to(rng.random((4, seqlen, 16, 16)), "fp16")
        zero = np.zeros((4, seqlen, 16, 16))
        out, lse, _, _ = oracle.kvcache_fwd(x, zero, zero, x, x, None, None, 0,
                                            causal=False, fmt="fp16", lib=lib)
        if seqlen == 1:
            assert np.array_equal(out, x)
        for bi in range(4):
            for h in range(16):
                qh = x[bi, :, h]
                sc = 0.25 * qh @ qh.T
                assert np.allclose(out[bi, :, h], softmax(sc, axis=1) @ qh, atol=1e-13)


def pin_issue_1402_double_rotation(lib):
    """The RoPE reproducer of issue #1402 rotates q/k itself and then passes the
    rotated tensors with rotary_cos/sin again.  At seqlen 1 (position 0,
    cos=1, sin=0) the double rotation is invisible; at seqlen 2 it is not
    (FLASHCACHE differs from SDPA at atol 1e-3).  Rotating once matches the
    unrotated-input path with kernel RoPE."""
    with open(os.path.join(GOLDEN, "issue1402_rope_outcomes.json")) as f:
        printed = json.load(f)
    rng = np.random.default_rng(17)
    c, s, _ = _tables(512, 16)
    c16, s16 = oracle.round_to(c, "fp16"), oracle.round_to(s, "fp16")
    for seqlen in (1, 2):
        x = oracle.round_to(rng.random((2, seqlen, 16, 16)), "fp16")
        zero = np.zeros((2, seqlen, 16, 16))
        pos = np.arange(seqlen)[None, :, None]
        xr = oracle.round_to(oracle.rope(x, np.broadcast_to(pos, x.shape[:3]), c16, s16, 16,
                                         False, lib=lib), "fp16")
        # SDPA on the rotated tensors, value = unrotated query (the script's value = query)
        sdpa, _, _, _ = oracle.kvcache_fwd(xr, zero, zero, xr, x, None, None, 0,
                                           causal=False, fmt="fp16", lib=lib)
        once, _, _, _ = oracle.kvcache_fwd(x, zero, zero, x, x, c16, s16, 0, rotary_dim=16,
                                           causal=False, fmt="fp16", lib=lib)
        twice, _, _, _ = oracle.kvcache_fwd(xr, zero, zero, xr, x, c16, s16, 0, rotary_dim=16,
                                            causal=False, fmt="fp16", lib=lib)
        agree_twice = bool(np.allclose(sdpa, twice, atol=1e-3, rtol=0))
        assert agree_twice == printed[str(seqlen)]["FLASHCACHE_matches_SDPA_atol_1e-3"]
        assert np.allclose(sdpa, once, atol=1e-3, rtol=0)


def pin_rotary_conjugate_inverts(lib):
    """CONJUGATE ([P2] standalone rotary) undoes the rotation: in float64 the
    conjugate of the rotated rows gives the rows back, for both pairings and
    a partial rotary_dim."""
    rng = np.random.default_rng(31)
    c, s, _ = _tables(40, 12)
    x = rng.standard_normal((3, 5, 2, 16))
    for inter in (False, True):
        y = oracle.rotary(x, c, s, [0, 7, 20], 12, inter, False, lib=lib)
        assert not np.allclose(y, x)
        back = oracle.rotary(y, c, s, [0, 7, 20], 12, inter, True, lib=lib)
        assert np.allclose(back, x, atol=1e-13, rtol=0)
        back = oracle.rotary(oracle.rotary(x, c, s, [0, 7, 20], 12, inter, True, lib=lib), c, s,
                             [0, 7, 20], 12, inter, False, lib=lib)
        assert np.allclose(back, x, atol=1e-13, rtol=0)


def pin_rotary_conjugate_is_adjoint(lib):
    """The conjugate rotation is the transpose of the rotation:
    <R x, y> = <x, R* y> for every row."""
    rng = np.random.default_rng(32)
    c, s, _ = _tables(30, 16)
    x = rng.standard_normal((2, 6, 3, 16))
    y = rng.standard_normal((2, 6, 3, 16))
    for inter in (False, True):
        rx = oracle.rotary(x, c, s, 5, 16, inter, False, lib=lib)
        cy = oracle.rotary(y, c, s, 5, 16, inter, True, lib=lib)
        assert np.allclose((rx * y).sum(-1), (x * cy).sum(-1), atol=1e-12, rtol=0)


def pin_rotary_conjugate_composes_as_negative_angle(lib):
    """Rotations compose by adding angles: the conjugate rotation at position p
    followed by the rotation at position p + q equals the rotation at q
    (tables built in float64 from base^(-2j/r) angles)."""
    rng = np.random.default_rng(33)
    c, s, _ = _tables(64, 8)
    x = rng.standard_normal((1, 1, 1, 8))
    for inter in (False, True):
        for p, q in ((3, 5), (17, 0), (30, 21)):
            a = oracle.rotary(oracle.rotary(x, c, s, p, 8, inter, True, lib=lib), c, s, p + q, 8, inter,
                              False, lib=lib)
            b = oracle.rotary(x, c, s, q, 8, inter, False, lib=lib)
            assert np.allclose(a, b, atol=1e-12, rtol=0)


def pin_rotary_equals_attention_rope_and_rounds(lib):
    """Without CONJUGATE the standalone rotary is the attention path's RoPE of
    every head at position offset + i, and the fp16/bf16 results are the
    float64 ones rounded to nearest even."""
    rng = np.random.default_rng(34)
    c, s, _ = _tables(50, 16)
    x = oracle.round_to(rng.standard_normal((2, 4, 3, 16)), "bf16")
    offs = np.array([2, 9])
    y = oracle.rotary(x, c, s, offs, 16, False, False, lib=lib)
    pos = (offs[:, None] + np.arange(4)[None, :])[:, :, None].repeat(3, axis=2)
    assert np.array_equal(y, oracle.rope(x, pos, c, s, 16, False, lib=lib))
    for fmt in ("fp16", "bf16"):
        assert np.array_equal(oracle.rotary(x, c, s, offs, 16, False, False, fmt=fmt, lib=lib),
                              oracle.round_to(y, fmt))


def pin_rotary_varlen_positions(lib):
    """Packed rows ([P2] IS_VARLEN): entry k holds rows cu[k] .. cu[k+1] - 1 and
    row t sits at offset_k + t - cu[k], so the packed result equals the
    batched result of each entry; an int offset equals the same value per
    entry."""
    rng = np.random.default_rng(35)
    c, s, _ = _tables(40, 8)
    lens = [3, 1, 5]
    cu = np.concatenate([[0], np.cumsum(lens)])
    offs = np.array([4, 0, 11])
    xp = rng.standard_normal((cu[-1], 2, 8))
    yp = oracle.rotary(xp, c, s, offs, 8, True, True, cu_seqlens=cu, lib=lib)
    for k, n in enumerate(lens):
        yb = oracle.rotary(xp[None, cu[k]:cu[k + 1]], c, s, int(offs[k]), 8, True, True, lib=lib)
        assert np.array_equal(yp[cu[k]:cu[k + 1]], yb[0])
    assert np.array_equal(oracle.rotary(xp, c, s, 6, 8, False, False, cu_seqlens=cu, lib=lib),
                          oracle.rotary(xp, c, s, [6, 6, 6], 8, False, False, cu_seqlens=cu, lib=lib))


def pin_window_covering_everything_is_no_window(lib):
    """A window wider than the sequence ("optimizing-attention-flash",
    window_size=(left, right)) changes nothing: equal to (-1, -1)."""
    rng = np.random.default_rng(41)
    q, k, v = (rng.standard_normal((2, 6, 2, 8)) for _ in range(3))
    for causal in (False, True):
        a = oracle.fwd(q, k, v, causal=causal, scale=0.5, lib=lib)
        b = oracle.fwd(q, k, v, causal=causal, scale=0.5, lib=lib, window=(6, 6))
        assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)


def pin_window_zero_sees_only_the_aligned_key(lib):
    """window (0, 0): query i sees only key a = i + s_k - s_q, so out = v[a]
    exactly and lse = scale q.k[a] (the single-key case)."""
    rng = np.random.default_rng(42)
    q = rng.standard_normal((1, 3, 2, 8))
    k = rng.standard_normal((1, 7, 2, 8))
    v = rng.standard_normal((1, 7, 2, 5))
    out, lse = oracle.fwd(q, k, v, causal=False, scale=0.3, lib=lib, window=(0, 0))
    for i in range(3):
        a = i + 7 - 3
        assert np.array_equal(out[0, i], v[0, a])
        for h in range(2):
            assert np.isclose(lse[0, h, i], 0.3 * q[0, i, h] @ k[0, a, h], atol=1e-14)


def pin_window_left_matches_slice_softmax(lib):
    """Causal with a left window w: query i attends to keys a - w .. a, the
    textbook softmax over that slice (scipy), and keys outside the window do
    not matter."""
    from scipy.special import softmax, logsumexp
    rng = np.random.default_rng(43)
    q = rng.standard_normal((1, 5, 1, 8))
    k = rng.standard_normal((1, 9, 1, 8))
    v = rng.standard_normal((1, 9, 1, 4))
    w = 2
    out, lse = oracle.fwd(q, k, v, causal=True, scale=0.4, lib=lib, window=(w, -1))
    for i in range(5):
        a = i + 9 - 5
        lo = max(0, a - w)
        sc = 0.4 * k[0, lo:a + 1, 0] @ q[0, i, 0]
        assert np.allclose(out[0, i, 0], softmax(sc) @ v[0, lo:a + 1, 0], atol=1e-13)
        assert np.isclose(lse[0, 0, i], logsumexp(sc), atol=1e-13)
    # perturbing a key outside every window leaves the result unchanged
    k2, v2 = k.copy(), v.copy()
    k2[0, 0] += 5.0
    v2[0, 0] -= 3.0
    out2, lse2 = oracle.fwd(q, k2, v2, causal=True, scale=0.4, lib=lib, window=(w, -1))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def pin_window_in_kvcache_mode(lib):
    """The window applies to the cache path too, on the keys now in the cache:
    a decode row (s_new 1) with window (w, -1) equals plain attention over the
    last w + 1 keys."""
    rng = np.random.default_rng(44)
    kc = rng.standard_normal((1, 12, 1, 8))
    vc = rng.standard_normal((1, 12, 1, 8))
    q = rng.standard_normal((1, 1, 1, 8))
    kn = rng.standard_normal((1, 1, 1, 8))
    vn = rng.standard_normal((1, 1, 1, 8))
    out, lse, kc2, vc2 = oracle.kvcache_fwd(q, kc, vc, kn, vn, None, None, [9], causal=True, scale=0.5,
                                            window=(3, -1), lib=lib)
    ref, rlse = oracle.fwd(q, kc2[:, 6:10], vc2[:, 6:10], causal=False, scale=0.5, lib=lib)
    assert np.allclose(out, ref, atol=1e-14) and np.allclose(lse, rlse, atol=1e-14)


def pin_brute_force_windows(lib):
    """The oracle's window bounds agree with the brute force's distance
    predicate ("optimizing-attention-flash", window_size=(left, right)) on
    tiny shapes: causal and not, s_q below, equal to and above the key count,
    one- and two-sided windows, GQA."""
    rng = np.random.default_rng(71)
    for s_q, s_k in ((3, 6), (5, 5), (6, 3)):
        for causal in (True, False):
            for window in ((1, -1), (0, 2), (2, 1), (-1, 0), (4, 3)):
                q = rng.standard_normal((1, s_q, 2, 3))
                k = rng.standard_normal((1, s_k, 1, 3))
                v = rng.standard_normal((1, s_k, 1, 2))
                out, lse = oracle.fwd(q, k, v, causal=causal, window=window, lib=lib)
                for h in range(2):
                    bo, bl = brute.attention([list(r) for r in q[0, :, h]], [list(r) for r in k[0, :, 0]],
                                             [list(r) for r in v[0, :, 0]], s_q, causal, 1 / math.sqrt(3), window)
                    assert np.allclose(out[0, :, h], np.array(bo), rtol=0, atol=1e-12)
                    assert np.array_equal(np.isinf(lse[0, h]), np.isinf(np.array(bl)))
                    fin = np.isfinite(lse[0, h])
                    assert np.allclose(lse[0, h][fin], np.array(bl)[fin], rtol=0, atol=1e-12)


def pin_varlen_sequences_are_independent(lib):
    """Packed sequences ([P2] IS_VARLEN) do not see each other: changing one
    sequence's keys and values leaves every other sequence's output and lse
    bit-identical, and a single packed sequence equals the batched call."""
    rng = np.random.default_rng(51)
    cq = [0, 3, 3, 10]
    ck = [0, 5, 9, 21]
    q = rng.standard_normal((10, 2, 8))
    k = rng.standard_normal((21, 1, 8))
    v = rng.standard_normal((21, 1, 4))
    out, lse = oracle.fwd_varlen(q, k, v, cq, ck, causal=True, lib=lib)
    k2, v2 = k.copy(), v.copy()
    k2[9:] += 1.0
    v2[9:] -= 2.0
    out2, lse2 = oracle.fwd_varlen(q, k2, v2, cq, ck, causal=True, lib=lib)
    assert np.array_equal(out[:3], out2[:3]) and np.array_equal(lse[:, :3], lse2[:, :3])
    assert not np.allclose(out[3:], out2[3:])
    one, l1 = oracle.fwd_varlen(q[:3], k[:5], v[:5], [0, 3], [0, 5], causal=True, lib=lib)
    ref, rl = oracle.fwd(q[None, :3], k[None, :5], v[None, :5], causal=True, lib=lib)
    assert np.array_equal(one, ref[0]) and np.array_equal(l1, rl[0])


def _loss_grad_fd(q, k, v, dout, causal, window, lib, eps=1e-5):
    """Central finite differences of sum(dout * fwd(q, k, v)) in float64."""
    def loss(qq, kk, vv):
        out, _ = oracle.fwd(qq, kk, vv, causal=causal, window=window, lib=lib)
        return float((out * dout).sum())
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(*g.shape):
            a = [x.copy() for x in args]
            a[which][idx] += eps
            up = loss(*a)
            a[which][idx] -= 2 * eps
            g[idx] = (up - loss(*a)) / (2 * eps)
        grads.append(g)
    return grads


def pin_bwd_matches_finite_differences(lib):
    """The backward ("Support hdimQK != hdimV backward") is the gradient of
    the pinned forward: central differences of sum(dout * out) agree with
    dq, dk, dv for d_qk != d_v, GQA, causal (with rows that see no key),
    and a two-sided window."""
    rng = np.random.default_rng(61)
    for (s_q, s_k, h_q, h_kv, d_qk, d_v, causal, window) in (
            (3, 5, 2, 1, 4, 3, True, (-1, -1)),
            (4, 2, 2, 2, 3, 2, True, (-1, -1)),      # s_q > s_k: rows 0, 1 see no key
            (4, 4, 3, 1, 3, 4, False, (1, 1))):
        q = rng.standard_normal((1, s_q, h_q, d_qk))
        k = rng.standard_normal((1, s_k, h_kv, d_qk))
        v = rng.standard_normal((1, s_k, h_kv, d_v))
        dout = rng.standard_normal((1, s_q, h_q, d_v))
        got = oracle.bwd(q, k, v, dout, causal=causal, window=window, lib=lib)
        fd = _loss_grad_fd(q, k, v, dout, causal, window, lib)
        for name, a, e in zip(("dq", "dk", "dv"), got, fd):
            assert np.abs(a - e).max() <= 1e-7 * max(1.0, np.abs(e).max()), name


def pin_bwd_key_and_value_sums(lib):
    """Softmax rows sum to one, so each row of dS sums to zero: the keys'
    gradients sum to zero, and the values' gradients sum to the upstream
    gradient of every row that sees a key, over the group's query heads."""
    rng = np.random.default_rng(62)
    b, s_q, s_k, h_q, h_kv = 2, 6, 9, 4, 2
    q = rng.standard_normal((b, s_q, h_q, 8))
    k = rng.standard_normal((b, s_k, h_kv, 8))
    v = rng.standard_normal((b, s_k, h_kv, 5))
    dout = rng.standard_normal((b, s_q, h_q, 5))
    _, dk, dv = oracle.bwd(q, k, v, dout, causal=True, lib=lib)
    assert np.abs(dk.sum(axis=1)).max() <= 1e-12
    g = h_q // h_kv
    want = dout.reshape(b, s_q, h_kv, g, 5).sum(axis=(1, 3))
    assert np.abs(dv.sum(axis=1) - want).max() <= 1e-12


def pin_bwd_single_key(lib):
    """One key: P = 1 whatever the scores, so dq = dk = 0 and dv is the sum
    of the upstream gradients."""
    rng = np.random.default_rng(63)
    q = rng.standard_normal((1, 3, 2, 4))
    k = rng.standard_normal((1, 1, 1, 4))
    v = rng.standard_normal((1, 1, 1, 2))
    dout = rng.standard_normal((1, 3, 2, 2))
    dq, dk, dv = oracle.bwd(q, k, v, dout, causal=False, lib=lib)
    assert np.abs(dq).max() == 0.0 and np.abs(dk).max() == 0.0
    assert np.allclose(dv[0, 0, 0], dout.sum(axis=(0, 1, 2)), rtol=0, atol=1e-14)


def pin_bwd_zero_window_and_unseen_keys(lib):
    """A (0, 0) window gives each query exactly its aligned key (P = 1): dq =
    dk = 0 and dv_j = dout_j.  Keys no query sees (causal with a short left
    window) get no gradient at all."""
    rng = np.random.default_rng(64)
    q = rng.standard_normal((1, 5, 1, 4))
    k = rng.standard_normal((1, 5, 1, 4))
    v = rng.standard_normal((1, 5, 1, 3))
    dout = rng.standard_normal((1, 5, 1, 3))
    dq, dk, dv = oracle.bwd(q, k, v, dout, causal=False, window=(0, 0), lib=lib)
    assert np.abs(dq).max() == 0.0 and np.abs(dk).max() == 0.0
    assert np.array_equal(dv, dout)
    k2 = rng.standard_normal((1, 12, 1, 4))
    v2 = rng.standard_normal((1, 12, 1, 3))
    dq, dk, dv = oracle.bwd(q, k2, v2, dout, causal=True, window=(2, -1), lib=lib)
    # query i sits at key 7 + i and sees keys 5 + i .. 7 + i: keys 0 .. 4 unseen
    assert np.abs(dk[:, :5]).max() == 0.0 and np.abs(dv[:, :5]).max() == 0.0
    assert np.abs(dk[:, 5:]).max() > 0.0 and np.abs(dv[:, 5:]).max() > 0.0


def pin_bwd_gqa_equals_repeated_heads(lib):
    """GQA backward: a kv head's gradient is the sum of the gradients of its
    query heads' copies when every query head gets its own copy of k and v."""
    rng = np.random.default_rng(65)
    b, s_q, s_k, h_q, h_kv, d_qk, d_v = 1, 4, 7, 6, 2, 5, 3
    g = h_q // h_kv
    q = rng.standard_normal((b, s_q, h_q, d_qk))
    k = rng.standard_normal((b, s_k, h_kv, d_qk))
    v = rng.standard_normal((b, s_k, h_kv, d_v))
    dout = rng.standard_normal((b, s_q, h_q, d_v))
    dq, dk, dv = oracle.bwd(q, k, v, dout, causal=True, lib=lib)
    kr, vr = np.repeat(k, g, axis=2), np.repeat(v, g, axis=2)
    dq_r, dk_r, dv_r = oracle.bwd(q, kr, vr, dout, causal=True, lib=lib)
    assert np.abs(dq - dq_r).max() <= 1e-13
    assert np.abs(dk - dk_r.reshape(b, s_k, h_kv, g, d_qk).sum(axis=3)).max() <= 1e-13
    assert np.abs(dv - dv_r.reshape(b, s_k, h_kv, g, d_v).sum(axis=3)).max() <= 1e-13


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
