"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module only draws inputs; it holds none of the attention or rotation
arithmetic.  Each workload follows the shapes, dtypes and value
distributions of the attention-with-KV-cache configurations studied on the
pages (the reproducer of flash-attention issue #1402, the decode and chunked
prefill uses of flash_attn_with_kvcache, the dense timing harness of the
"optimizing-attention-flash" page, and the 192/128 head dims of
flash-attention PR #1604).

Draw order is fixed (q, k_new, v_new, k_cache, v_cache, cache_seqlens) on a
CPU ``torch.Generator`` seeded with 0, as the kvcache test of
ROCm/flash-attention PR #99 seeds with 0.  Floating values are drawn in
fp32 and rounded to the element type, so every consumer sees the same
dtype-exact values.

The rotary cos/sin tables are an input the caller builds (the RoPE
reproducer of issue #1402 builds them from inv_freq = base^(-2j/r) and the
position): they are built here in float64 and rounded to the element type.
"""
from __future__ import annotations

import dataclasses
import math

import torch

_DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str                 # "kvcache" (fa_kvcache_fwd), "dense" (fa_fwd), "rotary" (fa_rotary),
                              # "varlen" (fa_fwd_varlen: batch packed sequences, lengths ~ U{seqlens})
                              # or "bwd" (fa_bwd over the dense shapes, with an upstream gradient dout)
    dtype: str                # "fp16" | "bf16"
    batch: int
    h_q: int
    h_kv: int
    d_qk: int
    d_v: int
    s_q: int                  # query rows (= seqlen_new in kvcache mode)
    s_k: int = 0              # dense mode: key rows
    cap: int = 0              # kvcache mode: cache capacity
    seqlens: tuple = (0, 0)   # kvcache mode: cache_seqlens ~ U{lo..hi}
    seqlens_scalar: bool = False   # pass cache_seqlens as a host int
    causal: bool = True
    rotary_dim: int = 0
    interleaved: bool = False
    rotary_base: float = 10000.0
    scale: float = 0.0        # <= 0 means 1/sqrt(d_qk)
    dist: str = "randn"       # "randn" (N(0,1)) or "rand" (U[0,1))
    kv_is_q: bool = False     # the issue-#1402 reproducer passes key = value = query
    zero_cache: bool = False
    conjugate: bool = False   # rotary mode: rotate by the negated angle
    window: tuple = (-1, -1)  # sliding window (left, right) keys around the aligned position; -1 = none

    @property
    def torch_dtype(self):
        return _DT[self.dtype]

    def softmax_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d_qk)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five configurations (plus the decode variant of the fifth).
ISSUE_REPRO = Workload(
    name="issue-repro fp16 b4 h16 d16 s_new2 cap2", mode="kvcache", dtype="fp16",
    batch=4, h_q=16, h_kv=16, d_qk=16, d_v=16, s_q=2, cap=2, seqlens=(0, 0),
    seqlens_scalar=True, causal=False, scale=0.25, dist="rand", kv_is_q=True,
    zero_cache=True)
GQA_DECODE = Workload(
    name="gqa-decode-rope bf16 b8 hq32 hkv8 d128 cap8192 L~U{1024..8000}",
    mode="kvcache", dtype="bf16", batch=8, h_q=32, h_kv=8, d_qk=128, d_v=128, s_q=1,
    cap=8192, seqlens=(1024, 8000), causal=True, rotary_dim=64, interleaved=False)
CHUNKED_PREFILL = Workload(
    name="chunked-prefill fp16 b4 h16 d128 s_new512 cap4096 L~U{0..3000} rope128-interleaved",
    mode="kvcache", dtype="fp16", batch=4, h_q=16, h_kv=16, d_qk=128, d_v=128, s_q=512,
    cap=4096, seqlens=(0, 3000), causal=True, rotary_dim=128, interleaved=True)
DENSE_CAUSAL = Workload(
    name="dense fp16 b2 h8 s2048 d64 causal", mode="dense", dtype="fp16", batch=2,
    h_q=8, h_kv=8, d_qk=64, d_v=64, s_q=2048, s_k=2048, causal=True, scale=0.125)
DENSE_NONCAUSAL = DENSE_CAUSAL.scaled(name="dense fp16 b2 h8 s2048 d64 non-causal", causal=False)
MLA_PREFILL = Workload(
    name="mla-prefill bf16 b4 h16 s4096 dqk192 dv128 causal", mode="dense", dtype="bf16",
    batch=4, h_q=16, h_kv=16, d_qk=192, d_v=128, s_q=4096, s_k=4096, causal=True)
MLA_DECODE = Workload(
    name="mla-decode bf16 b4 h16 dqk192 dv128 cap16384 L16383", mode="kvcache",
    dtype="bf16", batch=4, h_q=16, h_kv=16, d_qk=192, d_v=128, s_q=1, cap=16384,
    seqlens=(16383, 16383), causal=True)

# The standalone rotary kernel (the next step widened from the path): q of a
# long prefill, rotated in place of the attention kernel's fused RoPE.
ROTARY_Q = Workload(
    name="rotary-q bf16 b4 s4096 h32 d128 rope128 half-split offsets~U{0..4096}", mode="rotary",
    dtype="bf16", batch=4, h_q=32, h_kv=32, d_qk=128, d_v=128, s_q=4096, cap=8192,
    seqlens=(0, 4096), rotary_dim=128, interleaved=False)

# Sliding-window prefill (the window_size=(left, right) of the
# "optimizing-attention-flash" page): causal, 1024 keys to the left.
WINDOW_PREFILL = Workload(
    name="window-prefill bf16 b2 h16 s8192 d128 causal window(1024,0)", mode="dense", dtype="bf16",
    batch=2, h_q=16, h_kv=16, d_qk=128, d_v=128, s_q=8192, s_k=8192, causal=True, window=(1024, 0))

# Packed prefill of sequences of mixed lengths ([P2] IS_VARLEN).
VARLEN_PREFILL = Workload(
    name="varlen-prefill bf16 8 seqs len~U{256..4096} h16 d128 causal", mode="varlen", dtype="bf16",
    batch=8, h_q=16, h_kv=16, d_qk=128, d_v=128, s_q=4096, seqlens=(256, 4096), causal=True)

# Backward of the MLA prefill (flash-attention PR #1604: d_qk 192, d_v 128).
MLA_BACKWARD = MLA_PREFILL.scaled(name="mla-backward bf16 b4 h16 s4096 dqk192 dv128 causal", mode="bwd")

CONFIGS = {
    "mla-backward": MLA_BACKWARD,
    "rotary-q": ROTARY_Q,
    "varlen-prefill": VARLEN_PREFILL,
    "window-prefill": WINDOW_PREFILL,
    "issue-repro": ISSUE_REPRO,
    "gqa-decode": GQA_DECODE,
    "chunked-prefill": CHUNKED_PREFILL,
    "dense-causal": DENSE_CAUSAL,
    "dense-noncausal": DENSE_NONCAUSAL,
    "mla-prefill": MLA_PREFILL,
    "mla-decode": MLA_DECODE,
}


def rotary_tables(rows: int, rotary_dim: int, base: float, dtype) -> tuple:
    """cos/sin tables [rows, rotary_dim/2]: angle(p, j) = p * base^(-2j/r), rounded to dtype."""
    j = torch.arange(rotary_dim // 2, dtype=torch.float64)
    inv_freq = base ** (-2.0 * j / rotary_dim)
    ang = torch.outer(torch.arange(rows, dtype=torch.float64), inv_freq)
    return torch.cos(ang).to(dtype), torch.sin(ang).to(dtype)


def _draw(gen, shape, dist, dtype):
    if dist == "rand":
        x = torch.rand(shape, generator=gen, dtype=torch.float32)
    else:
        x = torch.randn(shape, generator=gen, dtype=torch.float32)
    return x.to(dtype)


def make_inputs(w: Workload, seed: int = 0) -> dict:
    """Draw one batch of inputs for workload `w` on the CPU (contiguous tensors)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    dt = w.torch_dtype
    if w.mode == "rotary":
        # x as "q" [b, s, h, d]; per-batch position offsets as "cache_seqlens"
        q = _draw(g, (w.batch, w.s_q, w.h_q, w.d_qk), w.dist, dt)
        lo, hi = w.seqlens
        offs = torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int32)
        cos, sin = rotary_tables(w.cap, w.rotary_dim, w.rotary_base, dt)
        return {"q": q, "cache_seqlens": offs, "cos": cos, "sin": sin}
    if w.mode == "varlen":
        lo, hi = w.seqlens
        lens = torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int32)
        total = int(lens.sum())
        q = _draw(g, (total, w.h_q, w.d_qk), w.dist, dt)
        k = _draw(g, (total, w.h_kv, w.d_qk), w.dist, dt)
        v = _draw(g, (total, w.h_kv, w.d_v), w.dist, dt)
        cu = torch.zeros(w.batch + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lens, 0)
        return {"q": q, "k": k, "v": v, "cu_seqlens": cu}
    if w.mode in ("dense", "bwd"):
        q = _draw(g, (w.batch, w.s_q, w.h_q, w.d_qk), w.dist, dt)
        k = _draw(g, (w.batch, w.s_k, w.h_kv, w.d_qk), w.dist, dt)
        v = _draw(g, (w.batch, w.s_k, w.h_kv, w.d_v), w.dist, dt)
        if w.mode == "dense":
            return {"q": q, "k": k, "v": v}
        dout = _draw(g, (w.batch, w.s_q, w.h_q, w.d_v), w.dist, dt)
        return {"q": q, "k": k, "v": v, "dout": dout}
    q = _draw(g, (w.batch, w.s_q, w.h_q, w.d_qk), w.dist, dt)
    if w.kv_is_q:
        k_new, v_new = q.clone(), q.clone()
    else:
        k_new = _draw(g, (w.batch, w.s_q, w.h_kv, w.d_qk), w.dist, dt)
        v_new = _draw(g, (w.batch, w.s_q, w.h_kv, w.d_v), w.dist, dt)
    if w.zero_cache:
        k_cache = torch.zeros((w.batch, w.cap, w.h_kv, w.d_qk), dtype=dt)
        v_cache = torch.zeros((w.batch, w.cap, w.h_kv, w.d_v), dtype=dt)
    else:
        k_cache = _draw(g, (w.batch, w.cap, w.h_kv, w.d_qk), w.dist, dt)
        v_cache = _draw(g, (w.batch, w.cap, w.h_kv, w.d_v), w.dist, dt)
    lo, hi = w.seqlens
    seqlens = torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int32)
    out = {"q": q, "k_new": k_new, "v_new": v_new, "k_cache": k_cache, "v_cache": v_cache,
           "cache_seqlens": seqlens}
    if w.rotary_dim:
        out["cos"], out["sin"] = rotary_tables(w.cap, w.rotary_dim, w.rotary_base, dt)
    return out


def rotary_bytes(w: Workload) -> int:
    """Algorithmic bytes of one standalone rotary call: x read, out written,
    and the cos/sin row of every row read."""
    e = 2
    return (2 * w.batch * w.s_q * w.h_q * w.d_qk * e
            + w.batch * w.s_q * w.rotary_dim * e)


def kvcache_bytes(w: Workload, seqlens) -> int:
    """Algorithmic bytes of one kvcache call: cache rows attended (read), new rows
    read and written, q read, out written, lse written, cos/sin rows read."""
    e = 2
    old_rows = sum(int(x) for x in seqlens)
    b = old_rows * w.h_kv * (w.d_qk + w.d_v) * e                     # cache rows read
    b += w.batch * w.s_q * w.h_kv * (w.d_qk + w.d_v) * e * 2         # new rows: read + write
    b += w.batch * w.s_q * w.h_q * (w.d_qk + w.d_v) * e              # q read, out write
    b += w.batch * w.h_q * w.s_q * 4                                 # lse
    if w.rotary_dim:
        b += w.batch * w.s_q * w.rotary_dim * e                      # cos + sin rows
    return b


def visible_pairs(w: Workload, seqlens=None) -> int:
    """Number of visible (query row, key) pairs summed over batch and query heads."""
    total = 0
    if w.mode == "varlen":
        # seqlens: the drawn lengths; each sequence is a batch of one with s_q = s_k
        return sum(visible_pairs(w.scaled(mode="dense", batch=1, s_q=int(n), s_k=int(n)))
                   for n in seqlens) if seqlens is not None else 0
    if w.mode in ("dense", "bwd"):
        lens = [w.s_k] * w.batch
        s_q = w.s_q
    else:
        s_q = w.s_q
        lens = [int(x) + w.s_q for x in seqlens]
    for n in lens:
        if w.window != (-1, -1):
            # query i at a = i + n - s_q sees keys max(0, a - left) .. min(n - 1, a [causal], a + right)
            left, right = w.window
            for i in range(s_q):
                a = i + n - s_q
                hi = n - 1
                if w.causal:
                    hi = min(hi, a)
                if right >= 0:
                    hi = min(hi, a + right)
                lo = max(0, a - left) if left >= 0 else 0
                total += max(0, hi - lo + 1)
        elif not w.causal:
            total += s_q * n
        else:
            # query i sees keys j <= i + n - s_q
            lo = n - s_q + 1   # keys visible to row 0
            if lo >= 1:
                total += s_q * lo + s_q * (s_q - 1) // 2
            else:
                total += sum(max(0, min(n, i + n - s_q + 1)) for i in range(s_q))
    return total * w.h_q


def flops(w: Workload, seqlens=None) -> float:
    """Algorithmic FLOPs per visible (query, key) pair: forward 2*(d_qk + d_v)
    (q.k and p*v); backward 2*(3*d_qk + 2*d_v) (q.k, dout.v, p*dout into dv,
    ds*q into dk, ds*k into dq)."""
    per_pair = 2.0 * (3 * w.d_qk + 2 * w.d_v) if w.mode == "bwd" else 2.0 * (w.d_qk + w.d_v)
    return per_pair * visible_pairs(w, seqlens)
