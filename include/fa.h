/*
 * fa.h -- C ABI of the B200 (sm_100a) attention-with-KV-cache library (libfa.so).
 *
 * One hot path: the FlashAttention-style forward with a KV cache and fused
 * rotary position embedding (RoPE), plus plain cache-less attention.
 *
 * Sources (page title, then section):
 *  - flash-attention issue #1402 "is flash_attn_with_kvcache() supposed to
 *    work for seqlen > 1 ?": the call shape flash_attn_with_kvcache(q,
 *    k_cache, v_cache, k, v, rotary_cos, rotary_sin, cache_seqlens,
 *    rotary_interleaved) on [batch, seq, heads, dim] views that need not be
 *    contiguous (the reproducers pass transposed tensors); cos/sin hold
 *    rotary_dim/2 columns ("flash expects dim1 of size half the
 *    rotary_dim"); apply_rotary_emb / rotate_half define the rotation.
 *  - ROCm/flash-attention PR #99 "Added Support for Rotary Positional
 *    Embeddings (both non-fused and fused kernel)": COS/SIN of shape
 *    (seqlen, rotary_dim/2); the per-batch offset into them given either as
 *    an int or as a (batch,) tensor; INTERLEAVED pairing; partial rotary
 *    (rotary_fraction 0, 0.5, 1).
 *  - s2.cpp PR #40 "feat: Flash Attention and modernized KV Cache layout for
 *    Slow-AR": new k/v rows are written into the cache at their offsets and
 *    attention must read them after the write.
 *  - flash-attention PR #1604 "Support hdimQK != hdimV backward": d_qk may
 *    differ from d_v (192/128).
 *  - "optimizing-attention-flash" skill page, Workflow 2 Steps 2-3: layout
 *    [batch, seq, heads, dim], causal flag, softmax_scale=None meaning
 *    1/sqrt(d), fewer KV heads than query heads.
 *
 * What the library computes (all steps run in its CUDA kernels):
 *  1. RoPE of q and k_new at positions p = L_b + i (L_b = cache_seqlens[b],
 *     i = row within the new chunk): each pair (x0, x1) with angle index
 *     j < rotary_dim/2 becomes (x0 c - x1 s, x0 s + x1 c), c = cos[p][j],
 *     s = sin[p][j]; half-split pairs are (j, j + rotary_dim/2), interleaved
 *     pairs (2j, 2j+1); dims >= rotary_dim pass through; the result is
 *     rounded to the element type (round to nearest even).
 *  2. Append: k_cache[b][L_b+i][h] = rotated k_new[b][i][h],
 *     v_cache[b][L_b+i][h] = v_new[b][i][h] (bit copy).  Other cache rows
 *     are not written.  cache_seqlens is not advanced.
 *  3. Attention over the N_b = L_b + s_new keys now in the cache:
 *     out = softmax(scale * q' k^T + mask) v, query head h reading kv head
 *     h / (h_q / h_kv); causal masking aligned bottom-right (query i of s_q
 *     sees key j iff j <= i + N_b - s_q); lse = natural-log log-sum-exp of
 *     the scaled, masked scores (fp32).  A query row with no visible key
 *     gets out = 0 and lse = -inf.
 *
 * Conventions for every entry point:
 *  - All tensor data are DEVICE addresses owned by the caller.  The library
 *    allocates no memory and keeps no pointer after a call returns.  Work is
 *    enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and is asynchronous with respect to the host.
 *  - A tensor is described by fa_tensor: element strides, innermost (head
 *    dim) stride must be 1, every other stride and the base address must be
 *    multiples of 16 bytes (otherwise FA_ERR_LAYOUT; the caller can make a
 *    contiguous copy).  Layout is [batch, seq, heads, dim].
 *  - dtype is FA_DTYPE_F16 or FA_DTYPE_BF16 and is the same for q, k, v,
 *    caches, new rows, cos/sin and out.  Head dims are multiples of 8 in
 *    8..256.
 *  - Which kernel runs: a kvcache call with s_q <= 8 and at most 32 query
 *    rows per kv head (g * s_q) uses the split-KV decode kernel for head
 *    dims (d_qk, d_v) 16/16, 32/32, 64/64, 128/128, 192/128 and 256/256;
 *    other calls use the tcgen05 prefill kernels for 64/64, 128/128,
 *    192/128, 128/64, 64/128 and 192/64.  Every other accepted pair (for
 *    example 16/16, 32/32, 96/96 or 256/256 outside decode) runs on a
 *    generic CUDA-core kernel without tensor cores: same results, far
 *    lower throughput.  fa_kvcache_plan / fa_fwd_plan report the path.
 *  - Return value: FA_OK (0) or a negative FA_ERR_* code; fa_last_error()
 *    then gives a message (thread-local, valid until the next call on the
 *    same thread).  Arguments are fully validated on the host before any
 *    work is enqueued; no entry point throws.
 *  - Device-side preconditions (0 <= L_b, L_b + s_new <= cache capacity,
 *    L_b + s_q <= rows of cos/sin when RoPE is on) cannot be checked on the
 *    host when cache_seqlens lives on the device.  The kernels check them;
 *    a batch entry that violates them is skipped (its out/lse rows are left
 *    unwritten and its cache rows untouched) and FA_ERR_DEVICE_PRECONDITION
 *    is recorded in a device status word that fa_device_status() returns.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = -1,        /* null pointer, bad rank/shape, mismatched sizes */
    FA_ERR_UNSUPPORTED = -2,        /* dtype or head dim outside what the kernels cover */
    FA_ERR_LAYOUT = -3,             /* head-dim stride != 1, or strides/base not 16-byte aligned */
    FA_ERR_WORKSPACE = -4,          /* workspace missing or smaller than *_workspace_size */
    FA_ERR_CUDA = -5,               /* a CUDA runtime/driver call failed */
    FA_ERR_DEVICE_PRECONDITION = -6,/* recorded on the device: cache_seqlens out of range */
    FA_ERR_DEVICE_TIMEOUT = -7      /* recorded on the device: a bounded wait gave up */
};

enum fa_dtype {
    FA_DTYPE_F16 = 1,
    FA_DTYPE_BF16 = 2
};

typedef struct fa_tensor {
    void *data;          /* device address of element [0][0][0][0] */
    int32_t dtype;       /* enum fa_dtype */
    int32_t ndim;        /* 4 for q/k/v/out/caches/new rows, 2 for cos/sin */
    int64_t shape[4];    /* sizes; unused trailing entries ignored */
    int64_t stride[4];   /* element strides; stride[ndim-1] must be 1 */
} fa_tensor;

/*
 * fa_kvcache_fwd -- RoPE + cache append + attention over cache and new rows
 * (flash_attn_with_kvcache of issue #1402 / PR #99).
 *
 *   q        [b, s_q, h_q, d_qk]        read
 *   k_cache  [b, cap, h_kv, d_qk]       read; rows L_b..L_b+s_new-1 written
 *   v_cache  [b, cap, h_kv, d_v]        read; rows L_b..L_b+s_new-1 written
 *   k_new    [b, s_new, h_kv, d_qk]     read; NULL = no new rows (then v_new NULL)
 *   v_new    [b, s_new, h_kv, d_v]      read; s_new must equal s_q when given
 *   cos, sin [S_ro, rotary_dim/2]       read; NULL (both) = no RoPE
 *   cache_seqlens  int32 device array [b], or NULL to use cache_seqlens_scalar
 *                  for every batch entry (the int form of PR #99)
 *   rotary_dim     even, <= d_qk; ignored (treated as 0) when cos is NULL
 *   interleaved    0 = half-split pairs (j, j+r/2), 1 = pairs (2j, 2j+1)
 *   causal         0/1; bottom-right aligned
 *   scale          softmax scale; <= 0 means 1/sqrt(d_qk)
 *   out      [b, s_q, h_q, d_v]         written
 *   lse      fp32 device array [b, h_q, s_q] (contiguous) or NULL
 *   (These fourteen arguments, in this order, are the call the attention-
 *   with-KV-cache contract names; what follows is this library's addition.)
 *   cache_seqlens_scalar  the offset of every batch entry when cache_seqlens
 *                  is NULL; ignored otherwise
 *   workspace / workspace_bytes   device scratch of at least the size that
 *                  fa_kvcache_workspace_size() reports for the same shapes
 *                  (may be NULL when that size is 0); contents on entry are
 *                  ignored and on exit undefined.
 *   stream         cudaStream_t
 * out must not alias any input.  Concurrent calls on different streams must
 * not share a workspace or write the same cache rows.
 */
int fa_kvcache_fwd(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                   const fa_tensor *k_new, const fa_tensor *v_new,
                   const fa_tensor *cos, const fa_tensor *sin,
                   const int32_t *cache_seqlens,
                   int32_t rotary_dim, int32_t interleaved, int32_t causal, float scale,
                   const fa_tensor *out, float *lse,
                   int32_t cache_seqlens_scalar,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_kvcache_fwd_noalloc -- the same call as fa_kvcache_fwd, without a
 * workspace argument.  (The pages have no counterpart: this exists for
 * callers of this library.)
 *
 * For callers that cannot allocate device memory when they run attention:
 * a plug-in whose host application owns every device allocation and gives
 * it no allocator, or a latency-critical loop that must never enter the CUDA
 * allocator (cudaMalloc can synchronise the device).  The caller still
 * passes inputs and outputs; the scratch comes from a fixed array of
 * FA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.
 *
 *  - Arguments, layouts and results are those of fa_kvcache_fwd.
 *  - Shapes whose fa_kvcache_workspace_size exceeds FA_NOALLOC_SCRATCH_BYTES
 *    are rejected with FA_ERR_WORKSPACE (fa_last_error() says how much they
 *    need); nothing is enqueued.
 *  - The first call on a device looks up the scratch array's device address
 *    (cudaGetSymbolAddress) with that device current.  Under CUDA's lazy
 *    module loading (the default) that lookup is also what loads the
 *    array's module on the device, reserving its 32 MiB there, and it may
 *    synchronise.  So make one call on each device as a warm-up, before the
 *    region that must not allocate and before any stream capture; later
 *    calls allocate nothing and do not synchronise.
 *  - No cudaMalloc, cudaFree or other allocating routine is called.
 *  - Every call on a device shares the one scratch array: calls whose work
 *    overlaps on the GPU (different streams, or another thread) race on it
 *    and must be serialised by the caller.  The array keeps the last call's
 *    contents; nothing in it needs to start at zero.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

int fa_kvcache_fwd_noalloc(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                           const fa_tensor *k_new, const fa_tensor *v_new,
                           const fa_tensor *cos, const fa_tensor *sin,
                           const int32_t *cache_seqlens,
                           int32_t rotary_dim, int32_t interleaved, int32_t causal, float scale,
                           const fa_tensor *out, float *lse,
                           int32_t cache_seqlens_scalar, void *stream);

/* Workspace bytes fa_kvcache_fwd needs for these shapes (k_new may be NULL). */
int fa_kvcache_workspace_size(const fa_tensor *q, const fa_tensor *k_cache,
                              const fa_tensor *v_cache, const fa_tensor *k_new,
                              int32_t rotary_dim, size_t *bytes);

/*
 * fa_fwd -- cache-less attention (flash_attn_func of the
 * "optimizing-attention-flash" page, Quick start / Workflow 2).
 *   q [b, s_q, h_q, d_qk], k [b, s_k, h_kv, d_qk], v [b, s_k, h_kv, d_v],
 *   out [b, s_q, h_q, d_v], lse fp32 [b, h_q, s_q] or NULL.
 * Causal masking is bottom-right aligned (query i sees key j iff
 * j <= i + s_k - s_q); rows with no visible key get out = 0, lse = -inf.
 */
int fa_fwd(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
           int32_t causal, float scale, const fa_tensor *out, float *lse,
           void *workspace, size_t workspace_bytes, void *stream);

/* Sliding-window forms of fa_kvcache_fwd and fa_fwd: the window_size=(left,
 * right) of the "optimizing-attention-flash" page (Workflow 2 Steps 2-3;
 * (-1, -1) means no window).  Query row i, aligned bottom-right at key
 * position a = i + N - s_q (N = keys), sees keys a - window_left ..
 * a + window_right (each bound -1 = unbounded on that side), and with causal
 * also no key past a.  Every other argument, and the behaviour with
 * (-1, -1), is that of fa_kvcache_fwd / fa_fwd (which call these).  A row
 * with no visible key gets out = 0 and lse = -inf.  Returns
 * FA_ERR_INVALID_ARG for bounds below -1. */
int fa_kvcache_fwd_window(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                          const fa_tensor *k_new, const fa_tensor *v_new,
                          const fa_tensor *cos, const fa_tensor *sin,
                          const int32_t *cache_seqlens,
                          int32_t rotary_dim, int32_t interleaved, int32_t causal,
                          int32_t window_left, int32_t window_right, float scale,
                          const fa_tensor *out, float *lse,
                          int32_t cache_seqlens_scalar,
                          void *workspace, size_t workspace_bytes, void *stream);
int fa_fwd_window(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
                  int32_t causal, int32_t window_left, int32_t window_right, float scale,
                  const fa_tensor *out, float *lse,
                  void *workspace, size_t workspace_bytes, void *stream);

/* Attention over packed sequences (the IS_VARLEN option of ROCm/flash-
 * attention PR #99): sequences of different lengths stored back to back.
 *  - q [total_q, h_q, d_qk], k [total_k, h_kv, d_qk], v [total_k, h_kv, d_v],
 *    out [total_q, h_q, d_v]: fp16/bf16, head-dim stride 1, other strides and
 *    base multiples of 16 bytes.  Head dims: the pairs the tcgen05 kernel
 *    takes (64/64, 128/128, 192/128, 128/64, 64/128, 192/64), else
 *    FA_ERR_UNSUPPORTED.
 *  - cu_seqlens_q, cu_seqlens_k: int32 DEVICE arrays [n_seqs + 1] of
 *    non-decreasing row starts; sequence s owns query rows cu_q[s] ..
 *    cu_q[s+1]-1 and key rows cu_k[s] .. cu_k[s+1]-1, and is attended as a
 *    batch of one (bottom-right causal alignment, window as in
 *    fa_fwd_window, inside the sequence).
 *  - max_seqlen_q: an upper bound of cu_q[s+1] - cu_q[s] (sizes the grid;
 *    rows past it are not computed).
 *  - lse: fp32 DEVICE array [h_q, total_q] (contiguous) or NULL.
 *  - Device-side precondition: every sequence lies inside the packed rows;
 *    a sequence that does not is skipped and FA_ERR_DEVICE_PRECONDITION is
 *    recorded (fa_device_status).
 * Allocates nothing; asynchronous on `stream`. */
int fa_fwd_varlen(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t n_seqs,
                  int32_t max_seqlen_q, int32_t causal, int32_t window_left, int32_t window_right,
                  float scale, const fa_tensor *out, float *lse, void *stream);

/*
 * fa_bwd -- gradients of fa_fwd_window (flash-attention PR #1604 "Support
 * hdimQK != hdimV backward": d_qk may differ from d_v).  For out =
 * softmax(scale q k^T + mask) v and an upstream gradient dout it writes
 *   dq = d sum(dout * out) / dq, and likewise dk and dv,
 * with the forward's mask (causal aligned bottom-right, window as in
 * fa_fwd_window) and GQA mapping; a kv head's dk and dv sum the gradients of
 * its group's query heads.
 *  - q, dq [b, s_q, h_q, d_qk]; k, dk [b, s_k, h_kv, d_qk]; v, dv
 *    [b, s_k, h_kv, d_v]; out, dout [b, s_q, h_q, d_v]: fp16/bf16 (one type
 *    for all), head-dim stride 1, other strides and base addresses multiples
 *    of 16 bytes.  q, k, v, out, dout are read only; dq, dk, dv are written
 *    in full (zeros where no visible pair reaches an element) and must not
 *    overlap the inputs.
 *  - out and lse are the forward's results for the same q, k, v, mask and
 *    scale (fa_fwd_window): lse fp32 [b, h_q, s_q], natural log, 4-byte
 *    aligned.  P is recomputed as exp(scale q.k - lse).
 *  - Head dims (d_qk, d_v): 64/64, 128/128, 192/128, else
 *    FA_ERR_UNSUPPORTED.  scale <= 0 means 1/sqrt(d_qk).
 *  - workspace: caller-owned device memory of fa_bwd_workspace_size bytes,
 *    16-byte aligned (FA_ERR_WORKSPACE if smaller); it holds lse_i log2(e)
 *    and D_i = dout_i . out_i as two fp32 arrays [b, h_q, s_q rounded up to
 *    64] and is dead after the call.
 *  - Enqueued on `stream`; returns without synchronising.  The result does
 *    not depend on scheduling (no atomics).  Errors: FA_ERR_INVALID_ARG
 *    (shapes, types, window bounds below -1, lse missing), FA_ERR_LAYOUT,
 *    FA_ERR_UNSUPPORTED, FA_ERR_CUDA.
 */
int fa_bwd(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
           const fa_tensor *out, const fa_tensor *dout, const float *lse,
           int32_t causal, int32_t window_left, int32_t window_right, float scale,
           const fa_tensor *dq, const fa_tensor *dk, const fa_tensor *dv,
           void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes fa_bwd needs for q of shape [b, s_q, h_q, d_qk]. */
int fa_bwd_workspace_size(const fa_tensor *q, size_t *bytes);

/* Workspace bytes fa_fwd needs for these shapes. */
int fa_fwd_workspace_size(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v,
                          size_t *bytes);

/* How a call with these shapes will run (for tests, benchmarks, tracing). */
typedef struct fa_plan {
    int32_t path;            /* FA_PATH_DECODE, FA_PATH_PREFILL or FA_PATH_DENSE */
    int32_t launches;        /* kernels one call enqueues */
    int32_t n_splits;        /* decode: key splits per (batch, kv head); else 1 */
    int32_t chunk;           /* decode: key rows per split; else 0 */
    size_t workspace_bytes;  /* same as the *_workspace_size functions */
} fa_plan;

enum fa_path { FA_PATH_DECODE = 1, FA_PATH_PREFILL = 2, FA_PATH_DENSE = 3 };

/* Plan of fa_kvcache_fwd for these shapes; host only, no device access.
 * `k_new` may be NULL; launches assume cache_seqlens leaves work to do. */
int fa_kvcache_plan(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                    const fa_tensor *k_new, int32_t rotary_dim, fa_plan *plan);

/* Plan of fa_fwd for these shapes; host only. */
int fa_fwd_plan(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, fa_plan *plan);

/* Reads (and clears) the device status word of the current device after
 * synchronising `stream`; *status receives FA_OK or an FA_ERR_DEVICE_* code. */
int fa_device_status(void *stream, int32_t *status);

/* Standalone rotary embedding: the "non-fused" rotary kernel of
 * ROCm/flash-attention PR #99 (COS/SIN of shape (seqlen, rotary_dim/2),
 * SEQLEN_OFFSET as an int or one value per batch entry, INTERLEAVED,
 * CONJUGATE, IS_VARLEN), with the pairing of the RoFormer rotation that
 * page's "Motivation" describes.
 *  - x: [b, s, h, d] (batched), or [1, total, h, d] holding packed sequences
 *    when cu_seqlens is given.  fp16/bf16, head-dim stride 1, other strides
 *    multiples of 16 bytes, d a multiple of 8 and <= 256.
 *  - out: same shape and type as x; may be x itself (in place).
 *  - cos, sin: [S_ro, rotary_dim/2] in x's type (row stride free).
 *  - seqlen_offsets: int32 device array with one offset per batch entry (or
 *    per packed sequence), or NULL to use seqlen_offset_scalar for all.
 *  - cu_seqlens: NULL (batched: row i of entry b is at table row
 *    offset_b + i), or an int32 device array [n_seqs + 1] of increasing row
 *    starts (packed: row t of sequence k, cu_seqlens[k] <= t <
 *    cu_seqlens[k+1], is at table row offset_k + t - cu_seqlens[k]).  Rows
 *    outside every sequence are copied unchanged.
 *  - rotary_dim: even, <= d; dims >= rotary_dim are copied.  0: plain copy.
 *  - interleaved: 0 pairs (j, j + rotary_dim/2), 1 pairs (2j, 2j+1).
 *  - conjugate: 1 rotates by the negated angle (sin replaced by -sin), the
 *    inverse rotation.  Pairs are computed in fp32 and rounded to nearest
 *    even.
 *  - Device-side precondition: every position lies in [0, S_ro); a row that
 *    does not is left as it is and FA_ERR_DEVICE_PRECONDITION is recorded
 *    (fa_device_status).
 * Allocates nothing; asynchronous on `stream`. */
int fa_rotary(const fa_tensor *x, const fa_tensor *cos, const fa_tensor *sin,
              const int32_t *seqlen_offsets, int32_t seqlen_offset_scalar,
              const int32_t *cu_seqlens, int32_t n_seqs,
              int32_t rotary_dim, int32_t interleaved, int32_t conjugate,
              const fa_tensor *out, void *stream);

/* Profiling hook; the pages have no counterpart (it exists so that a
 * benchmark can time the attention kernel alone, apart from the RoPE/append
 * kernel before it and the split-combine kernel after it).
 *  - start, stop: cudaEvent_t handles created by the caller with timing
 *    enabled, or both NULL to switch the hook off.  The library does not own
 *    them; the caller keeps them alive while the hook is on.
 *  - While set, every fa_kvcache_fwd / fa_kvcache_fwd_noalloc / fa_fwd /
 *    fa_fwd_varlen / fa_rotary call records `start` on its stream just before
 *    the launch of its main kernel (decode, prefill, generic attention or
 *    rotary) and `stop` just after it; fa_bwd records them around its dk/dv
 *    and dq kernels (after the D_i kernel) (inside a
 *    stream capture as external event-record nodes).  The events sit between
 *    the decode and combine kernels, so while the hook is on the combine
 *    launch no longer overlaps the decode kernel's tail.
 *  - Process-wide state, not synchronised: set it while no other thread is
 *    calling the library.  Returns FA_ERR_INVALID_ARG if exactly one is NULL. */
int fa_set_kernel_events(void *start, void *stop);

/* Static message for a status code. */
const char *fa_status_string(int status);

/* Message describing the last failing call on this thread ("" if none). */
const char *fa_last_error(void);

/* Library ABI version (major * 100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
