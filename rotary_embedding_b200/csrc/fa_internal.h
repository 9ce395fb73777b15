// fa_internal.h -- parameter blocks and launchers shared between the host
// planner (fa_api.cu) and the kernels.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"

namespace fa {

// Strides of a [batch, seq, heads, dim] tensor in elements (dim stride is 1).
struct Strides3 {
    int64_t b, s, h;
};

// Rotary + append (+ optional rotated copy of q), before the decode or the
// prefill attention kernel.
struct RopeAppendParams {
    int32_t *status;  // device status word (see fa_device_status)
    const void *k_new;
    Strides3 kn;
    const void *v_new;
    Strides3 vn;
    void *k_cache;
    Strides3 kc;
    void *v_cache;
    Strides3 vc;
    const void *q;
    Strides3 qs;
    void *q_rot;  // contiguous [b, s_q, h_q, d_qk]; nullptr = do not rotate q
    const void *cos, *sin;
    int64_t cs_row;   // row stride of cos/sin in elements
    int64_t cs_rows;  // rows of cos/sin
    const int32_t *seqlens;
    int32_t seqlen_scalar;
    int b, s_q, s_new, h_q, h_kv, d_qk, d_v, r, interleaved;
    int64_t cap;
    int32_t *zero_word;  // set to 0 by the kernel when not null (the decode work-pool counter)
};

// Split-KV decode over the cache after the RoPE/append kernel (s_q * h_q / h_kv
// <= 32 query rows per kv head).
struct DecodeParams {
    int32_t *status;  // device status word (see fa_device_status)
    int64_t cs_rows;  // rows of the cos/sin table (precondition check only)
    const int32_t *seqlens;
    int32_t seqlen_scalar;
    void *out;
    Strides3 os;
    float *lse;      // [b, h_q, s_q] or nullptr
    float *o_part;   // [b, h_q, s_q, n_splits, d_v]
    float *lse_part; // [b, h_q, s_q, n_splits]
    int b, s_q, s_new, h_q, h_kv, g, r, causal;
    int64_t cap;
    float scale_log2;
    int chunk;     // key rows per split, multiple of 64
    int n_stages;  // K/V ring depth (set by the launcher from the shared-memory budget)
    int n_splits;  // slots per output row (one per 64-row item of the longest segment)
    int *pool;     // work-pool counter (zeroed by the RoPE/append kernel)
    int win_left, win_right;  // sliding window (keys a - left .. a + right); -1 = unbounded
};

// Standalone rotary (fa_rotary): x [b, s, h, d] with element strides xs
// (batch, row, head), out likewise.  Row R = b * s + i; batched: position
// offsets[b] + i.  Packed (b = 1): rows cu[k] .. cu[k+1]-1 are sequence k and
// row R sits at offsets[k] + R - cu[k].
struct RotaryParams {
    int32_t *status;
    const void *x;
    Strides3 xs;
    void *out;
    Strides3 os;
    const void *cos, *sin;
    int64_t cs_row, cs_rows;
    const int32_t *offsets;  // [b] or [n_seqs]; nullptr: offset_scalar
    int32_t offset_scalar;
    const int32_t *cu_seqlens;  // [n_seqs + 1] or nullptr (batched)
    int n_seqs;
    int64_t rows;   // b * s, or total packed rows
    int s;          // batched: rows per batch entry
    int h, d, r, interleaved, conjugate;
};

// Generic attention (any supported head dim): keys from k/v (dense) or
// from the cache after the append kernel ran.
struct SimtAttnParams {
    int32_t *status;  // device status word (see fa_device_status)
    const void *q;
    Strides3 qs;
    const void *k;
    Strides3 ks;
    const void *v;
    Strides3 vs;
    void *out;
    Strides3 os;
    float *lse;
    const int32_t *seqlens;  // kvcache mode: N_b = seqlens[b] + s_new; nullptr = dense
    int32_t seqlen_scalar;
    int s_new;
    int64_t s_k;   // dense mode key rows
    int64_t cap;   // kvcache mode capacity (precondition check)
    int b, s_q, h_q, h_kv, g, d_qk, d_v, causal;
    int win_left, win_right;  // sliding window; -1 = unbounded
    float scale_log2;
};

// tcgen05 prefill / dense attention over Q, K, V described by TMA maps.
struct PrefillParams {
    int32_t *status;
    void *out;
    Strides3 os;
    float *lse;
    const int32_t *seqlens;  // kvcache mode: N_b = seqlens[b] + s_new
    int32_t seqlen_scalar;
    int s_new;
    int64_t s_k;   // dense mode key rows
    int64_t cap;   // kvcache mode capacity (precondition check)
    int kvcache, b, s_q, h_q, h_kv, g, pack, causal, n_q_tiles;
    int tiles_per_cta;  // 1: one 128-row tile per CTA; 2: two tiles, two softmax warpgroups
    // two-tile kernel: 0 = CTA k takes query tiles 2k and 2k+1; 1 = tiles k
    // and n_q_tiles-1-k (equal causal work per CTA, for single-wave grids)
    int pair_ends;
    // two-tile kernel: 1 = both tiles of a CTA are the same query tile, with
    // the key range cut in two halves merged at the end (grid: one CTA per
    // query tile)
    int key_split;
    // cache grids of one tile per CTA (one-tile kernel, key split): CTAs take
    // (batch entry, query tile) items heaviest first by visible keys,
    // computed on the device from cache_seqlens (b x n_q_tiles <= 256)
    int work_order;
    int win_left, win_right;  // sliding window; -1 = unbounded
    // packed sequences (varlen): grid z = sequence s with query rows
    // cu_q[s] .. cu_q[s+1]-1 and key rows cu_k[s] .. of batch entry 0;
    // lse is [h_q, total_q].  nullptr: batched.
    const int32_t *cu_q, *cu_k;
    int64_t total_q, total_k;
    float scale_log2;
};

// Visible keys of query row i (of s_q) over N keys, aligned bottom-right at
// a = i + N - s_q: first .. last (first > last: none).  Causal caps the last
// key at a; a sliding window (left, right) keeps a - left .. a + right.
__host__ __device__ __forceinline__ void visible_keys(int64_t i, int64_t N, int64_t s_q, int causal, int left,
                                                      int right, int64_t &first, int64_t &last) {
    const int64_t a = i + N - s_q;
    last = N - 1;
    if (causal && a < last) last = a;
    if (right >= 0 && a + right < last) last = a + right;
    first = left >= 0 ? a - left : 0;
    if (first < 0) first = 0;
}

int sm_count();

// Sets the thread-local message fa_last_error() returns; returns `code`.
int set_last_error(int code, const char *msg);

// Records the caller's profiling event (fa_set_kernel_events) on `st`, if set:
// which = 0 before the attention kernel's launch, 1 after it.
void kernel_event(int which, cudaStream_t st);

// Attention backward (dq, dk, dv) over dense [b, s, h, d] tensors.
struct BwdParams {
    int32_t *status;   // device status word (bounded waits record timeouts here)
    const void *q;
    Strides3 qs;
    const void *k;
    Strides3 ks;
    const void *v;
    Strides3 vs;
    const void *out;
    Strides3 os;
    const void *dout;
    Strides3 dos;
    const float *lse;  // [b, h_q, s_q], natural log, from the forward
    // workspace, [b, h_q, s_q_pad] each (s_q rounded up to 64 rows, so that
    // every 64-row tile of a (batch, head) is one aligned 256-byte run):
    float *lsum;       //   lse_i * log2(e) (+inf on the padding rows)
    float *dsum;       //   D_i = dout_i . out_i (0 on the padding rows)
    int s_q_pad;
    void *dq;
    Strides3 dqs;
    void *dk;
    Strides3 dks;
    void *dv;
    Strides3 dvs;
    int b, s_q, s_k, h_q, h_kv, g, d_qk, d_v, causal;
    int win_left, win_right;  // sliding window; -1 = unbounded
    float scale, scale_log2;
};

cudaError_t launch_rope_append(const RopeAppendParams &p, int dtype, cudaStream_t st);
cudaError_t launch_rotary(const RotaryParams &p, int dtype, cudaStream_t st);
bool prefill_supported(int d_qk, int d_v);
int prefill_block_n(int d_qk, int d_v, int tiles_per_cta);  // key rows per K/V tile (TMA box rows)
cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &tmQ, const CUtensorMap &tmK,
                           const CUtensorMap &tmV, int dtype, int d_qk, int d_v, cudaStream_t st);
// tmQ: the rotated q rows in the workspace, box (64 cols, g heads, s_q rows);
// tmK / tmV: the caches, box (64 cols, 1 head, 64 rows).
cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmQ, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, int dtype, int d_qk, int d_v, int mt, cudaStream_t st);
bool decode_supported(int d_qk, int d_v, int mt);
cudaError_t launch_simt_attn(const SimtAttnParams &p, int dtype, cudaStream_t st);
// TMA maps of the backward kernels over the caller's [b, s, h, d] tensors,
// named by the rows of their box: the dk/dv kernel reads 128-row K and V
// tiles and 64-row Q and dO tiles, the dq kernel 128-row Q and dO tiles and
// 64-row K and V tiles.
struct BwdMaps {
    CUtensorMap k128, v128, q64, do64, q128, do128, k64, v64;
};
bool bwd_supported(int d_qk, int d_v);
cudaError_t launch_bwd(const BwdParams &p, const BwdMaps &m, int dtype, cudaStream_t st);

}  // namespace fa
