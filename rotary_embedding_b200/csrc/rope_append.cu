// rope_append.cu -- fused RoPE + KV-cache append, ahead of the decode or the
// prefill attention kernel.
//
// One thread per 16-byte chunk (8 elements) of a row.  Rows are, in order:
// the new key rows (rotated at position L_b + i, rounded, written to
// k_cache row L_b + i), the new value rows (bit copy to v_cache row
// L_b + i) and, when a rotated copy of q is requested, the query rows
// (rotated at position L_b + i into a contiguous buffer).  Loads and stores
// are 128-bit and consecutive threads touch consecutive chunks of a row.
//
// Follows flash-attention issue #1402 (apply_rotary_emb / rotate_half,
// cache_seqlens offsets), ROCm/flash-attention PR #99 (COS/SIN (seqlen,
// rotary_dim/2), int or per-batch SEQLEN_OFFSET, INTERLEAVED) and s2.cpp
// PR #40 (write the new k/v rows at their offsets before attention reads
// them; the attention kernel is enqueued after this one on the same stream).
// The decode kernel is launched as this kernel's programmatic dependent: every
// CTA releases it at once, and it waits for this grid's completion (and the
// visibility of its writes) before it reads q or new cache rows.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

// At most 40 registers per thread, so that one of these blocks and two CTAs
// of the decode kernel (its programmatic dependent) fit on an SM together.
template <typename T>
__global__ void __launch_bounds__(256, 6) rope_append_kernel(RopeAppendParams p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (p.zero_word && blockIdx.x == 0 && threadIdx.x == 0) *p.zero_word = 0;
    const int ck = p.d_qk / 8, cv = p.d_v / 8;
    const int64_t n_k = (int64_t)p.b * p.s_new * p.h_kv * ck;
    const int64_t n_v = (int64_t)p.b * p.s_new * p.h_kv * cv;
    const int64_t n_q = p.q_rot ? (int64_t)p.b * p.s_q * p.h_q * ck : 0;
    const int64_t total = n_k + n_v + n_q;
    const bool inter = p.interleaved != 0;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        int64_t t = idx;
        int kind;  // 0 = k_new, 1 = v_new, 2 = q
        int c, h, i, b;
        if (t < n_k) {
            kind = 0;
            c = (int)(t % ck); t /= ck;
            h = (int)(t % p.h_kv); t /= p.h_kv;
            i = (int)(t % p.s_new); b = (int)(t / p.s_new);
        } else if ((t -= n_k) < n_v) {
            kind = 1;
            c = (int)(t % cv); t /= cv;
            h = (int)(t % p.h_kv); t /= p.h_kv;
            i = (int)(t % p.s_new); b = (int)(t / p.s_new);
        } else {
            t -= n_v;
            kind = 2;
            c = (int)(t % ck); t /= ck;
            h = (int)(t % p.h_q); t /= p.h_q;
            i = (int)(t % p.s_q); b = (int)(t / p.s_q);
        }
        const int L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
        // device-side preconditions: the new rows fit the cache and the table
        if (L < 0 || (int64_t)L + p.s_new > p.cap ||
            (p.r > 0 && (int64_t)L + (kind == 2 ? p.s_q : p.s_new) > p.cs_rows)) {
            if (c == 0 && h == 0 && i == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
            continue;
        }
        const int64_t pos = (int64_t)L + i;
        const T *cos_row = p.r > 0 ? static_cast<const T *>(p.cos) + pos * p.cs_row : nullptr;
        const T *sin_row = p.r > 0 ? static_cast<const T *>(p.sin) + pos * p.cs_row : nullptr;
        if (kind == 1) {
            const T *src = static_cast<const T *>(p.v_new) + b * p.vn.b + i * p.vn.s + h * p.vn.h;
            T *dst = static_cast<T *>(p.v_cache) + b * p.vc.b + pos * p.vc.s + h * p.vc.h;
            reinterpret_cast<uint4 *>(dst)[c] = __ldg(reinterpret_cast<const uint4 *>(src) + c);
            continue;
        }
        const T *src;
        T *dst;
        if (kind == 0) {
            src = static_cast<const T *>(p.k_new) + b * p.kn.b + i * p.kn.s + h * p.kn.h;
            dst = static_cast<T *>(p.k_cache) + b * p.kc.b + pos * p.kc.s + h * p.kc.h;
        } else {
            src = static_cast<const T *>(p.q) + b * p.qs.b + i * p.qs.s + h * p.qs.h;
            dst = static_cast<T *>(p.q_rot) + (((int64_t)b * p.s_q + i) * p.h_q + h) * p.d_qk;
        }
        float f[8];
        load_rotated_chunk<T>(src, c, p.r, inter, cos_row, sin_row, f);
        reinterpret_cast<uint4 *>(dst)[c] = pack8<T>(f);
    }
}

cudaError_t launch_rope_append(const RopeAppendParams &p, int dtype, cudaStream_t st) {
    const int64_t total = (int64_t)p.b * p.s_new * p.h_kv * (p.d_qk / 8 + p.d_v / 8) +
                          (p.q_rot ? (int64_t)p.b * p.s_q * p.h_q * (p.d_qk / 8) : 0);
    if (total == 0 && !p.zero_word) return cudaSuccess;
    int64_t blocks = total > 0 ? (total + 255) / 256 : 1;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (dtype == FA_DTYPE_F16)
        rope_append_kernel<__half><<<(unsigned)blocks, 256, 0, st>>>(p);
    else
        rope_append_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace fa
