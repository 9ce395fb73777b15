// rope_append.cu -- fused RoPE + KV-cache append, ahead of the decode or the
// prefill attention kernel.
//
// One 128-thread block per (batch entry b, row i) and group of 256 16-byte
// chunks of that row's work: the new key row of every kv head (rotated at
// position L_b + i, rounded, written to k_cache row L_b + i), the new value
// row of every kv head (bit copy to v_cache row L_b + i) and, when a rotated
// copy of q is requested, the query row of every head (rotated at position
// L_b + i into a contiguous buffer).  Each thread first issues the 128-bit
// loads of its two chunks (they do not depend on cache_seqlens), then the
// block reads L_b and stages the cos/sin row of position L_b + i in shared
// memory once for all heads, and the thread rotates and stores.
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

constexpr int kRopeThreads = 128;
constexpr int kRopeOps = 2;   // 16-byte chunks per thread

// At most 64 registers per thread, so that one of these blocks and two CTAs
// of the decode kernel (its programmatic dependent) fit on an SM together.
template <typename T>
__global__ void __launch_bounds__(kRopeThreads, 8) rope_append_kernel(RopeAppendParams p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (p.zero_word && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.zero_word = 0;
    __shared__ __align__(16) float cs_s[128], sn_s[128];
    const int rows = max(1, max(p.q_rot ? p.s_q : 0, p.s_new));
    const int b = blockIdx.x / rows, i = blockIdx.x % rows;
    const int ck = p.d_qk >> 3, cv = p.d_v >> 3;
    const bool has_new = i < p.s_new;
    const bool has_q = p.q_rot != nullptr && i < p.s_q;
    const int n_k = has_new ? p.h_kv * ck : 0;
    const int n_v = has_new ? p.h_kv * cv : 0;
    const int n_q = has_q ? p.h_q * ck : 0;
    const int total = n_k + n_v + n_q;
    if ((int)blockIdx.y * kRopeOps * kRopeThreads >= total) return;
    const bool inter = p.interleaved != 0;
    const int half = p.r >> 1;
    const bool chunk_partner = !inter && (half & 7) == 0;

    // this thread's chunks: kind 0 = k_new, 1 = v_new, 2 = q; source loads first
    int kind[kRopeOps], head[kRopeOps], chunk[kRopeOps];
    const T *srow[kRopeOps];
    uint4 raw[kRopeOps], praw[kRopeOps];
#pragma unroll
    for (int u = 0; u < kRopeOps; ++u) {
        const int t = ((int)blockIdx.y * kRopeOps + u) * kRopeThreads + (int)threadIdx.x;
        kind[u] = -1;
        head[u] = chunk[u] = 0;
        srow[u] = nullptr;
        raw[u] = praw[u] = make_uint4(0, 0, 0, 0);
        if (t >= total) continue;
        int c, h, kd;
        if (t < n_k) {
            kd = 0; h = t / ck; c = t - h * ck;
            srow[u] = static_cast<const T *>(p.k_new) + b * p.kn.b + i * p.kn.s + h * p.kn.h;
        } else if (t < n_k + n_v) {
            const int t2 = t - n_k;
            kd = 1; h = t2 / cv; c = t2 - h * cv;
            srow[u] = static_cast<const T *>(p.v_new) + b * p.vn.b + i * p.vn.s + h * p.vn.h;
        } else {
            const int t2 = t - n_k - n_v;
            kd = 2; h = t2 / ck; c = t2 - h * ck;
            srow[u] = static_cast<const T *>(p.q) + b * p.qs.b + i * p.qs.s + h * p.qs.h;
        }
        kind[u] = kd;
        head[u] = h;
        chunk[u] = c;
        raw[u] = __ldg(reinterpret_cast<const uint4 *>(srow[u]) + c);
        if (kd != 1 && chunk_partner && 8 * c < p.r) {
            const int pc = (8 * c < half) ? c + (half >> 3) : c - (half >> 3);
            praw[u] = __ldg(reinterpret_cast<const uint4 *>(srow[u]) + pc);
        }
    }

    const int L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
    // device-side preconditions: the new rows fit the cache and the table
    if (L < 0 || (int64_t)L + p.s_new > p.cap ||
        (p.r > 0 && (int64_t)L + rows > p.cs_rows)) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && i == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
        return;
    }
    const int64_t pos = (int64_t)L + i;
    if (p.r > 0) {
        const T *cos_row = static_cast<const T *>(p.cos) + pos * p.cs_row;
        const T *sin_row = static_cast<const T *>(p.sin) + pos * p.cs_row;
        for (int j = threadIdx.x; j < half; j += kRopeThreads) {
            cs_s[j] = Elem<T>::to_f(cos_row[j]);
            sn_s[j] = Elem<T>::to_f(sin_row[j]);
        }
    }
    __syncthreads();

#pragma unroll
    for (int u = 0; u < kRopeOps; ++u) {
        if (kind[u] < 0) continue;
        const int c = chunk[u], h = head[u];
        T *dst;
        if (kind[u] == 0)
            dst = static_cast<T *>(p.k_cache) + b * p.kc.b + pos * p.kc.s + h * p.kc.h;
        else if (kind[u] == 1)
            dst = static_cast<T *>(p.v_cache) + b * p.vc.b + pos * p.vc.s + h * p.vc.h;
        else
            dst = static_cast<T *>(p.q_rot) + (((int64_t)b * p.s_q + i) * p.h_q + h) * p.d_qk;
        const int t0 = 8 * c;
        if (kind[u] == 1 || t0 >= p.r) {
            reinterpret_cast<uint4 *>(dst)[c] = raw[u];   // unrotated dims: bit copy
            continue;
        }
        float f[8], pf[8];
        unpack8<T>(raw[u], f);
        if (t0 + 8 <= p.r && (inter || chunk_partner)) {
            // a whole chunk of pairs (the common case): straight-line code,
            // the chunk's cos/sin values read as float4 from shared memory
            float c8[8], s8[8];
            if (inter) {
                // pairs (2j, 2j+1), j = t0/2 .. t0/2 + 3
                const float4 cv = *reinterpret_cast<const float4 *>(cs_s + (t0 >> 1));
                const float4 sv = *reinterpret_cast<const float4 *>(sn_s + (t0 >> 1));
                c8[0] = c8[1] = cv.x; c8[2] = c8[3] = cv.y; c8[4] = c8[5] = cv.z; c8[6] = c8[7] = cv.w;
                s8[0] = s8[1] = sv.x; s8[2] = s8[3] = sv.y; s8[4] = s8[5] = sv.z; s8[6] = s8[7] = sv.w;
#pragma unroll
                for (int k = 0; k < 8; k += 2) {
                    const float a = f[k], b = f[k + 1];
                    f[k] = rope_elem(a, b, c8[k], s8[k], true);
                    f[k + 1] = rope_elem(b, a, c8[k], s8[k], false);
                }
            } else {
                // pairs (j, j + r/2): the chunk lies wholly in one half
                unpack8<T>(praw[u], pf);
                const bool first = t0 < half;
                const int j0 = first ? t0 : t0 - half;
                const float4 *cq = reinterpret_cast<const float4 *>(cs_s + j0);
                const float4 *sq = reinterpret_cast<const float4 *>(sn_s + j0);
                const float4 c0 = cq[0], c1 = cq[1], s0 = sq[0], s1 = sq[1];
                c8[0] = c0.x; c8[1] = c0.y; c8[2] = c0.z; c8[3] = c0.w;
                c8[4] = c1.x; c8[5] = c1.y; c8[6] = c1.z; c8[7] = c1.w;
                s8[0] = s0.x; s8[1] = s0.y; s8[2] = s0.z; s8[3] = s0.w;
                s8[4] = s1.x; s8[5] = s1.y; s8[6] = s1.z; s8[7] = s1.w;
                if (first) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) f[k] = rope_elem(f[k], pf[k], c8[k], s8[k], true);
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) f[k] = rope_elem(f[k], pf[k], c8[k], s8[k], false);
                }
            }
            reinterpret_cast<uint4 *>(dst)[c] = pack8<T>(f);
            continue;
        }
        if (inter) {
#pragma unroll
            for (int k = 0; k < 8; ++k) pf[k] = f[k ^ 1];
        } else if (chunk_partner) {
            unpack8<T>(praw[u], pf);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int t = t0 + k;
                const int partner = t < half ? t + half : t - half;
                pf[k] = t < p.r ? Elem<T>::to_f(srow[u][partner]) : 0.f;
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int t = t0 + k;
            if (t < p.r) {
                int partner, j;
                bool first;
                rope_pair_index(t, p.r, inter, partner, j, first);
                f[k] = rope_elem(f[k], pf[k], cs_s[j], sn_s[j], first);
            }
        }
        reinterpret_cast<uint4 *>(dst)[c] = pack8<T>(f);
    }
}

cudaError_t launch_rope_append(const RopeAppendParams &p, int dtype, cudaStream_t st) {
    const int rows = std::max(p.q_rot ? p.s_q : 0, p.s_new);
    const int64_t per_row = (int64_t)p.h_kv * (p.d_qk / 8 + p.d_v / 8) + (p.q_rot ? (int64_t)p.h_q * (p.d_qk / 8) : 0);
    const int64_t grid_x = (int64_t)p.b * std::max(rows, 1);
    if ((rows == 0 || p.b == 0) && !p.zero_word) return cudaSuccess;
    const int64_t grid_y = std::max<int64_t>(1, (per_row + kRopeOps * kRopeThreads - 1) / (kRopeOps * kRopeThreads));
    if (grid_x > 0x7fffffff || grid_y > 65535) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)std::max<int64_t>(grid_x, 1), (unsigned)grid_y);
    if (dtype == FA_DTYPE_F16)
        rope_append_kernel<__half><<<grid, kRopeThreads, 0, st>>>(p);
    else
        rope_append_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace fa
