// simt_attn.cu -- generic attention kernel on the CUDA cores.
//
// Covers every head-dim pair the ABI accepts (multiples of 8 up to 256) for
// shapes the specialised kernels do not take.  One warp per (batch, query
// head, query row); lanes score 32 keys at a time (online softmax in base 2,
// the softmax scale folded in) and then accumulate the value rows with each
// lane owning d_v / 32 output columns.  Keys come either from dense k/v
// (flash_attn_func of the "optimizing-attention-flash" page) or from the KV
// cache after the append kernel has written the new rows (the write precedes
// this launch on the same stream, as s2.cpp PR #40 requires).  Query rows
// are read already rotated.  Causal masking is aligned bottom-right.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

template <typename T>
__global__ void __launch_bounds__(256) simt_attn_kernel(const SimtAttnParams p) {
    extern __shared__ float sq_all[];
    const int warp_in_block = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t total = (int64_t)p.b * p.h_q * p.s_q;
    if (w >= total) return;
    const int i = (int)(w % p.s_q);
    const int hq = (int)((w / p.s_q) % p.h_q);
    const int b = (int)(w / ((int64_t)p.s_q * p.h_q));
    const int hk = hq / p.g;
    int64_t n_keys;
    if (p.seqlens != nullptr || p.cap > 0) {
        const int L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
        n_keys = (int64_t)L + p.s_new;
        if (L < 0 || n_keys > p.cap) {
            if (lane == 0 && i == 0 && hq == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
            return;
        }
    } else {
        n_keys = p.s_k;
    }
    int64_t first_vis, last_vis;
    visible_keys(i, n_keys, p.s_q, p.causal, p.win_left, p.win_right, first_vis, last_vis);
    const int64_t n_vis = max((int64_t)0, last_vis + 1);   // keys first_vis .. n_vis - 1

    float *sq = sq_all + warp_in_block * p.d_qk;
    const T *qrow = static_cast<const T *>(p.q) + b * p.qs.b + i * p.qs.s + hq * p.qs.h;
    for (int t = lane; t < p.d_qk; t += 32) sq[t] = Elem<T>::to_f(qrow[t]);
    __syncwarp();

    constexpr int MAXC = 8;  // d_v <= 256
    float acc[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) acc[c] = 0.f;
    float m = -INFINITY, l = 0.f;
    const T *kbase = static_cast<const T *>(p.k) + b * p.ks.b + hk * p.ks.h;
    const T *vbase = static_cast<const T *>(p.v) + b * p.vs.b + hk * p.vs.h;
    for (int64_t j0 = first_vis; j0 < n_vis; j0 += 32) {
        const int64_t j = j0 + lane;
        float s = -INFINITY;
        if (j < n_vis) {
            const T *krow = kbase + j * p.ks.s;
            float dot = 0.f;
            for (int t = 0; t < p.d_qk; t += 8) {
                float f[8];
                unpack8<T>(__ldg(reinterpret_cast<const uint4 *>(krow + t)), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) dot = fmaf(sq[t + e], f[e], dot);
            }
            s = dot * p.scale_log2;
        }
        float cm = s;
#pragma unroll
        for (int o = 16; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
        const float m_new = fmaxf(m, cm);
        const float corr = ex2(m - m_new);
        const float pj = ex2(s - m_new);
        float ps = pj;
#pragma unroll
        for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l = l * corr + ps;
#pragma unroll
        for (int c = 0; c < MAXC; ++c) acc[c] *= corr;
        m = m_new;
        const int cnt = (int)min((int64_t)32, n_vis - j0);
        for (int jj = 0; jj < cnt; ++jj) {
            const float pw = __shfl_sync(0xffffffffu, pj, jj);
            const T *vrow = vbase + (j0 + jj) * p.vs.s;
#pragma unroll
            for (int c = 0; c < MAXC; ++c) {
                const int col = lane + 32 * c;
                if (col < p.d_v) acc[c] = fmaf(pw, Elem<T>::to_f(vrow[col]), acc[c]);
            }
        }
    }
    T *orow = static_cast<T *>(p.out) + b * p.os.b + i * p.os.s + hq * p.os.h;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        const int col = lane + 32 * c;
        if (col < p.d_v) orow[col] = Elem<T>::from_f(acc[c] * inv);
    }
    if (lane == 0 && p.lse)
        p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
}

cudaError_t launch_simt_attn(const SimtAttnParams &p, int dtype, cudaStream_t st) {
    const int64_t warps = (int64_t)p.b * p.h_q * p.s_q;
    if (warps == 0) return cudaSuccess;
    const int64_t blocks = (warps * 32 + 255) / 256;
    const size_t smem = 8 * p.d_qk * sizeof(float);
    kernel_event(0, st);
    if (dtype == FA_DTYPE_F16)
        simt_attn_kernel<__half><<<(unsigned)blocks, 256, smem, st>>>(p);
    else
        simt_attn_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, smem, st>>>(p);
    const cudaError_t e = cudaGetLastError();
    kernel_event(1, st);
    return e;
}

}  // namespace fa
