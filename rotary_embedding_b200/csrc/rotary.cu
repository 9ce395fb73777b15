// rotary.cu -- standalone rotary embedding (the "non-fused" kernel of
// ROCm/flash-attention PR #99: COS/SIN (seqlen, rotary_dim/2), SEQLEN_OFFSET
// as an int or one value per batch entry, INTERLEAVED, CONJUGATE, IS_VARLEN).
//
// A block takes RT consecutive rows and HG heads (RT * HG * d / 8 <= 2048
// 16-byte chunks; HG < h only when one row's heads exceed that).  Its 256
// threads copy the chunks into shared memory with cp.async (no registers held
// while they are in flight) while the first RT threads find the rows'
// positions; after a barrier the block stages the cos/sin rows of those
// positions in shared memory as fp32 (one parallel round trip to L2, where
// the tables stay); after a second barrier every thread rotates its chunks
// from shared memory and stores them.  Every load precedes the barriers that
// precede every store, so out may be x itself.  CONJUGATE rotates by the negated angle (sin replaced by -sin).
// Positions: batched row i of entry b at offsets[b] + i; packed rows of
// sequence k (rows cu[k] .. cu[k+1]-1) at offsets[k] + R - cu[k].  Rows of a
// packed tensor outside every sequence are copied unchanged.
#include <algorithm>

#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

constexpr int kRotThreads = 256;
constexpr int kRotChunks = 2048;                       // 16-byte chunks per block (32 KB)
constexpr int kRotPer = kRotChunks / kRotThreads;       // chunks per thread
constexpr int kRotMaxRows = 16;                        // rows per block

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src)
                 : "memory");
}

// n / d for 0 <= n < 2^31 by a multiply-high and a shift (the round-up
// reciprocal method of Granlund and Montgomery, "Division by invariant
// integers using multiplication"): s = ceil(log2 d),
// m = floor(2^32 (2^s - d) / d) + 1, n / d = (mulhi(n, m) + n) >> s.
struct FastDiv {
    uint32_t d, m, s;
};
static FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    f.s = 0;
    while ((1u << f.s) < d) ++f.s;
    f.m = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << f.s) - d)) / d + 1);
    return f;
}
__device__ __forceinline__ int fdiv(int n, const FastDiv &f) {
    return (int)((__umulhi((uint32_t)n, f.m) + (uint32_t)n) >> f.s);
}

struct RotaryGrid {
    int RT, HG, per_row, total;
    FastDiv div_row, div_ck, div_s;
};

// Pairing: 0 interleaved; 1 half-split with rotary_dim/2 a multiple of 8 (the
// partner of a chunk is a chunk); 2 half-split otherwise (element partners).
template <typename T, int PAIR>
__global__ void __launch_bounds__(kRotThreads, 4) rotary_kernel(RotaryParams p, RotaryGrid g) {
    extern __shared__ uint4 sbuf[];                    // [kRotChunks]
    __shared__ int64_t pos_s[kRotMaxRows];
    __shared__ __align__(16) float cs_s[kRotMaxRows][128];
    __shared__ __align__(16) float sn_s[kRotMaxRows][128];
    const int tid = threadIdx.x;
    const int R0 = blockIdx.x * g.RT;
    const int h0 = blockIdx.y * g.HG;
    const int ck = p.d >> 3;
    const int half = p.r >> 1;
    constexpr bool inter = PAIR == 0;

    // the block's chunks into shared memory: chunk idx = (row r, head hl, chunk c)
    for (int idx = tid; idx < g.total; idx += kRotThreads) {
        const int r = fdiv(idx, g.div_row), rem = idx - r * g.per_row;
        const int hl = fdiv(rem, g.div_ck), c = rem - hl * ck;
        const int R = R0 + r, h = h0 + hl;
        if (R >= p.rows || h >= p.h) continue;
        const int rb = fdiv(R, g.div_s), ri = R - rb * p.s;
        const T *xrow = static_cast<const T *>(p.x) + rb * p.xs.b + ri * p.xs.s + (int64_t)h * p.xs.h;
        cp_async16(&sbuf[idx], reinterpret_cast<const uint4 *>(xrow) + c);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    // positions of the block's rows: -1 = outside every packed sequence (copy),
    // -2 = outside the table (left as it is)
    if (tid < g.RT) {
        const int R = R0 + tid;
        int64_t pos = -1;
        if (R < p.rows) {
            if (!p.cu_seqlens) {
                const int rb = fdiv(R, g.div_s), ri = R - rb * p.s;
                pos = (int64_t)(p.offsets ? __ldg(p.offsets + rb) : p.offset_scalar) + ri;
            } else if (R >= __ldg(p.cu_seqlens) && R < __ldg(p.cu_seqlens + p.n_seqs)) {
                int lo = 0, hi = p.n_seqs;   // cu[lo] <= R < cu[hi]
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (__ldg(p.cu_seqlens + mid) <= R) lo = mid; else hi = mid;
                }
                pos = (int64_t)(p.offsets ? __ldg(p.offsets + lo) : p.offset_scalar) + R - __ldg(p.cu_seqlens + lo);
            }
            if (p.r > 0 && pos != -1 && (pos < 0 || pos >= p.cs_rows)) {
                if (blockIdx.y == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
                pos = -2;
            }
        }
        pos_s[tid] = pos;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (p.r > 0) {
        const float sgn = p.conjugate ? -1.f : 1.f;
        for (int idx = tid; idx < g.RT * half; idx += kRotThreads) {
            const int r = idx / half, j = idx - r * half;
            const int64_t pos = pos_s[r];
            if (pos < 0) continue;
            cs_s[r][j] = Elem<T>::to_f(static_cast<const T *>(p.cos)[pos * p.cs_row + j]);
            sn_s[r][j] = sgn * Elem<T>::to_f(static_cast<const T *>(p.sin)[pos * p.cs_row + j]);
        }
    }
    __syncthreads();

    for (int idx = tid; idx < g.total; idx += kRotThreads) {
        const int r = fdiv(idx, g.div_row), rem = idx - r * g.per_row;
        const int hl = fdiv(rem, g.div_ck), c = rem - hl * ck;
        const int R = R0 + r, h = h0 + hl;
        if (R >= p.rows || h >= p.h) continue;
        const int64_t pos = pos_s[r];
        if (pos == -2) continue;
        const int rb = fdiv(R, g.div_s), ri = R - rb * p.s;
        T *orow = static_cast<T *>(p.out) + rb * p.os.b + ri * p.os.s + (int64_t)h * p.os.h;
        const uint4 raw = sbuf[idx];
        const int t0 = 8 * c;
        if (p.r == 0 || pos < 0 || t0 >= p.r) {
            reinterpret_cast<uint4 *>(orow)[c] = raw;   // unrotated dims: bit copy
            continue;
        }
        float f[8], q[8], cv[8], sv[8];
        unpack8<T>(raw, f);
        if (PAIR == 0) {
            // pairs (2j, 2j+1), j = t0/2 .. t0/2 + 3
            const float4 c4 = *reinterpret_cast<const float4 *>(&cs_s[r][t0 >> 1]);
            const float4 s4 = *reinterpret_cast<const float4 *>(&sn_s[r][t0 >> 1]);
            const float ca[4] = {c4.x, c4.y, c4.z, c4.w}, sa[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                q[k] = f[k ^ 1];
                cv[k] = ca[k >> 1];
                sv[k] = sa[k >> 1];
            }
        } else if (PAIR == 1) {
            // pairs (j, j + r/2): the chunk's angles are j0 .. j0 + 7
            const int pc = (t0 < half) ? c + (half >> 3) : c - (half >> 3);
            unpack8<T>(sbuf[idx - c + pc], q);
            const int j0 = t0 < half ? t0 : t0 - half;
            const float4 c0 = *reinterpret_cast<const float4 *>(&cs_s[r][j0]);
            const float4 c1 = *reinterpret_cast<const float4 *>(&cs_s[r][j0 + 4]);
            const float4 s0 = *reinterpret_cast<const float4 *>(&sn_s[r][j0]);
            const float4 s1 = *reinterpret_cast<const float4 *>(&sn_s[r][j0 + 4]);
            cv[0] = c0.x; cv[1] = c0.y; cv[2] = c0.z; cv[3] = c0.w;
            cv[4] = c1.x; cv[5] = c1.y; cv[6] = c1.z; cv[7] = c1.w;
            sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
            sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
        } else {
            const T *hrow = reinterpret_cast<const T *>(&sbuf[idx - c]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int t = t0 + k;
                const int tt = t < p.r ? t : 0;
                const int partner = tt < half ? tt + half : tt - half;
                const int j = tt < half ? tt : tt - half;
                q[k] = Elem<T>::to_f(hrow[partner]);
                cv[k] = cs_s[r][j];
                sv[k] = sn_s[r][j];
            }
        }
        const bool first_half = t0 < half;   // half-split: every element of the chunk on one side
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int t = t0 + k;
            if (t < p.r) {
                const bool first = PAIR == 0 ? (k & 1) == 0 : (PAIR == 1 ? first_half : t < half);
                f[k] = rope_elem(f[k], q[k], cv[k], sv[k], first);
            }
        }
        reinterpret_cast<uint4 *>(orow)[c] = pack8<T>(f);
    }
}

cudaError_t launch_rotary(const RotaryParams &p, int dtype, cudaStream_t st) {
    if (p.rows == 0 || p.h == 0) return cudaSuccess;
    const int ck = p.d / 8;
    RotaryGrid g;
    g.HG = std::min(p.h, std::max(1, kRotChunks / ck));   // heads per block
    g.RT = std::max(1, std::min(kRotMaxRows, kRotChunks / (g.HG * ck)));
    g.per_row = g.HG * ck;
    g.total = g.RT * g.per_row;
    g.div_row = make_fastdiv((uint32_t)g.per_row);
    g.div_ck = make_fastdiv((uint32_t)ck);
    g.div_s = make_fastdiv((uint32_t)std::max(p.s, 1));
    const int64_t gx = (p.rows + g.RT - 1) / g.RT;
    const int64_t gy = (p.h + g.HG - 1) / g.HG;
    // rows are indexed with 32-bit arithmetic in the kernel (fdiv needs < 2^31)
    if (p.rows > 0x7fffffff - kRotMaxRows || gx > 0x7fffffff || gy > 65535) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)gx, (unsigned)gy);
    const size_t smem = (size_t)kRotChunks * 16;
    const int pair = p.interleaved ? 0 : ((p.r / 2) % 8 == 0 ? 1 : 2);
    kernel_event(0, st);
#define FA_ROT_LAUNCH(T, P)                                                                              \
    do {                                                                                                 \
        cudaFuncSetAttribute(rotary_kernel<T, P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        rotary_kernel<T, P><<<grid, kRotThreads, smem, st>>>(p, g);                                      \
    } while (0)
    if (dtype == FA_DTYPE_F16) {
        if (pair == 0) FA_ROT_LAUNCH(__half, 0); else if (pair == 1) FA_ROT_LAUNCH(__half, 1); else FA_ROT_LAUNCH(__half, 2);
    } else {
        if (pair == 0) FA_ROT_LAUNCH(__nv_bfloat16, 0);
        else if (pair == 1) FA_ROT_LAUNCH(__nv_bfloat16, 1);
        else FA_ROT_LAUNCH(__nv_bfloat16, 2);
    }
#undef FA_ROT_LAUNCH
    const cudaError_t e = cudaGetLastError();
    kernel_event(1, st);
    return e;
}

}  // namespace fa
