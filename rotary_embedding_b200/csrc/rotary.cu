// rotary.cu -- standalone rotary embedding (the "non-fused" kernel of
// ROCm/flash-attention PR #99: COS/SIN (seqlen, rotary_dim/2), SEQLEN_OFFSET
// as an int or one value per batch entry, INTERLEAVED, CONJUGATE, IS_VARLEN).
//
// A pure stream: every thread takes one unit of up to four heads of one row
// -- with half-split pairs a 16-byte chunk of the first half and its partner
// chunk rotary_dim/2 further on, with interleaved pairs one chunk holding
// four pairs -- issues the 16-byte loads of all those heads at once, reads
// the row's cos/sin values once for them (a few hundred bytes per row,
// served from L1/L2), rotates in fp32 with the shared RoPE pair formula,
// rounds, and stores.  There is no staging and no block-wide barrier; one
// wave of resident blocks walks the items with a grid-stride loop, each
// thread keeping up to 128 bytes of loads in flight.  Dims past rotary_dim are
// copied (out of place) or left untouched (in place, out = x).  CONJUGATE
// rotates by the negated angle (sin replaced by -sin).  Positions: batched
// row i of entry b at offsets[b] + i; packed rows of sequence k (rows
// cu[k] .. cu[k+1]-1) at offsets[k] + R - cu[k] (the sequence found by
// binary search); rows of a packed tensor outside every sequence are copied
// unchanged; a row whose position falls outside the table is left as it is
// and the device status records it.
#include <algorithm>

#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

constexpr int kRotThreads = 256;

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

// Units of a (row, head): MODE 0 interleaved (chunk c, four pairs; then the
// chunks past rotary_dim), MODE 1 half-split with rotary_dim/2 a multiple of
// 8 (chunk c < r/16 and its partner; then the chunks past rotary_dim), MODE 2
// half-split otherwise (pair j < r/2, i.e. elements j and j + r/2, one by
// one; then the elements past rotary_dim).  Every unit owns what it writes,
// so out may be x.
struct RotaryGrid {
    int units;            // units per (row, head)
    int rot_units;        // units that rotate (the rest copy)
    int copy_from;        // MODE 1: first chunk of the copied dims
    int in_place;         // out == x: copy units are skipped
    int cs_vec;           // cos/sin rows 16-byte aligned: vector loads
    FastDiv div_units, div_h, div_s;
};

// Table row of packed / batched row R (kOutside: a packed row outside every
// sequence).
constexpr int64_t kOutside = INT64_MIN;
__device__ __forceinline__ int64_t row_position(const RotaryParams &p, const RotaryGrid &g, int R) {
    if (!p.cu_seqlens) {
        const int rb = fdiv(R, g.div_s), ri = R - rb * p.s;
        return (int64_t)(p.offsets ? __ldg(p.offsets + rb) : p.offset_scalar) + ri;
    }
    if (R < __ldg(p.cu_seqlens) || R >= __ldg(p.cu_seqlens + p.n_seqs)) return kOutside;
    int lo = 0, hi = p.n_seqs;   // cu[lo] <= R < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.cu_seqlens + mid) <= R) lo = mid; else hi = mid;
    }
    return (int64_t)(p.offsets ? __ldg(p.offsets + lo) : p.offset_scalar) + R - __ldg(p.cu_seqlens + lo);
}

// NV consecutive table values from column j0 of a row, as fp32 times
// `sign` (-1 for the conjugate); columns at or past `ncols` read as 0.
template <typename T, int NV>
__device__ __forceinline__ void table_vals(const T *row, int j0, int ncols, bool vec, float sign, float *v) {
    if (NV == 8 && vec && j0 + 8 <= ncols) {
        float f[8];
        unpack8<T>(__ldg(reinterpret_cast<const uint4 *>(row + j0)), f);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = sign * f[k];
    } else {
#pragma unroll
        for (int k = 0; k < NV; ++k) v[k] = j0 + k < ncols ? sign * Elem<T>::to_f(row[j0 + k]) : 0.f;
    }
}

// One item = unit u of heads hg HU .. hg HU + HU - 1 of row R: the heads
// share the row's position and cos/sin values, and the thread issues the
// 16-byte loads of all its heads before it waits on any of them (HU x 32
// bytes in flight per thread in MODE 1).
template <typename T, int MODE, int HU>
__global__ void __launch_bounds__(kRotThreads) rotary_kernel(RotaryParams p, RotaryGrid g) {
    const int n_hg = p.h / HU;
    const int64_t total = (int64_t)p.rows * n_hg * g.units;
    for (int64_t item = (int64_t)blockIdx.x * kRotThreads + threadIdx.x; item < total;
         item += (int64_t)gridDim.x * kRotThreads) {
        const int it = (int)item;   // total < 2^31 (checked at launch)
        const int rh = fdiv(it, g.div_units), u = it - rh * g.units;
        const int R = fdiv(rh, g.div_h), h0 = (rh - R * n_hg) * HU;
        const bool rot = u < g.rot_units && p.r > 0;
        if (!rot && g.in_place) continue;   // dims past rotary_dim stay as they are
        const int rb = fdiv(R, g.div_s), ri = R - rb * p.s;
        const T *xrow0 = static_cast<const T *>(p.x) + rb * p.xs.b + ri * p.xs.s + (int64_t)h0 * p.xs.h;
        T *orow0 = static_cast<T *>(p.out) + rb * p.os.b + ri * p.os.s + (int64_t)h0 * p.os.h;
        int64_t pos = 0;
        if (p.r > 0) {
            pos = row_position(p, g, R);
            if (pos != kOutside && (pos < 0 || pos >= p.cs_rows)) {
                if (h0 == 0 && u == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
                continue;                      // the whole row is left as it is
            }
        }
        if (!rot || pos == kOutside) {
            // copied chunks: past rotary_dim, or a packed row outside every sequence
#pragma unroll
            for (int k = 0; k < HU; ++k) {
                const T *xrow = xrow0 + (int64_t)k * p.xs.h;
                T *orow = orow0 + (int64_t)k * p.os.h;
                if (MODE == 1) {
                    if (!rot) {
                        const int c = g.copy_from + (u - g.rot_units);
                        reinterpret_cast<uint4 *>(orow)[c] = __ldg(reinterpret_cast<const uint4 *>(xrow) + c);
                    } else if (!g.in_place) {
                        const int c0 = u, c1 = u + (p.r >> 4);
                        reinterpret_cast<uint4 *>(orow)[c0] = __ldg(reinterpret_cast<const uint4 *>(xrow) + c0);
                        reinterpret_cast<uint4 *>(orow)[c1] = __ldg(reinterpret_cast<const uint4 *>(xrow) + c1);
                    }
                } else if (MODE == 2) {
                    if (!rot) {
                        const int t = p.r + (u - g.rot_units);
                        orow[t] = xrow[t];
                    } else if (!g.in_place) {
                        orow[u] = xrow[u];
                        orow[u + (p.r >> 1)] = xrow[u + (p.r >> 1)];
                    }
                } else if (!g.in_place) {
                    const int c = rot ? u : g.copy_from + (u - g.rot_units);
                    reinterpret_cast<uint4 *>(orow)[c] = __ldg(reinterpret_cast<const uint4 *>(xrow) + c);
                }
            }
            continue;
        }
        const T *crow = static_cast<const T *>(p.cos) + pos * p.cs_row;
        const T *srow = static_cast<const T *>(p.sin) + pos * p.cs_row;
        const float sgn = p.conjugate ? -1.f : 1.f;
        if (MODE == 1) {
            // pairs (j, j + r/2): chunk u of the first half and its partner
            const int half = p.r >> 1;
            const int c0 = u, c1 = u + (half >> 3);
            uint4 ra[HU], rb2[HU];
#pragma unroll
            for (int k = 0; k < HU; ++k) {
                const uint4 *xr = reinterpret_cast<const uint4 *>(xrow0 + (int64_t)k * p.xs.h);
                ra[k] = __ldg(xr + c0);
                rb2[k] = __ldg(xr + c1);
            }
            float cs[8], sn[8];
            table_vals<T, 8>(crow, 8 * u, half, g.cs_vec, 1.f, cs);
            table_vals<T, 8>(srow, 8 * u, half, g.cs_vec, sgn, sn);
#pragma unroll
            for (int k = 0; k < HU; ++k) {
                float a[8], b[8], ya[8], yb[8];
                unpack8<T>(ra[k], a);
                unpack8<T>(rb2[k], b);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    ya[e] = rope_elem(a[e], b[e], cs[e], sn[e], true);
                    yb[e] = rope_elem(b[e], a[e], cs[e], sn[e], false);
                }
                uint4 *orow = reinterpret_cast<uint4 *>(orow0 + (int64_t)k * p.os.h);
                orow[c0] = pack8<T>(ya);
                orow[c1] = pack8<T>(yb);
            }
        } else if (MODE == 0) {
            // pairs (2j, 2j+1) inside chunk u: angles 4u .. 4u+3
            uint4 rx[HU];
#pragma unroll
            for (int k = 0; k < HU; ++k) rx[k] = __ldg(reinterpret_cast<const uint4 *>(xrow0 + (int64_t)k * p.xs.h) + u);
            float cs[4], sn[4];
            table_vals<T, 4>(crow, 4 * u, p.r >> 1, false, 1.f, cs);
            table_vals<T, 4>(srow, 4 * u, p.r >> 1, false, sgn, sn);
#pragma unroll
            for (int k = 0; k < HU; ++k) {
                float f[8], y[8];
                unpack8<T>(rx[k], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 8 * u + e;
                    y[e] = t < p.r ? rope_elem(f[e], f[e ^ 1], cs[e >> 1], sn[e >> 1], (e & 1) == 0) : f[e];
                }
                reinterpret_cast<uint4 *>(orow0 + (int64_t)k * p.os.h)[u] = pack8<T>(y);
            }
        } else {
            // half-split with rotary_dim/2 not a multiple of 8: pair u, elements u and u + r/2
            const int half = p.r >> 1;
            const float cs = Elem<T>::to_f(crow[u]), sn = sgn * Elem<T>::to_f(srow[u]);
#pragma unroll
            for (int k = 0; k < HU; ++k) {
                const T *xrow = xrow0 + (int64_t)k * p.xs.h;
                T *orow = orow0 + (int64_t)k * p.os.h;
                const float a = Elem<T>::to_f(xrow[u]), b = Elem<T>::to_f(xrow[u + half]);
                orow[u] = Elem<T>::from_f(rope_elem(a, b, cs, sn, true));
                orow[u + half] = Elem<T>::from_f(rope_elem(b, a, cs, sn, false));
            }
        }
    }
}

template <typename T, int MODE, int HU>
static cudaError_t run_rotary(const RotaryParams &p, const RotaryGrid &g, int64_t total, cudaStream_t st) {
    // one wave of resident blocks; the grid-stride loop covers the rest
    static int per_sm = 0;
    if (per_sm == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotary_kernel<T, MODE, HU>,
                                                                      kRotThreads, 0);
        if (e != cudaSuccess || per_sm < 1) per_sm = 1;
    }
    const int64_t want = (total + kRotThreads - 1) / kRotThreads;
    const int64_t wave = (int64_t)sm_count() * per_sm;
    dim3 grid((unsigned)std::min(want, wave));
    kernel_event(0, st);
    rotary_kernel<T, MODE, HU><<<grid, kRotThreads, 0, st>>>(p, g);
    const cudaError_t e = cudaGetLastError();
    kernel_event(1, st);
    return e;
}

template <typename T, int MODE>
static cudaError_t run_rotary_hu(const RotaryParams &p, RotaryGrid &g, cudaStream_t st) {
    const int hu = p.h % 4 == 0 ? 4 : (p.h % 2 == 0 ? 2 : 1);
    g.div_h = make_fastdiv((uint32_t)(p.h / hu));
    const int64_t total = (int64_t)p.rows * (p.h / hu) * g.units;
    if (total == 0) return cudaSuccess;
    // item indices are 32-bit in the kernel (fdiv needs < 2^31)
    if (total > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (hu == 4) return run_rotary<T, MODE, 4>(p, g, total, st);
    if (hu == 2) return run_rotary<T, MODE, 2>(p, g, total, st);
    return run_rotary<T, MODE, 1>(p, g, total, st);
}

cudaError_t launch_rotary(const RotaryParams &p, int dtype, cudaStream_t st) {
    if (p.rows == 0 || p.h == 0) return cudaSuccess;
    const int ck = p.d / 8;
    const int half = p.r / 2;
    // rotary_dim 0 (a plain copy) takes the chunk units of MODE 0
    const int mode = (p.interleaved || p.r == 0) ? 0 : (half % 8 == 0 ? 1 : 2);
    RotaryGrid g;
    g.in_place = p.out == p.x;
    if (mode == 1) {
        g.rot_units = half / 8;
        g.copy_from = p.r / 8;
        g.units = g.rot_units + (ck - g.copy_from);
    } else if (mode == 0) {
        g.rot_units = p.r > 0 ? (p.r + 7) / 8 : 0;
        g.copy_from = g.rot_units;
        g.units = ck;
    } else {
        g.rot_units = half;           // pairs
        g.copy_from = p.r;            // elements past rotary_dim
        g.units = half + (p.d - p.r);
    }
    const int elem = 2;
    g.cs_vec = p.cos && (reinterpret_cast<uintptr_t>(p.cos) % 16 == 0) &&
               (reinterpret_cast<uintptr_t>(p.sin) % 16 == 0) && ((p.cs_row * elem) % 16 == 0);
    g.div_units = make_fastdiv((uint32_t)std::max(g.units, 1));
    g.div_s = make_fastdiv((uint32_t)std::max(p.s, 1));
    if (dtype == FA_DTYPE_F16) {
        if (mode == 0) return run_rotary_hu<__half, 0>(p, g, st);
        if (mode == 1) return run_rotary_hu<__half, 1>(p, g, st);
        return run_rotary_hu<__half, 2>(p, g, st);
    }
    if (mode == 0) return run_rotary_hu<__nv_bfloat16, 0>(p, g, st);
    if (mode == 1) return run_rotary_hu<__nv_bfloat16, 1>(p, g, st);
    return run_rotary_hu<__nv_bfloat16, 2>(p, g, st);
}

}  // namespace fa
