// fa_common.cuh -- device helpers shared by the sm_100a kernels of libfa.so:
// element conversion, the RoPE pair rotation, swizzled shared-memory
// addressing, mbarrier / TMA / ldmatrix / mma.sync PTX wrappers and the
// bounded waits that keep a kernel from spinning forever.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "fa.h"

namespace fa {

// ----------------------------------------------------------------------------
// Device status word: kernels record precondition failures and bounded-wait
// timeouts in the word `status` points to (first error wins);
// fa_device_status() reads and clears it.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void record_status(int32_t *status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

// ----------------------------------------------------------------------------
// Element types.
// ----------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<__half> {
    static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
    static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

// Unpack 8 elements held in a 16-byte vector into floats.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    const T *e = reinterpret_cast<const T *>(&v);
#pragma unroll
    for (int t = 0; t < 8; ++t) f[t] = Elem<T>::to_f(e[t]);
}
template <typename T>
__device__ __forceinline__ uint4 pack8(const float *f) {
    uint4 v;
    v.x = Elem<T>::pack2(f[0], f[1]);
    v.y = Elem<T>::pack2(f[2], f[3]);
    v.z = Elem<T>::pack2(f[4], f[5]);
    v.w = Elem<T>::pack2(f[6], f[7]);
    return v;
}

// ----------------------------------------------------------------------------
// RoPE of element t of a row (RoFormer rotation as used by flash_attn's
// rotary path: the pair (a, b) becomes (a c - b s, a s + b c)).  `x` is the
// whole row in fp32, r the rotary dim.  Half-split pairs are (j, j + r/2),
// interleaved pairs (2j, 2j+1).  Every kernel that rotates uses this one
// function, so a rotated key written to the cache and the same key used
// inside attention are bit-identical.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void rope_pair_index(int t, int r, bool interleaved, int &partner,
                                                int &j, bool &first) {
    if (interleaved) {
        j = t >> 1;
        first = (t & 1) == 0;
        partner = t ^ 1;
    } else {
        int half = r >> 1;
        first = t < half;
        j = first ? t : t - half;
        partner = first ? t + half : t - half;
    }
}

__device__ __forceinline__ float rope_elem(float self, float partner, float c, float s, bool first) {
    // first element of the pair: a c - b s ; second: b c + a s (b = self)
    return first ? fmaf(self, c, -partner * s) : fmaf(self, c, partner * s);
}

// ----------------------------------------------------------------------------
// Swizzled shared-memory tiles.  A tile of `rows` rows x d columns is stored
// as d / CH boxes of [rows][CH] elements (CH = min(d, 64) 16-bit elements,
// i.e. 32, 64 or 128 bytes per row), each box written by one TMA copy with
// the matching swizzle mode.  The swizzle XORs the 16-byte chunk index with
// bits 7.. of the byte offset inside the box: off ^ (((off >> 7) & mask) << 4)
// with mask = row_bytes / 16 - 1.
// ----------------------------------------------------------------------------
__host__ __device__ constexpr int box_cols(int d) { return d < 64 ? d : 64; }
__host__ __device__ constexpr int box_row_bytes(int d) { return box_cols(d) * 2; }
__host__ __device__ constexpr int swz_mask(int d) { return box_row_bytes(d) / 16 - 1; }

// Byte offset of element (row, col) in a tile with `rows` rows per box.
template <int D>
__device__ __forceinline__ uint32_t swz_offset(int row, int col, int rows) {
    constexpr int CH = box_cols(D);
    constexpr int RB = box_row_bytes(D);
    constexpr int MASK = swz_mask(D);
    uint32_t off = (uint32_t)((col / CH) * rows * RB + row * RB + (col % CH) * 2);
    return off ^ (((off >> 7) & MASK) << 4);
}

// ----------------------------------------------------------------------------
// PTX wrappers.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after roughly
// two seconds of SM clock; on give-up the device status records a timeout
// and the function returns false so the caller can leave its loop.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    long long start = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - start > 4000000000LL) {
            record_status(status, FA_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled TMA load into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

// L2 policy for data read exactly once: its lines are the first to go, so a
// stream larger than L2 does not evict what was written or read around it.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// tma_load_4d with an L2 cache policy (from createpolicy).
__device__ __forceinline__ void tma_load_4d_hint(void *dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                                 int c1, int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "l"(policy)
        : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                            uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                                  uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

template <typename T> struct Mma;
template <> struct Mma<__half> {
    static __device__ __forceinline__ void run(float *d, const uint32_t *a, uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};
template <> struct Mma<__nv_bfloat16> {
    static __device__ __forceinline__ void run(float *d, const uint32_t *a, uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32); ex2(-inf) = +0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (sm_100 FFMA2 / FADD2: two fp32 operations per lane and
// per issued instruction) and the three-input max.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for a pair of values on the FMA / integer pipes, leaving the special
// function unit free (Cody-Waite reduction x = n + f, n = round(x),
// f in [-1/2, 1/2]; 2^f by a degree-3 minimax polynomial whose coefficients
// exp2_poly.py derives by the Remez exchange; 2^n added to the exponent
// field).  Maximum relative error 7.5e-5.  x is clamped to >= -126 first, so
// very negative inputs give a result in [0, 2^-125] instead of exactly 0;
// callers that need exact zeros (masked scores) use ex2().
__device__ __forceinline__ uint64_t ex2_poly2(float x0, float x1) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: x + kMagic rounds x to an integer
    x0 = fmaxf(x0, -126.0f);
    x1 = fmaxf(x1, -126.0f);
    const uint64_t x = f2_pack(x0, x1);
    const uint64_t t = f2_add(x, f2_pack(kMagic, kMagic));
    const uint64_t n = f2_add(t, f2_pack(-kMagic, -kMagic));
    const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), x);           // x - n
    uint64_t p = f2_fma(f2_pack(0.0551716685295105f, 0.0551716685295105f), f,
                        f2_pack(0.2426111251115799f, 0.2426111251115799f));
    p = f2_fma(p, f, f2_pack(0.6932609677314758f, 0.6932609677314758f));
    p = f2_fma(p, f, f2_pack(0.9999280571937561f, 0.9999280571937561f));
    // the low bits of t hold n (two's complement); shift it into the exponent
    const uint32_t t_lo = static_cast<uint32_t>(t), t_hi = static_cast<uint32_t>(t >> 32);
    const uint32_t p_lo = static_cast<uint32_t>(p), p_hi = static_cast<uint32_t>(p >> 32);
    const uint32_t r_lo = p_lo + (t_lo << 23), r_hi = p_hi + (t_hi << 23);
    return (static_cast<uint64_t>(r_hi) << 32) | r_lo;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace fa

namespace fa {

// ----------------------------------------------------------------------------
// Load elements [8c, 8c+8) of one row of head dim d and apply RoPE at the
// table row given by cos_row / sin_row (rotary dim r, 0 = none).  The row
// and the table rows are in global memory; the row start is 16-byte
// aligned.  Result in fp32, not yet rounded to the element type.
// ----------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void load_rotated_chunk(const T *row, int c, int r, bool interleaved,
                                                   const T *cos_row, const T *sin_row, float *f) {
    uint4 v = __ldg(reinterpret_cast<const uint4 *>(row + 8 * c));
    unpack8<T>(v, f);
    const int t0 = 8 * c;
    if (t0 >= r) return;
    float pf[8];
    if (interleaved) {
#pragma unroll
        for (int k = 0; k < 8; ++k) pf[k] = f[k ^ 1];
    } else {
        const int half = r >> 1;
        if ((half & 7) == 0) {
            const int pc = (t0 < half) ? c + (half >> 3) : c - (half >> 3);
            uint4 pv = __ldg(reinterpret_cast<const uint4 *>(row + 8 * pc));
            unpack8<T>(pv, pf);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                int t = t0 + k;
                int partner = t < half ? t + half : t - half;
                pf[k] = t < r ? Elem<T>::to_f(row[partner]) : 0.f;
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        int t = t0 + k;
        if (t < r) {
            int partner, j;
            bool first;
            rope_pair_index(t, r, interleaved, partner, j, first);
            float cs = Elem<T>::to_f(cos_row[j]);
            float sn = Elem<T>::to_f(sin_row[j]);
            f[k] = rope_elem(f[k], pf[k], cs, sn, first);
        }
    }
}

// cache_seqlens[b], or the scalar form.
__device__ __forceinline__ int seqlen_of(const int32_t *seqlens, int32_t scalar, int b) {
    return seqlens ? __ldg(seqlens + b) : scalar;
}

}  // namespace fa
