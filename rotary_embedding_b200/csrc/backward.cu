// Attention backward: dq, dk, dv of out = softmax(scale q k^T + mask) v for a
// given dout, with d_qk != d_v allowed (flash-attention PR #1604 "Support
// hdimQK != hdimV backward": DeepSeek's 192/128), GQA, and the causal /
// sliding-window masks of the forward (aligned bottom-right).
//
// P is recomputed from the forward's lse, P_ij = exp(scale q_i.k_j - lse_i),
// and the softmax Jacobian's row term is D_i = dout_i . out_i, which equals
// sum_j P_ij dP_ij because out_i = sum_j P_ij v_j:
//   dv_j = sum_i P_ij dout_i          dP_ij = dout_i . v_j
//   dS_ij = P_ij (dP_ij - D_i)
//   dk_j = scale sum_i dS_ij q_i      dq_i = scale sum_j dS_ij k_j
// (a kv head's dk and dv sum over the query heads of its group).
//
// Three kernels, no atomics, no waits between CTAs (the result does not
// depend on scheduling):
//  - bwd_dot_kernel: D_i, one warp per (batch, row, query head).
//  - bwd_dkdv_kernel: one CTA per 64 keys of a (batch, kv head).  Its four
//    warps own 16 keys each and walk the query tiles, of every query head of
//    the group, that see any of those keys.  They form S^T = K Q^T and
//    dP^T = V dO^T, so that P^T and dS^T leave the accumulators in the
//    register layout the next products take as their A operand:
//    dV += P^T dO and dK += dS^T Q.  dk and dv are written once, at the end.
//  - bwd_dq_kernel: one CTA per 64 query rows of a (batch, query head); its
//    warps own 16 rows each and walk the key tiles those rows see:
//    S = Q K^T, dP = dO V^T, dQ += dS K.  (S and dP are formed twice, once
//    per kernel: the price of writing dq without atomics.)
// Products run on mma.sync m16n8k16 with fp32 accumulation; P and dS are
// rounded to the element type as MMA operands.  Tiles are staged in shared
// memory with cp.async (two buffers), in the swizzled layout of swz_offset so
// that ldmatrix reads are free of bank conflicts; rows past the sequence are
// zero-filled.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBwdThreads = 128;  // four warps
constexpr int kKeysPerCta = 64;   // dk/dv kernel: 16 keys per warp
constexpr int kRowsPerCta = 64;   // dq kernel: 16 query rows per warp
constexpr int kDqBK = 32;         // dq kernel: keys per staged K/V tile

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Stage rows 0 .. ROWS-1 of a [rows][D] tile (row r at g + r * stride) into
// the swizzled tile at `tile`; rows >= valid are zero-filled.
template <typename T, int D, int ROWS>
__device__ __forceinline__ void stage_rows(char *tile, const T *g, int64_t stride, int valid, int tid) {
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    for (int idx = tid; idx < ROWS * CPR; idx += kBwdThreads) {
        const int r = idx / CPR, c = idx % CPR;
        char *dst = tile + swz_offset<D>(r, c * 8, ROWS);
        if (r < valid)
            cp_async16(dst, g + r * stride + c * 8);
        else
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
}

// acc[0 .. N8) += A (16 x K, rows of tile a at row a0) * B^T where B is the
// tile b (rows b0 .. b0 + 8*N8 - 1, K columns): the product of two row-major
// tiles over their shared column dimension (Q K^T, K Q^T, dO V^T, V dO^T).
template <typename T, int K, int AROWS, int BROWS, int N8>
__device__ __forceinline__ void mma_rows_rows(float (*acc)[4], uint32_t a_tile, int a0, uint32_t b_tile, int b0,
                                              int lane) {
#pragma unroll
    for (int kk = 0; kk < K / 16; ++kk) {
        uint32_t a[4];
        ldmatrix_x4(a_tile + swz_offset<K>(a0 + (lane & 15), kk * 16 + ((lane >> 4) << 3), AROWS), a[0], a[1], a[2],
                    a[3]);
#pragma unroll
        for (int n2 = 0; n2 < N8 / 2; ++n2) {
            uint32_t b[4];
            ldmatrix_x4(b_tile + swz_offset<K>(b0 + n2 * 16 + (lane & 7) + ((lane >> 4) << 3),
                                               kk * 16 + (((lane >> 3) & 1) << 3), BROWS),
                        b[0], b[1], b[2], b[3]);
            Mma<T>::run(acc[2 * n2], a, b[0], b[1]);
            Mma<T>::run(acc[2 * n2 + 1], a, b[2], b[3]);
        }
    }
}

// Two independent mma_rows_rows products (S and dP) interleaved in one
// k-loop, so that twice as many accumulators are in flight per warp.
template <typename T, int K1, int K2, int AROWS, int BROWS, int N8>
__device__ __forceinline__ void mma_rows_rows2(float (*acc1)[4], uint32_t a1_tile, uint32_t b1_tile,
                                               float (*acc2)[4], uint32_t a2_tile, uint32_t b2_tile, int a0,
                                               int lane) {
    constexpr int KS = (K1 > K2 ? K1 : K2) / 16;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        if (kk < K1 / 16) {
            uint32_t a[4];
            ldmatrix_x4(a1_tile + swz_offset<K1>(a0 + (lane & 15), kk * 16 + ((lane >> 4) << 3), AROWS), a[0], a[1],
                        a[2], a[3]);
#pragma unroll
            for (int n2 = 0; n2 < N8 / 2; ++n2) {
                uint32_t b[4];
                ldmatrix_x4(b1_tile + swz_offset<K1>(n2 * 16 + (lane & 7) + ((lane >> 4) << 3),
                                                     kk * 16 + (((lane >> 3) & 1) << 3), BROWS),
                            b[0], b[1], b[2], b[3]);
                Mma<T>::run(acc1[2 * n2], a, b[0], b[1]);
                Mma<T>::run(acc1[2 * n2 + 1], a, b[2], b[3]);
            }
        }
        if (kk < K2 / 16) {
            uint32_t a[4];
            ldmatrix_x4(a2_tile + swz_offset<K2>(a0 + (lane & 15), kk * 16 + ((lane >> 4) << 3), AROWS), a[0], a[1],
                        a[2], a[3]);
#pragma unroll
            for (int n2 = 0; n2 < N8 / 2; ++n2) {
                uint32_t b[4];
                ldmatrix_x4(b2_tile + swz_offset<K2>(n2 * 16 + (lane & 7) + ((lane >> 4) << 3),
                                                     kk * 16 + (((lane >> 3) & 1) << 3), BROWS),
                            b[0], b[1], b[2], b[3]);
                Mma<T>::run(acc2[2 * n2], a, b[0], b[1]);
                Mma<T>::run(acc2[2 * n2 + 1], a, b[2], b[3]);
            }
        }
    }
}

// acc[0 .. D/8) += X (16 x KR, given as accumulator fragments x[KR/8][4]) *
// tile (rows 0 .. KR-1, D columns): X's columns contract with the tile's
// rows (P^T dO, dS^T Q, dS K).
template <typename T, int D, int KR, int ROWS>
__device__ __forceinline__ void mma_frag_rows(float (*acc)[4], const float (*x)[4], uint32_t tile, int lane) {
#pragma unroll
    for (int kq = 0; kq < KR / 16; ++kq) {
        uint32_t a[4];
        a[0] = Elem<T>::pack2(x[2 * kq][0], x[2 * kq][1]);
        a[1] = Elem<T>::pack2(x[2 * kq][2], x[2 * kq][3]);
        a[2] = Elem<T>::pack2(x[2 * kq + 1][0], x[2 * kq + 1][1]);
        a[3] = Elem<T>::pack2(x[2 * kq + 1][2], x[2 * kq + 1][3]);
#pragma unroll
        for (int nn = 0; nn < D / 16; ++nn) {
            uint32_t b[4];
            ldmatrix_x4_trans(tile + swz_offset<D>(kq * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                                                   nn * 16 + ((lane >> 4) << 3), ROWS),
                              b[0], b[1], b[2], b[3]);
            Mma<T>::run(acc[2 * nn], a, b[0], b[1]);
            Mma<T>::run(acc[2 * nn + 1], a, b[2], b[3]);
        }
    }
}

// Store a warp's 16 x D accumulator block (rows row0 + 0..15, scaled by
// `mul`) as element-type rows at g + row * stride; rows >= valid are skipped.
template <typename T, int D>
__device__ __forceinline__ void store_rows(T *g, int64_t stride, const float (*acc)[4], int row0, int valid,
                                           float mul, int lane) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int r = row0 + (lane >> 2) + hr * 8;
        if (r >= valid) continue;
        T *dst = g + r * stride + ((lane & 3) << 1);
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<uint32_t *>(dst + n * 8) =
                Elem<T>::pack2(acc[n][hr * 2] * mul, acc[n][hr * 2 + 1] * mul);
    }
}

// ---------------------------------------------------------------- D_i
template <typename T>
__global__ void __launch_bounds__(256) bwd_dot_kernel(const BwdParams p) {
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.b * p.s_q * p.h_q;
    if (w >= rows) return;
    const int h = (int)(w % p.h_q);
    const int64_t bi_i = w / p.h_q;
    const int i = (int)(bi_i % p.s_q), bi = (int)(bi_i / p.s_q);
    const T *o = static_cast<const T *>(p.out) + bi * p.os.b + (int64_t)i * p.os.s + h * p.os.h;
    const T *d = static_cast<const T *>(p.dout) + bi * p.dos.b + (int64_t)i * p.dos.s + h * p.dos.h;
    float acc = 0.f;
    for (int t = lane * 2; t < p.d_v; t += 64)
        acc += Elem<T>::to_f(o[t]) * Elem<T>::to_f(d[t]) + Elem<T>::to_f(o[t + 1]) * Elem<T>::to_f(d[t + 1]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) p.dsum[((int64_t)bi * p.h_q + h) * p.s_q + i] = acc;
}

// ---------------------------------------------------------------- dk, dv
template <int D_QK, int D_V, int BQ>
struct DkdvSmem {
    static constexpr int K = kKeysPerCta * D_QK * 2;
    static constexpr int V = kKeysPerCta * D_V * 2;
    static constexpr int Q = BQ * D_QK * 2;
    static constexpr int DO = BQ * D_V * 2;
    static constexpr int OFF_V = K;
    static constexpr int OFF_Q = OFF_V + V;             // two buffers
    static constexpr int OFF_DO = OFF_Q + 2 * Q;        // two buffers
    static constexpr int OFF_L = OFF_DO + 2 * DO;       // [2][BQ] lse * log2(e)
    static constexpr int OFF_D = OFF_L + 2 * BQ * 4;    // [2][BQ] D
    static constexpr int BYTES = OFF_D + 2 * BQ * 4;
};

template <typename T, int D_QK, int D_V, int BQ>
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_dkdv_kernel(const BwdParams p) {
    using S = DkdvSmem<D_QK, D_V, BQ>;
    extern __shared__ __align__(128) char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // blocks are dispatched roughly in linear-index order: key tile = the
    // slowest index, so the low key tiles of every (batch, head), which the
    // most query rows see under a causal mask, start first
    const int slices = gridDim.y * gridDim.z;
    const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const int j0 = (lin / slices) * kKeysPerCta, hk = (lin % slices) % p.h_kv, bi = (lin % slices) / p.h_kv;
    const int N = p.s_k, s_q = p.s_q;
    const int kvalid = min(kKeysPerCta, N - j0);
    const int j_hi = j0 + kvalid - 1;

    // query rows that see any of keys j0 .. j_hi: the last visible key and
    // the first visible key of a row are both nondecreasing in the row
    int lo = 0, hi = s_q;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        int64_t f, l;
        visible_keys(mid, N, s_q, p.causal, p.win_left, p.win_right, f, l);
        if (l >= j0) hi = mid; else lo = mid + 1;
    }
    const int i_lo = lo;
    lo = 0;
    hi = s_q;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        int64_t f, l;
        visible_keys(mid, N, s_q, p.causal, p.win_left, p.win_right, f, l);
        if (f > j_hi) hi = mid; else lo = mid + 1;
    }
    const int i_hi = lo - 1;
    const int qt0 = i_lo / BQ;
    const int n_qt = i_lo <= i_hi ? i_hi / BQ - qt0 + 1 : 0;
    const int n_tiles = p.g * n_qt;

    const T *kbase = static_cast<const T *>(p.k) + bi * p.ks.b + hk * p.ks.h;
    const T *vbase = static_cast<const T *>(p.v) + bi * p.vs.b + hk * p.vs.h;
    auto issue = [&](int u) {
        const int hq = hk * p.g + u / n_qt;
        const int i0 = (qt0 + u % n_qt) * BQ;
        const int valid = min(BQ, s_q - i0);
        const int buf = u & 1;
        stage_rows<T, D_QK, BQ>(smem + S::OFF_Q + buf * S::Q,
                                static_cast<const T *>(p.q) + bi * p.qs.b + (int64_t)i0 * p.qs.s + hq * p.qs.h,
                                p.qs.s, valid, tid);
        stage_rows<T, D_V, BQ>(smem + S::OFF_DO + buf * S::DO,
                               static_cast<const T *>(p.dout) + bi * p.dos.b + (int64_t)i0 * p.dos.s + hq * p.dos.h,
                               p.dos.s, valid, tid);
        if (tid < BQ) {
            const int64_t row = ((int64_t)bi * p.h_q + hq) * s_q + i0 + tid;
            float *sl = reinterpret_cast<float *>(smem + S::OFF_L) + buf * BQ;
            float *sd = reinterpret_cast<float *>(smem + S::OFF_D) + buf * BQ;
            sl[tid] = tid < valid ? p.lse[row] * kLog2e : 0.f;
            sd[tid] = tid < valid ? p.dsum[row] : 0.f;
        }
        cp_async_commit();
    };

    float dk[D_QK / 8][4], dv[D_V / 8][4];
#pragma unroll
    for (int n = 0; n < D_QK / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[n][e] = 0.f;
#pragma unroll
    for (int n = 0; n < D_V / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dv[n][e] = 0.f;

    if (n_tiles > 0) {
        stage_rows<T, D_QK, kKeysPerCta>(smem, kbase + (int64_t)j0 * p.ks.s, p.ks.s, kvalid, tid);
        stage_rows<T, D_V, kKeysPerCta>(smem + S::OFF_V, vbase + (int64_t)j0 * p.vs.s, p.vs.s, kvalid, tid);
        issue(0);
    }
    const uint32_t sK = smem_addr(smem), sV = smem_addr(smem + S::OFF_V);
    const int key_r = warp * 16 + (lane >> 2);  // this thread's key rows: key_r, key_r + 8
    for (int u = 0; u < n_tiles; ++u) {
        if (u + 1 < n_tiles) {
            issue(u + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int buf = u & 1;
        const int i0 = (qt0 + u % n_qt) * BQ;
        const uint32_t sQ = smem_addr(smem + S::OFF_Q + buf * S::Q);
        const uint32_t sDO = smem_addr(smem + S::OFF_DO + buf * S::DO);
        const float *sl = reinterpret_cast<const float *>(smem + S::OFF_L) + buf * BQ;
        const float *sd = reinterpret_cast<const float *>(smem + S::OFF_D) + buf * BQ;

        float s[BQ / 8][4], dp[BQ / 8][4];
#pragma unroll
        for (int n = 0; n < BQ / 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
        // S^T = K Q^T and dP^T = V dO^T
        mma_rows_rows2<T, D_QK, D_V, kKeysPerCta, BQ, BQ / 8>(s, sK, sQ, dp, sV, sDO, warp * 16, lane);

        // the whole tile is visible when its rows all exist, its last row's
        // first visible key is at most j0 and its first row's last visible
        // key at least j0 + 63 (both bounds are nondecreasing in the row)
        bool full = i0 + BQ <= s_q && kvalid == kKeysPerCta;
        if (full) {
            int64_t f, l;
            visible_keys(i0, N, s_q, p.causal, p.win_left, p.win_right, f, l);
            full = l >= j_hi;
            visible_keys(i0 + BQ - 1, N, s_q, p.causal, p.win_left, p.win_right, f, l);
            full = full && f <= j0;
        }
        // P^T and dS^T in place: element (key j, query i)
#pragma unroll
        for (int n = 0; n < BQ / 8; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int qc = n * 8 + ((lane & 3) << 1) + c;
                const int i = i0 + qc;
                int64_t f = 0, l = N;
                if (!full) visible_keys(i, N, s_q, p.causal, p.win_left, p.win_right, f, l);
                const float L = sl[qc], Dd = sd[qc];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int j = j0 + key_r + hr * 8;
                    const bool vis = full || (i < s_q && j < N && j >= f && j <= l);
                    const float pv = vis ? ex2(s[n][hr * 2 + c] * p.scale_log2 - L) : 0.f;
                    s[n][hr * 2 + c] = pv;
                    dp[n][hr * 2 + c] = pv * (dp[n][hr * 2 + c] - Dd);
                }
            }
        mma_frag_rows<T, D_V, BQ, BQ>(dv, s, sDO, lane);    // dV += P^T dO
        mma_frag_rows<T, D_QK, BQ, BQ>(dk, dp, sQ, lane);   // dK += dS^T Q
        __syncthreads();
    }

    store_rows<T, D_QK>(static_cast<T *>(p.dk) + bi * p.dks.b + (int64_t)j0 * p.dks.s + hk * p.dks.h, p.dks.s, dk,
                        warp * 16, kvalid, p.scale, lane);
    store_rows<T, D_V>(static_cast<T *>(p.dv) + bi * p.dvs.b + (int64_t)j0 * p.dvs.s + hk * p.dvs.h, p.dvs.s, dv,
                       warp * 16, kvalid, 1.f, lane);
}

// ---------------------------------------------------------------- dq
template <int D_QK, int D_V>
struct DqSmem {
    static constexpr int Q = kRowsPerCta * D_QK * 2;
    static constexpr int DO = kRowsPerCta * D_V * 2;
    static constexpr int K = kDqBK * D_QK * 2;
    static constexpr int V = kDqBK * D_V * 2;
    static constexpr int OFF_DO = Q;
    static constexpr int OFF_K = OFF_DO + DO;   // two buffers
    static constexpr int OFF_V = OFF_K + 2 * K;  // two buffers
    static constexpr int BYTES = OFF_V + 2 * V;
};

template <typename T, int D_QK, int D_V>
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_dq_kernel(const BwdParams p) {
    using S = DqSmem<D_QK, D_V>;
    extern __shared__ __align__(128) char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the last query tiles of every (batch, head), which see the most keys
    // under a causal mask, start first (see bwd_dkdv_kernel)
    const int slices = gridDim.y * gridDim.z;
    const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const int i0 = (gridDim.x - 1 - lin / slices) * kRowsPerCta, hq = (lin % slices) % p.h_q,
              bi = (lin % slices) / p.h_q;
    const int hk = hq / p.g;
    const int N = p.s_k, s_q = p.s_q;
    const int qvalid = min(kRowsPerCta, s_q - i0);

    // keys seen by rows i0 .. i0 + qvalid - 1
    int64_t f0, l0, f1, l1;
    visible_keys(i0, N, s_q, p.causal, p.win_left, p.win_right, f0, l0);
    visible_keys(i0 + qvalid - 1, N, s_q, p.causal, p.win_left, p.win_right, f1, l1);
    const int kv_end = (int)max((int64_t)0, min((int64_t)N, l1 + 1));
    const int kt0 = (int)min(f0, (int64_t)kv_end) / kDqBK;
    const int n_kt = kv_end > 0 ? (kv_end + kDqBK - 1) / kDqBK - kt0 : 0;

    const T *kbase = static_cast<const T *>(p.k) + bi * p.ks.b + hk * p.ks.h;
    const T *vbase = static_cast<const T *>(p.v) + bi * p.vs.b + hk * p.vs.h;
    auto issue = [&](int u) {
        const int j0 = (kt0 + u) * kDqBK;
        const int valid = min(kDqBK, N - j0);
        const int buf = u & 1;
        stage_rows<T, D_QK, kDqBK>(smem + S::OFF_K + buf * S::K, kbase + (int64_t)j0 * p.ks.s, p.ks.s, valid, tid);
        stage_rows<T, D_V, kDqBK>(smem + S::OFF_V + buf * S::V, vbase + (int64_t)j0 * p.vs.s, p.vs.s, valid, tid);
        cp_async_commit();
    };

    // this thread's rows: r0 = i0 + warp*16 + lane/4 and r0 + 8
    const int rbase = i0 + warp * 16 + (lane >> 2);
    float L[2], Dd[2];
    int64_t fv[2], lv[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int i = rbase + hr * 8;
        visible_keys(i, N, s_q, p.causal, p.win_left, p.win_right, fv[hr], lv[hr]);
        if (i >= s_q) lv[hr] = -1;  // past the rows: nothing visible
        const int64_t row = ((int64_t)bi * p.h_q + hq) * s_q + min(i, s_q - 1);
        L[hr] = i < s_q ? p.lse[row] * kLog2e : 0.f;
        Dd[hr] = i < s_q ? p.dsum[row] : 0.f;
    }

    float dq[D_QK / 8][4];
#pragma unroll
    for (int n = 0; n < D_QK / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;

    if (n_kt > 0) {
        stage_rows<T, D_QK, kRowsPerCta>(smem, static_cast<const T *>(p.q) + bi * p.qs.b + (int64_t)i0 * p.qs.s +
                                                   hq * p.qs.h,
                                         p.qs.s, qvalid, tid);
        stage_rows<T, D_V, kRowsPerCta>(smem + S::OFF_DO, static_cast<const T *>(p.dout) + bi * p.dos.b +
                                                              (int64_t)i0 * p.dos.s + hq * p.dos.h,
                                        p.dos.s, qvalid, tid);
        issue(0);
    }
    const uint32_t sQ = smem_addr(smem), sDO = smem_addr(smem + S::OFF_DO);
    for (int u = 0; u < n_kt; ++u) {
        if (u + 1 < n_kt) {
            issue(u + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int buf = u & 1;
        const int j0 = (kt0 + u) * kDqBK;
        const uint32_t sK = smem_addr(smem + S::OFF_K + buf * S::K);
        const uint32_t sV = smem_addr(smem + S::OFF_V + buf * S::V);

        float s[kDqBK / 8][4], dp[kDqBK / 8][4];
#pragma unroll
        for (int n = 0; n < kDqBK / 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
        // S = Q K^T and dP = dO V^T
        mma_rows_rows2<T, D_QK, D_V, kRowsPerCta, kDqBK, kDqBK / 8>(s, sQ, sK, dp, sDO, sV, warp * 16, lane);

#pragma unroll
        for (int n = 0; n < kDqBK / 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hr = e >> 1;
                const int j = j0 + n * 8 + ((lane & 3) << 1) + (e & 1);
                const bool vis = j < N && j >= fv[hr] && j <= lv[hr];
                const float pv = vis ? ex2(s[n][e] * p.scale_log2 - L[hr]) : 0.f;
                dp[n][e] = pv * (dp[n][e] - Dd[hr]);
            }
        mma_frag_rows<T, D_QK, kDqBK, kDqBK>(dq, dp, sK, lane);  // dQ += dS K
        __syncthreads();
    }

    store_rows<T, D_QK>(static_cast<T *>(p.dq) + bi * p.dqs.b + (int64_t)i0 * p.dqs.s + hq * p.dqs.h, p.dqs.s, dq,
                        warp * 16, qvalid, p.scale, lane);
}

template <typename T, int D_QK, int D_V, int BQ>
cudaError_t run_bwd(const BwdParams &p, cudaStream_t st) {
    const int64_t rows = (int64_t)p.b * p.s_q * p.h_q;
    if (rows > 0) {
        bwd_dot_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    kernel_event(0, st);
    if (p.s_k > 0) {
        using SK = DkdvSmem<D_QK, D_V, BQ>;
        cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<T, D_QK, D_V, BQ>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SK::BYTES);
        if (e != cudaSuccess) return e;
        dim3 grid((p.s_k + kKeysPerCta - 1) / kKeysPerCta, p.h_kv, p.b);
        bwd_dkdv_kernel<T, D_QK, D_V, BQ><<<grid, kBwdThreads, SK::BYTES, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.s_q > 0) {
        using SQ = DqSmem<D_QK, D_V>;
        cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<T, D_QK, D_V>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SQ::BYTES);
        if (e != cudaSuccess) return e;
        dim3 grid((p.s_q + kRowsPerCta - 1) / kRowsPerCta, p.h_q, p.b);
        bwd_dq_kernel<T, D_QK, D_V><<<grid, kBwdThreads, SQ::BYTES, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    kernel_event(1, st);
    return cudaSuccess;
}

template <typename T>
cudaError_t dispatch_bwd(const BwdParams &p, cudaStream_t st) {
    if (p.d_qk == 64 && p.d_v == 64) return run_bwd<T, 64, 64, 64>(p, st);
    if (p.d_qk == 128 && p.d_v == 128) return run_bwd<T, 128, 128, 32>(p, st);
    if (p.d_qk == 192 && p.d_v == 128) return run_bwd<T, 192, 128, 32>(p, st);
    return cudaErrorInvalidValue;
}

}  // namespace

bool bwd_supported(int d_qk, int d_v) {
    return (d_qk == 64 && d_v == 64) || (d_qk == 128 && d_v == 128) || (d_qk == 192 && d_v == 128);
}

cudaError_t launch_bwd(const BwdParams &p, int dtype, cudaStream_t st) {
    return dtype == FA_DTYPE_BF16 ? dispatch_bwd<__nv_bfloat16>(p, st) : dispatch_bwd<__half>(p, st);
}

}  // namespace fa
