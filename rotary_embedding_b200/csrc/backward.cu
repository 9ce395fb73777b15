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
//  - bwd_dkdv_kernel: one CTA per 128 keys of a (batch, kv head), walking the
//    64-row query tiles, of every query head of the group, that see any of
//    those keys.  On the tensor cores (tcgen05, operands staged by TMA,
//    accumulators in TMEM): S^T = K Q^T and dP^T = V dO^T with the 128 keys
//    as M; the elementwise warpgroup (thread t = key row t = TMEM lane t)
//    turns them into P^T and dS^T, written back to TMEM as 16-bit pairs, the
//    A operand of dV += P^T dO and dK += dS^T Q, which accumulate in TMEM for
//    the whole walk.  S^T / dP^T of the next query tile are computed while
//    the elementwise warpgroup works on the current one.
//  - bwd_dq_kernel: one CTA per 128 query rows of a (batch, query head),
//    walking 64-key tiles: S = Q K^T, dP = dO V^T, dQ += dS K, likewise.
//    (S and dP are formed twice, once per kernel: the price of writing dq
//    without atomics.)
// P and dS are rounded to the element type as MMA operands; rows past a
// sequence arrive as zeros from the TMA (out-of-bounds fill) and are masked.
#include <type_traits>

#include "fa_common.cuh"
#include "fa_internal.h"
#include "tcgen05.cuh"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Untiled bulk copy global -> shared (16-byte aligned, size a multiple of
// 16), completing on `bar` like a TMA tile load.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// Register split of the backward kernels (384 threads launched at 168 per
// thread): warpgroup 0 (TMA, MMA, two idle warps) down to 64, the two
// elementwise warpgroups up to 200: 128 x 64 + 256 x 200 = 59392 <= 64512.
constexpr int kBwdRegsLow = 64, kBwdRegsHigh = 200;

// ---------------------------------------------------------------- D_i
// Per query row i of every (batch, query head), into the workspace: lse_i
// log2(e) and D_i = dout_i . out_i; the padding rows s_q .. s_q_pad - 1 get
// +inf and 0 (P = 0 there).  One 16-byte chunk (8 elements) of the row per
// lane (d_v / 8 lanes per row, 32 * 8 / d_v rows per warp, 8 warps per
// block), the chunks' partial sums reduced with shuffles inside the row's
// lanes.  Rows are taken in (batch, row, head) order, so a warp's loads of
// the heads of one row are contiguous.
template <typename T>
__global__ void __launch_bounds__(256) bwd_dot_kernel(const BwdParams p) {
    const int lanes_per_row = p.d_v / 8;                   // 8, 16 or 32 (d_v 64, 128, 256)
    const int rows_per_warp = 32 / lanes_per_row;
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int64_t rowg = w * rows_per_warp + lane / lanes_per_row;
    const int chunk = lane % lanes_per_row;
    const int64_t rows = (int64_t)p.b * p.s_q_pad * p.h_q;
    const int h = (int)(rowg % p.h_q);
    const int64_t bi_i = rowg / p.h_q;
    const int i = (int)(bi_i % p.s_q_pad), bi = (int)(bi_i / p.s_q_pad);
    const bool real = rowg < rows && i < p.s_q;
    float acc = 0.f;
    if (real) {
        const T *o = static_cast<const T *>(p.out) + bi * p.os.b + (int64_t)i * p.os.s + h * p.os.h;
        const T *d = static_cast<const T *>(p.dout) + bi * p.dos.b + (int64_t)i * p.dos.s + h * p.dos.h;
        float fo[8], fd[8];
        unpack8<T>(__ldg(reinterpret_cast<const uint4 *>(o) + chunk), fo);
        unpack8<T>(__ldg(reinterpret_cast<const uint4 *>(d) + chunk), fd);
#pragma unroll
        for (int t = 0; t < 8; ++t) acc = fmaf(fo[t], fd[t], acc);
    }
    for (int off = lanes_per_row / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (rowg < rows && chunk == 0) {
        const int64_t at = ((int64_t)bi * p.h_q + h) * p.s_q_pad + i;
        p.lsum[at] = real ? p.lse[((int64_t)bi * p.h_q + h) * p.s_q + i] * kLog2e : INFINITY;
        p.dsum[at] = acc;
    }
}

// ---------------------------------------------------------------- dk, dv
constexpr int kBK = 128;   // keys per dk/dv CTA (the MMA M)
constexpr int kBQ = 64;    // query rows per tile of the dk/dv walk
constexpr int kDqBM = 128; // query rows per dq CTA (the MMA M)
constexpr int kDqBN = 64;  // keys per tile of the dq walk

// Shared memory of the dk/dv kernel: the K and V tiles (loaded once), then a
// ring of stages, each holding a Q tile, a dO tile and the tile's
// lse * log2(e) and D values; every TMA destination is 1024-byte aligned
// (128-byte swizzle).  TMEM: S^T, dP^T, P^T, dS^T (16-bit pairs), dV, dK.
template <int D_QK, int D_V>
struct DkdvCfg {
    static constexpr int KBYTES = kBK * D_QK * 2;
    static constexpr int VBYTES = kBK * D_V * 2;
    static constexpr int KBOX = kBK * 128;     // bytes of one 64-column box of the K / V tile
    static constexpr int QBYTES = kBQ * D_QK * 2;
    static constexpr int DOBYTES = kBQ * D_V * 2;
    static constexpr int QBOX = kBQ * 128;     // ... of a Q / dO tile
    static constexpr int OFF_LD = QBYTES + DOBYTES;
    static constexpr int STAGE = (OFF_LD + 2 * kBQ * 4 + 1023) / 1024 * 1024;
    static constexpr int ST_RAW = (224 * 1024 - KBYTES - VBYTES) / STAGE;
    static constexpr int ST = ST_RAW > 4 ? 4 : ST_RAW;
    static constexpr int SMEM = 1024 + KBYTES + VBYTES + ST * STAGE + 256;
    static constexpr uint32_t T_S = 0, T_DP = kBQ, T_P = 2 * kBQ, T_DS = 2 * kBQ + kBQ / 2, T_DV = 3 * kBQ,
                              T_DK = 3 * kBQ + D_V;
    static_assert(T_DK + D_QK <= 512, "TMEM columns");
    static_assert(ST >= 2, "stage ring");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

template <typename T, int D_QK, int D_V>
__global__ void __launch_bounds__(384, 1) bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const __grid_constant__ CUtensorMap tmQ,
                                                          const __grid_constant__ CUtensorMap tmDO,
                                                          const BwdParams p) {
    using C = DkdvCfg<D_QK, D_V>;
    constexpr int ST = C::ST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem;
    uint8_t *sV = sK + C::KBYTES;
    uint8_t *sStage = sV + C::VBYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + ST * C::STAGE);
    uint64_t *kv_full = bars;              // 1
    uint64_t *full = kv_full + 1;          // ST: Q, dO (TMA) and lse / D (bulk copies)
    uint64_t *empty = full + ST;           // ST
    uint64_t *s_full = empty + ST;         // S^T, dP^T of the tile complete
    uint64_t *s_free = s_full + 1;         // ... read into registers
    uint64_t *p_full = s_free + 1;         // P^T, dS^T written
    uint64_t *pd_done = p_full + 1;        // dV, dK of the tile complete (P^T, dS^T free)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pd_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // key tile = the slowest index: the low key tiles of every (batch, kv
    // head), which the most query rows see under a causal mask, start first
    const int slices = p.h_kv * p.b;
    const int kt = (int)blockIdx.x / slices, rem = (int)blockIdx.x - kt * slices;
    const int hk = rem % p.h_kv, bi = rem / p.h_kv;
    const int j0 = kt * kBK;
    const int N = p.s_k, s_q = p.s_q;
    const int kvalid = min(kBK, N - j0);
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
    const int qt0 = i_lo / kBQ;
    const int n_qt = i_lo <= i_hi ? i_hi / kBQ - qt0 + 1 : 0;
    const int n_tiles = p.g * n_qt;   // tile u: query head hk g + u / n_qt, rows (qt0 + u % n_qt) kBQ ..

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 8);
        mbar_init(p_full, 8);
        mbar_init(pd_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;

    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kBwdRegsLow) : "memory");
    if (warp == 0) {
        // ------------------------------------------------ producer: TMA tiles and the lse / D runs
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(kv_full, C::KBYTES + C::VBYTES);
#pragma unroll
            for (int c = 0; c < D_QK / 64; ++c) tma_load_4d(sK + c * C::KBOX, &tmK, kv_full, c * 64, hk, j0, bi);
#pragma unroll
            for (int c = 0; c < D_V / 64; ++c) tma_load_4d(sV + c * C::KBOX, &tmV, kv_full, c * 64, hk, j0, bi);
            for (int u = 0; u < n_tiles; ++u) {
                const int st = u % ST;
                if (u >= ST && !mbar_wait(&empty[st], ((u / ST) - 1) & 1, p.status)) break;
                const int hq = hk * p.g + u / n_qt;
                const int i0 = (qt0 + u % n_qt) * kBQ;
                uint8_t *stage = sStage + st * C::STAGE;
                mbar_arrive_expect_tx(&full[st], C::QBYTES + C::DOBYTES + 2 * kBQ * 4);
#pragma unroll
                for (int c = 0; c < D_QK / 64; ++c)
                    tma_load_4d(stage + c * C::QBOX, &tmQ, &full[st], c * 64, hq, i0, bi);
#pragma unroll
                for (int c = 0; c < D_V / 64; ++c)
                    tma_load_4d(stage + C::QBYTES + c * C::QBOX, &tmDO, &full[st], c * 64, hq, i0, bi);
                // the tile's 64 rows are one aligned run of each workspace array
                const int64_t run = ((int64_t)bi * p.h_q + hq) * p.s_q_pad + i0;
                bulk_load(stage + C::OFF_LD, p.lsum + run, kBQ * 4, &full[st]);
                bulk_load(stage + C::OFF_LD + kBQ * 4, p.dsum + run, kBQ * 4, &full[st]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (whole warp loops, one lane issues)
        if (n_tiles > 0) {
            const bool leader = tc::elect_one();
            const uint32_t idesc_s = tc::idesc_f16(bf16, kBK, kBQ, false);
            const uint32_t idesc_dv = tc::idesc_f16(bf16, kBK, D_V, true);
            const uint32_t idesc_dk = tc::idesc_f16(bf16, kBK, D_QK, true);
            // descriptors of the first k-step of each operand; a k-step (and a
            // stage) only moves the start address field (16-byte units)
            const uint64_t dK0 = tc::smem_desc(smem_addr(sK), 16, 1024);
            const uint64_t dV0 = tc::smem_desc(smem_addr(sV), 16, 1024);
            const uint64_t dS0 = tc::smem_desc(smem_addr(sStage), 16, 1024);            // Q / dO, K-major
            const uint64_t dM0 = tc::smem_desc(smem_addr(sStage), C::QBOX, 1024);        // Q / dO, MN-major
            bool ok = mbar_wait(kv_full, 0, p.status);
            // S^T = K Q^T and dP^T = V dO^T (K-major operands)
            auto issue_sdp = [&](int u) {
                const uint64_t q = dS0 + (uint64_t)(((u % ST) * C::STAGE) >> 4), o = q + (uint64_t)(C::QBYTES >> 4);
                if (leader) {
#pragma unroll
                    for (int k = 0; k < D_QK / 16; ++k)
                        tc::mma_ss(tmem + C::T_S, dK0 + (uint64_t)(((k >> 2) * C::KBOX + (k & 3) * 32) >> 4),
                                   q + (uint64_t)(((k >> 2) * C::QBOX + (k & 3) * 32) >> 4), idesc_s, k > 0);
#pragma unroll
                    for (int k = 0; k < D_V / 16; ++k)
                        tc::mma_ss(tmem + C::T_DP, dV0 + (uint64_t)(((k >> 2) * C::KBOX + (k & 3) * 32) >> 4),
                                   o + (uint64_t)(((k >> 2) * C::QBOX + (k & 3) * 32) >> 4), idesc_s, k > 0);
                    tc::commit(s_full);
                }
                __syncwarp();
            };
            // dV += P^T dO and dK += dS^T Q (P^T, dS^T from TMEM; dO, Q as MN-major B)
            auto issue_acc = [&](int u) {
                const uint64_t q = dM0 + (uint64_t)(((u % ST) * C::STAGE) >> 4), o = q + (uint64_t)(C::QBYTES >> 4);
                if (leader) {
#pragma unroll
                    for (int k = 0; k < kBQ / 16; ++k)
                        tc::mma_ts(tmem + C::T_DV, tmem + C::T_P + k * 8, o + (uint64_t)(k * 16 * 128 / 16), idesc_dv,
                                   (u > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < kBQ / 16; ++k)
                        tc::mma_ts(tmem + C::T_DK, tmem + C::T_DS + k * 8, q + (uint64_t)(k * 16 * 128 / 16), idesc_dk,
                                   (u > 0 || k > 0) ? 1u : 0u);
                    tc::commit(&empty[u % ST]);
                    tc::commit(pd_done);
                }
                __syncwarp();
            };
            if (ok && (ok = mbar_wait(&full[0], 0, p.status))) {
                tc::fence_after_sync();
                issue_sdp(0);
            }
            for (int u = 0; u < n_tiles && ok; ++u) {
                if (u + 1 < n_tiles) {
                    if (!(ok = mbar_wait(&full[(u + 1) % ST], ((u + 1) / ST) & 1, p.status))) break;
                    if (!(ok = mbar_wait(s_free, u & 1, p.status))) break;
                    tc::fence_after_sync();
                    issue_sdp(u + 1);
                }
                if (!(ok = mbar_wait(p_full, u & 1, p.status))) break;
                tc::fence_after_sync();
                issue_acc(u);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ elementwise warpgroups: key row j = TMEM lane,
        // warpgroup hf takes query columns [32 hf, 32 hf + 32) of every tile
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kBwdRegsHigh) : "memory");
        const int hf = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int j = j0 + r;
        const bool key_valid = r < kvalid;
        // queries that see key j: i_min .. i_max (bottom-right alignment a_i = i + N - s_q)
        const int64_t off = (int64_t)N - s_q;
        int64_t i_min = 0, i_max = (int64_t)s_q - 1;
        if (p.causal) i_min = max(i_min, (int64_t)j - off);
        if (p.win_right >= 0) i_min = max(i_min, (int64_t)j - p.win_right - off);
        if (p.win_left >= 0) i_max = min(i_max, (int64_t)j + p.win_left - off);
        if (!key_valid) i_max = -1;
        // as 32-bit bounds (clamped to the query rows, which fit 32 bits)
        const int i_min32 = (int)min(i_min, (int64_t)s_q), i_max32 = (int)max(i_max, (int64_t)-1);
        const float c = p.scale_log2;
        bool ok = true;
        for (int u = 0; u < n_tiles && ok; ++u) {
            if (!(ok = mbar_wait(s_full, u & 1, p.status))) break;
            tc::fence_after_sync();
            uint32_t sr[32], dr[32];
            tc::ld32(tmem + lane_addr + C::T_S + 32 * hf, sr);
            tc::ld32(tmem + lane_addr + C::T_DP + 32 * hf, dr);
            tc::wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free);
            const int st = u % ST;
            if (!(ok = mbar_wait(&full[st], (u / ST) & 1, p.status))) break;
            // P^T and dS^T of the previous tile have been read by its dV / dK
            if (u > 0) {
                if (!(ok = mbar_wait(pd_done, (u - 1) & 1, p.status))) break;
                tc::fence_after_sync();
            }
            const float *ld = reinterpret_cast<const float *>(sStage + st * C::STAGE + C::OFF_LD) + 32 * hf;
            const int i0 = (qt0 + u % n_qt) * kBQ + 32 * hf;   // this warpgroup's first query
            uint32_t pp[16], pd[16];
            // P^T = 2^(s c - L), dS^T = P^T (dP^T - D); tiles on a mask edge
            // (masked = true) zero the pairs no mask admits
            auto math = [&](auto masked) {
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 L = *reinterpret_cast<const float4 *>(ld + e);
                    const float4 D = *reinterpret_cast<const float4 *>(ld + kBQ + e);
                    const float lv[4] = {L.x, L.y, L.z, L.w}, dv4[4] = {D.x, D.y, D.z, D.w};
#pragma unroll
                    for (int t = 0; t < 4; t += 2) {
                        float p0 = ex2(fmaf(__uint_as_float(sr[e + t]), c, -lv[t]));
                        float p1 = ex2(fmaf(__uint_as_float(sr[e + t + 1]), c, -lv[t + 1]));
                        if (decltype(masked)::value) {
                            const int q = i0 + e + t;
                            if (q < i_min32 || q > i_max32) p0 = 0.f;
                            if (q + 1 < i_min32 || q + 1 > i_max32) p1 = 0.f;
                        }
                        pp[(e + t) >> 1] = Elem<T>::pack2(p0, p1);
                        pd[(e + t) >> 1] = Elem<T>::pack2(p0 * (__uint_as_float(dr[e + t]) - dv4[t]),
                                                          p1 * (__uint_as_float(dr[e + t + 1]) - dv4[t + 1]));
                    }
                }
            };
            if (i0 >= i_min32 && i0 + 31 <= i_max32)
                math(std::integral_constant<bool, false>());
            else
                math(std::integral_constant<bool, true>());
            tc::st16(tmem + lane_addr + C::T_P + 16 * hf, pp);
            tc::st16(tmem + lane_addr + C::T_DS + 16 * hf, pd);
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ------------------------------------------------ epilogue: dv = dV, dk = scale dK (32-column
        // chunks alternate between the two warpgroups)
        const bool have = n_tiles > 0;
        if (have && ok) ok = mbar_wait(pd_done, (n_tiles - 1) & 1, p.status);
        tc::fence_after_sync();
        T *dvrow = static_cast<T *>(p.dv) + bi * p.dvs.b + (int64_t)j * p.dvs.s + hk * p.dvs.h;
        T *dkrow = static_cast<T *>(p.dk) + bi * p.dks.b + (int64_t)j * p.dks.s + hk * p.dks.h;
#pragma unroll
        for (int h = 0; h < (D_V + D_QK) / 32; ++h) {
            if ((h & 1) != hf) continue;
            const bool is_v = h < D_V / 32;
            const int col = is_v ? h * 32 : (h - D_V / 32) * 32;
            uint32_t orr[32];
            if (have) {
                tc::ld32(tmem + lane_addr + (is_v ? C::T_DV : C::T_DK) + col, orr);
                tc::wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) orr[e] = 0u;
            }
            if (key_valid) {
                const float mul = is_v ? 1.f : p.scale;
                T *dst = (is_v ? dvrow : dkrow) + col;
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    float f[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) f[t] = __uint_as_float(orr[e + t]) * mul;
                    reinterpret_cast<uint4 *>(dst + e)[0] = pack8<T>(f);
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- dq
// Shared memory: the Q and dO tiles (loaded once) and a ring of K / V
// stages.  TMEM: S, dP, dS (16-bit pairs), dQ.
template <int D_QK, int D_V>
struct DqCfg {
    static constexpr int QBYTES = kDqBM * D_QK * 2;
    static constexpr int DOBYTES = kDqBM * D_V * 2;
    static constexpr int QBOX = kDqBM * 128;
    static constexpr int KBYTES = kDqBN * D_QK * 2;
    static constexpr int VBYTES = kDqBN * D_V * 2;
    static constexpr int KBOX = kDqBN * 128;
    static constexpr int STAGE = KBYTES + VBYTES;
    static constexpr int ST_RAW = (224 * 1024 - QBYTES - DOBYTES) / STAGE;
    static constexpr int ST = ST_RAW > 4 ? 4 : ST_RAW;
    static constexpr int SMEM = 1024 + QBYTES + DOBYTES + ST * STAGE + 256;
    static constexpr uint32_t T_S = 0, T_DP = kDqBN, T_DS = 2 * kDqBN, T_DQ = 2 * kDqBN + kDqBN / 2;
    static_assert(T_DQ + D_QK <= 512, "TMEM columns");
    static_assert(STAGE % 1024 == 0 && ST >= 2, "stage ring");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

template <typename T, int D_QK, int D_V>
__global__ void __launch_bounds__(384, 1) bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                        const __grid_constant__ CUtensorMap tmDO,
                                                        const __grid_constant__ CUtensorMap tmK,
                                                        const __grid_constant__ CUtensorMap tmV,
                                                        const BwdParams p) {
    using C = DqCfg<D_QK, D_V>;
    constexpr int ST = C::ST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sDO = sQ + C::QBYTES;
    uint8_t *sStage = sDO + C::DOBYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + ST * C::STAGE);
    uint64_t *q_full = bars;               // 1
    uint64_t *full = q_full + 1;           // ST
    uint64_t *empty = full + ST;           // ST
    uint64_t *s_full = empty + ST;
    uint64_t *s_free = s_full + 1;
    uint64_t *p_full = s_free + 1;
    uint64_t *ds_done = p_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ds_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the last query tiles of every (batch, head), which see the most keys
    // under a causal mask, start first
    const int slices = p.h_q * p.b;
    const int n_qtiles = (int)gridDim.x / slices;
    const int t = (int)blockIdx.x / slices, rem = (int)blockIdx.x - t * slices;
    const int hq = rem % p.h_q, bi = rem / p.h_q;
    const int hk = hq / p.g;
    const int i0 = (n_qtiles - 1 - t) * kDqBM;
    const int N = p.s_k, s_q = p.s_q;
    const int qvalid = min(kDqBM, s_q - i0);
    int64_t f0, l0, f1, l1;
    visible_keys(i0, N, s_q, p.causal, p.win_left, p.win_right, f0, l0);
    visible_keys(i0 + qvalid - 1, N, s_q, p.causal, p.win_left, p.win_right, f1, l1);
    const int kv_end = (int)max((int64_t)0, min((int64_t)N, l1 + 1));
    const int kt0 = (int)min(f0, (int64_t)kv_end) / kDqBN;
    const int n_kt = kv_end > 0 ? (kv_end + kDqBN - 1) / kDqBN - kt0 : 0;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 8);
        mbar_init(p_full, 8);
        mbar_init(ds_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;

    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kBwdRegsLow) : "memory");
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n_kt > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmDO);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(q_full, C::QBYTES + C::DOBYTES);
#pragma unroll
            for (int c = 0; c < D_QK / 64; ++c) tma_load_4d(sQ + c * C::QBOX, &tmQ, q_full, c * 64, hq, i0, bi);
#pragma unroll
            for (int c = 0; c < D_V / 64; ++c) tma_load_4d(sDO + c * C::QBOX, &tmDO, q_full, c * 64, hq, i0, bi);
            for (int u = 0; u < n_kt; ++u) {
                const int st = u % ST;
                if (u >= ST && !mbar_wait(&empty[st], ((u / ST) - 1) & 1, p.status)) break;
                const int jt = (kt0 + u) * kDqBN;
                uint8_t *stage = sStage + st * C::STAGE;
                mbar_arrive_expect_tx(&full[st], C::STAGE);
#pragma unroll
                for (int c = 0; c < D_QK / 64; ++c) tma_load_4d(stage + c * C::KBOX, &tmK, &full[st], c * 64, hk, jt, bi);
#pragma unroll
                for (int c = 0; c < D_V / 64; ++c)
                    tma_load_4d(stage + C::KBYTES + c * C::KBOX, &tmV, &full[st], c * 64, hk, jt, bi);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (n_kt > 0) {
            const bool leader = tc::elect_one();
            const uint32_t idesc_s = tc::idesc_f16(bf16, kDqBM, kDqBN, false);
            const uint32_t idesc_dq = tc::idesc_f16(bf16, kDqBM, D_QK, true);
            const uint64_t dQ0 = tc::smem_desc(smem_addr(sQ), 16, 1024);
            const uint64_t dO0 = tc::smem_desc(smem_addr(sDO), 16, 1024);
            const uint64_t dS0 = tc::smem_desc(smem_addr(sStage), 16, 1024);            // K / V, K-major
            const uint64_t dM0 = tc::smem_desc(smem_addr(sStage), C::KBOX, 1024);        // K, MN-major
            bool ok = mbar_wait(q_full, 0, p.status);
            // S = Q K^T and dP = dO V^T
            auto issue_sdp = [&](int u) {
                const uint64_t kk = dS0 + (uint64_t)(((u % ST) * C::STAGE) >> 4), vv = kk + (uint64_t)(C::KBYTES >> 4);
                if (leader) {
#pragma unroll
                    for (int k = 0; k < D_QK / 16; ++k)
                        tc::mma_ss(tmem + C::T_S, dQ0 + (uint64_t)(((k >> 2) * C::QBOX + (k & 3) * 32) >> 4),
                                   kk + (uint64_t)(((k >> 2) * C::KBOX + (k & 3) * 32) >> 4), idesc_s, k > 0);
#pragma unroll
                    for (int k = 0; k < D_V / 16; ++k)
                        tc::mma_ss(tmem + C::T_DP, dO0 + (uint64_t)(((k >> 2) * C::QBOX + (k & 3) * 32) >> 4),
                                   vv + (uint64_t)(((k >> 2) * C::KBOX + (k & 3) * 32) >> 4), idesc_s, k > 0);
                    tc::commit(s_full);
                }
                __syncwarp();
            };
            // dQ += dS K (dS from TMEM, K as MN-major B)
            auto issue_dq = [&](int u) {
                const uint64_t kk = dM0 + (uint64_t)(((u % ST) * C::STAGE) >> 4);
                if (leader) {
#pragma unroll
                    for (int k = 0; k < kDqBN / 16; ++k)
                        tc::mma_ts(tmem + C::T_DQ, tmem + C::T_DS + k * 8, kk + (uint64_t)(k * 16 * 128 / 16), idesc_dq,
                                   (u > 0 || k > 0) ? 1u : 0u);
                    tc::commit(&empty[u % ST]);
                    tc::commit(ds_done);
                }
                __syncwarp();
            };
            if (ok && (ok = mbar_wait(&full[0], 0, p.status))) {
                tc::fence_after_sync();
                issue_sdp(0);
            }
            for (int u = 0; u < n_kt && ok; ++u) {
                if (u + 1 < n_kt) {
                    if (!(ok = mbar_wait(&full[(u + 1) % ST], ((u + 1) / ST) & 1, p.status))) break;
                    if (!(ok = mbar_wait(s_free, u & 1, p.status))) break;
                    tc::fence_after_sync();
                    issue_sdp(u + 1);
                }
                if (!(ok = mbar_wait(p_full, u & 1, p.status))) break;
                tc::fence_after_sync();
                issue_dq(u);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ elementwise warpgroups: query row i = TMEM lane,
        // warpgroup hf takes key columns [32 hf, 32 hf + 32) of every tile
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kBwdRegsHigh) : "memory");
        const int hf = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int i = i0 + r;
        const bool row_valid = r < qvalid;
        int64_t fv, lv;
        visible_keys(i, N, s_q, p.causal, p.win_left, p.win_right, fv, lv);
        if (!row_valid) lv = -1;
        // as 32-bit bounds (keys fit 32 bits)
        const int fv32 = (int)min(fv, (int64_t)N), lv32 = (int)max(lv, (int64_t)-1);
        const int64_t at = ((int64_t)bi * p.h_q + hq) * p.s_q_pad + (row_valid ? i : 0);
        const float L = row_valid ? p.lsum[at] : INFINITY;
        const float Dd = row_valid ? p.dsum[at] : 0.f;
        const float c = p.scale_log2;
        bool ok = true;
        for (int u = 0; u < n_kt && ok; ++u) {
            if (!(ok = mbar_wait(s_full, u & 1, p.status))) break;
            tc::fence_after_sync();
            uint32_t sr[32], dr[32];
            tc::ld32(tmem + lane_addr + C::T_S + 32 * hf, sr);
            tc::ld32(tmem + lane_addr + C::T_DP + 32 * hf, dr);
            tc::wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free);
            // dS of the previous key tile has been read by its dQ product
            if (u > 0) {
                if (!(ok = mbar_wait(ds_done, (u - 1) & 1, p.status))) break;
                tc::fence_after_sync();
            }
            const int jt = (kt0 + u) * kDqBN + 32 * hf;   // this warpgroup's first key
            uint32_t pd[16];
            // dS = 2^(s c - L) (dP - D); tiles on a mask edge (masked = true)
            // zero the pairs no mask admits
            auto math = [&](auto masked) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float p0 = ex2(fmaf(__uint_as_float(sr[e]), c, -L));
                    float p1 = ex2(fmaf(__uint_as_float(sr[e + 1]), c, -L));
                    if (decltype(masked)::value) {
                        if (jt + e < fv32 || jt + e > lv32) p0 = 0.f;
                        if (jt + e + 1 < fv32 || jt + e + 1 > lv32) p1 = 0.f;
                    }
                    pd[e >> 1] = Elem<T>::pack2(p0 * (__uint_as_float(dr[e]) - Dd), p1 * (__uint_as_float(dr[e + 1]) - Dd));
                }
            };
            if (jt >= fv32 && jt + 31 <= lv32)
                math(std::integral_constant<bool, false>());
            else
                math(std::integral_constant<bool, true>());
            tc::st16(tmem + lane_addr + C::T_DS + 16 * hf, pd);
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ------------------------------------------------ epilogue: dq = scale dQ (32-column chunks
        // alternate between the two warpgroups)
        const bool have = n_kt > 0;
        if (have && ok) ok = mbar_wait(ds_done, (n_kt - 1) & 1, p.status);
        tc::fence_after_sync();
        T *dqrow = static_cast<T *>(p.dq) + bi * p.dqs.b + (int64_t)i * p.dqs.s + hq * p.dqs.h;
#pragma unroll
        for (int h = 0; h < D_QK / 32; ++h) {
            if ((h & 1) != hf) continue;
            uint32_t orr[32];
            if (have) {
                tc::ld32(tmem + lane_addr + C::T_DQ + h * 32, orr);
                tc::wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) orr[e] = 0u;
            }
            if (row_valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    float f[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) f[q] = __uint_as_float(orr[e + q]) * p.scale;
                    reinterpret_cast<uint4 *>(dqrow + h * 32 + e)[0] = pack8<T>(f);
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// The register split must fit in what the block is launched with (384
// threads x the kernel's count), or setmaxnreg.inc would never return.
template <typename K>
bool regs_fit(K kernel) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return false;
    return a.numRegs * 384 >= 128 * kBwdRegsLow + 256 * kBwdRegsHigh;
}

template <typename T, int D_QK, int D_V>
cudaError_t run_bwd(const BwdParams &p, const BwdMaps &m, cudaStream_t st) {
    const int64_t rows = (int64_t)p.b * p.s_q_pad * p.h_q;
    if (rows > 0) {
        const int64_t rows_per_block = 8 * (32 / (D_V / 8));
        bwd_dot_kernel<T><<<(unsigned)((rows + rows_per_block - 1) / rows_per_block), 256, 0, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    kernel_event(0, st);
    if (p.s_k > 0) {
        using CK = DkdvCfg<D_QK, D_V>;
        cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<T, D_QK, D_V>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, CK::SMEM);
        if (e != cudaSuccess) return e;
        const int64_t grid = (int64_t)((p.s_k + kBK - 1) / kBK) * p.h_kv * p.b;
        if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
        if (!regs_fit(bwd_dkdv_kernel<T, D_QK, D_V>)) return cudaErrorInvalidConfiguration;
        bwd_dkdv_kernel<T, D_QK, D_V><<<(unsigned)grid, 384, CK::SMEM, st>>>(m.k128, m.v128, m.q64, m.do64, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.s_q > 0) {
        using CQ = DqCfg<D_QK, D_V>;
        cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<T, D_QK, D_V>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, CQ::SMEM);
        if (e != cudaSuccess) return e;
        const int64_t grid = (int64_t)((p.s_q + kDqBM - 1) / kDqBM) * p.h_q * p.b;
        if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
        if (!regs_fit(bwd_dq_kernel<T, D_QK, D_V>)) return cudaErrorInvalidConfiguration;
        bwd_dq_kernel<T, D_QK, D_V><<<(unsigned)grid, 384, CQ::SMEM, st>>>(m.q128, m.do128, m.k64, m.v64, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    kernel_event(1, st);
    return cudaSuccess;
}

template <typename T>
cudaError_t dispatch_bwd(const BwdParams &p, const BwdMaps &m, cudaStream_t st) {
    if (p.d_qk == 64 && p.d_v == 64) return run_bwd<T, 64, 64>(p, m, st);
    if (p.d_qk == 128 && p.d_v == 128) return run_bwd<T, 128, 128>(p, m, st);
    if (p.d_qk == 192 && p.d_v == 128) return run_bwd<T, 192, 128>(p, m, st);
    return cudaErrorInvalidValue;
}

}  // namespace

bool bwd_supported(int d_qk, int d_v) {
    return (d_qk == 64 && d_v == 64) || (d_qk == 128 && d_v == 128) || (d_qk == 192 && d_v == 128);
}

cudaError_t launch_bwd(const BwdParams &p, const BwdMaps &m, int dtype, cudaStream_t st) {
    return dtype == FA_DTYPE_BF16 ? dispatch_bwd<__nv_bfloat16>(p, m, st) : dispatch_bwd<__half>(p, m, st);
}

}  // namespace fa
