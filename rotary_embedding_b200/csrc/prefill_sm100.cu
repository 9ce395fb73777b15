// prefill_sm100.cu -- prefill / chunked-prefill / dense attention forward on
// the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA computes a 128-row query tile against every key tile it may see:
//   out = softmax(scale * Q K^T + mask) V  with the online (rescaled) softmax
// of the "optimizing-attention-flash" page (IO-aware tiling, no S in HBM).
//
// Roles (warp specialisation, 8 warps):
//   warp 0      TMA producer: the Q tile once, then K_j / V_j 128-row tiles
//               into a ring of shared-memory stages (128-byte swizzled boxes).
//   warp 1      TMEM allocator and MMA issuer (one thread): S_j = Q K_j^T into
//               one of two TMEM S buffers, then O += P_{j-1} V_{j-1} with P
//               read from TMEM; order S_0, S_1, PV_0, S_2, PV_1, ... so the
//               tensor core works on S_{j+1} while the softmax runs on S_j.
//   warps 4-7   softmax warpgroup: thread t owns query row t of the tile
//               (TMEM lane t).  Loads its S row, applies the bottom-right
//               causal / sequence-end mask, keeps the running max (rescaling
//               O in TMEM only when the max grows by more than 2^8), writes
//               P = 2^(s*scale*log2e - m) as 16-bit values into TMEM, and at
//               the end normalises O and writes out and lse.
// Tiles are sized separately for d_qk (Q/K boxes) and d_v (V/O), so a
// 192/128 head (flash-attention PR #1604) pays for neither padding.
// Grouped-query heads (the page's Workflow 2 Step 3) are packed: when
// g = h_q / h_kv divides 128, the tile's rows are (query position, head)
// pairs of one kv head, loaded by one TMA box, so K/V tiles are shared by
// the g heads.
#include <algorithm>
#include <type_traits>

#include "fa_common.cuh"
#include "fa_internal.h"
#include "tcgen05.cuh"

namespace fa {

// Pairs out of every 8 whose 2^x the two-tile softmax evaluates on the FMA
// pipe (ex2_poly2) instead of the special function unit, in unmasked tiles.
// At d_qk <= 64 a key tile's scores cost little tensor time next to their
// exponentials and the special function unit bounds the softmax, so 2 of 8
// pairs move; at larger d_qk that unit has room and the polynomial's extra
// instructions only lengthen the softmax (measured: d_qk 192 3 % faster with
// none; d_qk 64 with the 56 / 224 register split: 2 of 8 1.6 % faster than 3
// on the non-causal grid and equal on the causal one, 4 of 8 slower).
#ifndef FA_EXP2_EMU_PAIRS
#define FA_EXP2_EMU_PAIRS 2
#endif
template <int D_QK>
constexpr int exp2_emu_pairs() { return D_QK <= 64 ? FA_EXP2_EMU_PAIRS : 0; }

constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 128;  // key rows per tile

// The grid is one-dimensional over (tile index, head group, batch entry) with
// the tile index slowest and taken from the last: under a causal mask the
// work of a query tile grows with its index, so every head's and batch
// entry's heaviest tiles start first and the light ones fill the last wave.
__device__ __forceinline__ void grid_order(const PrefillParams &p, int &tile, int &hgrp, int &b) {
    const int nhg = p.h_q / p.pack;
    const int per = nhg * p.b;                         // blocks per tile index
    const int L = (int)blockIdx.x;
    const int t = L / per, rem = L - t * per;
    tile = (int)gridDim.x / per - 1 - t;
    hgrp = rem % nhg;
    b = rem / nhg;
}

// Grids over a cache whose batch entries hold different numbers of keys:
// the (batch entry, query tile) items are ordered by their visible keys,
// heaviest first (longest processing time first, ties by index), all head
// groups of an item adjacent, so the tiles of the longest entries start in
// the first wave whatever their batch index.  The host uses it when the
// items number b x n_q_tiles <= 256; every CTA ranks them in `scratch` (m + 1
// ints of shared memory that no TMA has written yet), one block-wide pass.
__device__ __forceinline__ void work_order(const PrefillParams &p, int *scratch, int &tile, int &hgrp, int &b) {
    const int nhg = p.h_q / p.pack;
    const int n_t = p.n_q_tiles, m = p.b * n_t;
    const int rows = kBM / p.pack;
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
        const int bb = i / n_t, t = i - bb * n_t;
        const int L = seqlen_of(p.seqlens, p.seqlen_scalar, bb);
        int w = 0;
        const int i0 = t * rows;
        if (L >= 0 && (int64_t)L + p.s_new <= p.cap && i0 < p.s_q) {
            const int N = L + p.s_new;
            const int i_last = min(p.s_q, i0 + rows) - 1;
            int64_t f0, l0, f1, l1;
            visible_keys(i0, N, p.s_q, p.causal, p.win_left, p.win_right, f0, l0);
            visible_keys(i_last, N, p.s_q, p.causal, p.win_left, p.win_right, f1, l1);
            w = (int)max((int64_t)0, min((int64_t)N - 1, l1) - max((int64_t)0, f0) + 1);
        }
        scratch[i] = w;
    }
    __syncthreads();
    const int r = (int)blockIdx.x / nhg;
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
        const int wi = scratch[i];
        int rank = 0;
        for (int j = 0; j < m; ++j) {
            const int wj = scratch[j];
            rank += (wj > wi) || (wj == wi && j < i);
        }
        if (rank == r) scratch[m] = i;   // ranks are a permutation: exactly one item
    }
    __syncthreads();
    const int item = scratch[m];
    b = item / n_t;
    tile = item - b * n_t;
    hgrp = (int)blockIdx.x % nhg;
}

template <int D_QK, int D_V>
struct PrefillCfg {
    static constexpr int QBYTES = kBM * D_QK * 2;
    static constexpr int KBYTES = kBN * D_QK * 2;
    static constexpr int VBYTES = kBN * D_V * 2;
    static constexpr int QBOX = kBM * 128;   // bytes of one 64-column box of Q
    static constexpr int KBOX = kBN * 128;
    static constexpr int VBOX = kBN * 128;
    static constexpr int BUDGET = 224 * 1024;
    static constexpr int KST_RAW = (BUDGET - QBYTES) / (KBYTES + VBYTES);
    static constexpr int KST = KST_RAW > 4 ? 4 : KST_RAW;
    static constexpr int SMEM = 1024 + QBYTES + KST * (KBYTES + VBYTES) + 256;
    // TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D_V), P [384, 448)
    static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O = 256, T_P = 384;
    static_assert(KST >= 2, "at least two K/V stages");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(D_QK % 64 == 0 && D_V % 64 == 0 && D_V <= 128, "head dims");
};

template <typename T, int D_QK, int D_V>
__global__ void __launch_bounds__(256, 1) prefill_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                         const __grid_constant__ CUtensorMap tmK,
                                                         const __grid_constant__ CUtensorMap tmV,
                                                         const PrefillParams p) {
    using C = PrefillCfg<D_QK, D_V>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = sQ + C::QBYTES;                 // KST stages of K
    uint8_t *sV = sK + C::KST * C::KBYTES;        // KST stages of V
    uint64_t *bars = reinterpret_cast<uint64_t *>(sV + C::KST * C::VBYTES);
    uint64_t *q_full = bars;                      // 1
    uint64_t *k_full = bars + 1;                  // KST
    uint64_t *v_full = k_full + C::KST;           // KST
    uint64_t *kv_empty = v_full + C::KST;         // KST
    uint64_t *s_full = kv_empty + C::KST;         // 2
    uint64_t *s_free = s_full + 2;                // 2
    uint64_t *p_full = s_free + 2;                // 1
    uint64_t *pv_done = p_full + 1;               // 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pv_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // heaviest causal tiles first across every head and batch entry: block L
    // takes tile n - 1 - L / (head groups x batch)
    int qt, hgrp, b;
    if (p.work_order)
        work_order(p, reinterpret_cast<int *>(sK), qt, hgrp, b);
    else
        grid_order(p, qt, hgrp, b);
    const int pack = p.pack;
    const int hq0 = hgrp * pack;                           // first query head of the tile
    const int hk = hq0 / p.g;
    const int i0 = qt * (kBM / pack);                      // first query position

    // keys N, query rows sq of this CTA's sequence, and the row offsets of a
    // packed (varlen) sequence: b is then the sequence, whose rows
    // qoff .. and koff .. sit in batch entry 0 of the packed tensors
    int N, sq = p.s_q, qoff = 0, koff = 0, tb = b;
    if (p.cu_q) {
        qoff = __ldg(p.cu_q + b);
        sq = __ldg(p.cu_q + b + 1) - qoff;
        koff = __ldg(p.cu_k + b);
        N = __ldg(p.cu_k + b + 1) - koff;
        tb = 0;
        // device-side preconditions: the sequence lies inside the packed rows
        if (qoff < 0 || sq < 0 || (int64_t)qoff + sq > p.total_q || koff < 0 || N < 0 ||
            (int64_t)koff + N > p.total_k) {
            if (threadIdx.x == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
            return;
        }
    } else if (p.kvcache) {
        const int L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
        if (L < 0 || (int64_t)L + p.s_new > p.cap) {
            if (threadIdx.x == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
            return;
        }
        N = L + p.s_new;
    } else {
        N = (int)p.s_k;
    }
    if (i0 >= sq) return;                                  // past this sequence's rows
    const int i_last = min(sq, i0 + kBM / pack) - 1;
    // visible keys of the tile's first and last query rows (causal, window)
    int64_t f_first, l_first, f_last, l_last;
    visible_keys(i0, N, sq, p.causal, p.win_left, p.win_right, f_first, l_first);
    visible_keys(i_last, N, sq, p.causal, p.win_left, p.win_right, f_last, l_last);
    const int kv_end = (int)max((int64_t)0, min((int64_t)N, l_last + 1));
    const int n_kv = (kv_end + kBN - 1) / kBN;
    const int kb = min((int)(f_first / kBN), n_kv);        // first key tile any row sees
    const int nblk = n_kv - kb;                             // key tiles kb .. n_kv - 1
    // key tiles that need an element mask: past the first row's last visible
    // key (diagonal band, right window or sequence end) or before the last
    // row's first visible key (left window)
    const int mask_from = (int)max((int64_t)0, min((int64_t)N, l_first + 1));
    const int lo_max = (int)f_last;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::KST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
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

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && nblk > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(q_full, C::QBYTES);
#pragma unroll
            for (int c = 0; c < D_QK / 64; ++c) tma_load_4d(sQ + c * C::QBOX, &tmQ, q_full, c * 64, hq0, qoff + i0, tb);
            for (int t = 0; t < nblk; ++t) {
                const int j = kb + t;
                const int st = t % C::KST;
                if (t >= C::KST && !mbar_wait(&kv_empty[st], ((t / C::KST) - 1) & 1, p.status)) break;
                mbar_arrive_expect_tx(&k_full[st], C::KBYTES);
#pragma unroll
                for (int c = 0; c < D_QK / 64; ++c)
                    tma_load_4d(sK + st * C::KBYTES + c * C::KBOX, &tmK, &k_full[st], c * 64, hk, koff + j * kBN, tb);
                mbar_arrive_expect_tx(&v_full[st], C::VBYTES);
#pragma unroll
                for (int c = 0; c < D_V / 64; ++c)
                    tma_load_4d(sV + st * C::VBYTES + c * C::VBOX, &tmV, &v_full[st], c * 64, hk, koff + j * kBN, tb);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && nblk > 0) {
            const uint32_t idesc_qk = tc::idesc_f16(bf16, kBM, kBN, false);
            const uint32_t idesc_pv = tc::idesc_f16(bf16, kBM, D_V, true);
            const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV);
            bool ok = mbar_wait(q_full, 0, p.status);
            // tt: index of the key tile relative to kb (stages, parities)
            auto issue_pv = [&](int tt) -> bool {
                const int st = tt % C::KST;
                if (!mbar_wait(p_full, tt & 1, p.status)) return false;
                if (!mbar_wait(&v_full[st], (tt / C::KST) & 1, p.status)) return false;
                tc::fence_after_sync();
#pragma unroll
                for (int k = 0; k < kBN / 16; ++k) {
                    const uint64_t bdesc = tc::smem_desc(aV + st * C::VBYTES + k * 16 * 128, C::VBOX, 1024);
                    tc::mma_ts(tmem + C::T_O, tmem + C::T_P + k * 8, bdesc, idesc_pv, (tt > 0 || k > 0) ? 1u : 0u);
                }
                tc::commit(&kv_empty[st]);
                tc::commit(pv_done);
                return true;
            };
            for (int t = 0; t < nblk && ok; ++t) {
                const int st = t % C::KST, sb = t & 1;
                if (!mbar_wait(&k_full[st], (t / C::KST) & 1, p.status)) break;
                if (t >= 2 && !mbar_wait(&s_free[sb], ((t >> 1) - 1) & 1, p.status)) break;
                tc::fence_after_sync();
#pragma unroll
                for (int k = 0; k < D_QK / 16; ++k) {
                    const uint64_t adesc = tc::smem_desc(aQ + (k >> 2) * C::QBOX + (k & 3) * 32, 16, 1024);
                    const uint64_t bdesc =
                        tc::smem_desc(aK + st * C::KBYTES + (k >> 2) * C::KBOX + (k & 3) * 32, 16, 1024);
                    tc::mma_ss(tmem + (sb ? C::T_S1 : C::T_S0), adesc, bdesc, idesc_qk, k > 0 ? 1u : 0u);
                }
                tc::commit(&s_full[sb]);
                if (t >= 1 && !issue_pv(t - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) issue_pv(nblk - 1);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax warpgroup
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;                  // tile row = TMEM lane
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int prow = qt * kBM + r;                 // packed row
        const int i = prow / pack;                     // query position
        const int hq = hq0 + (prow % pack);
        const bool row_valid = i < sq;
        int64_t fv64, lv64;
        visible_keys(i, N, sq, p.causal, p.win_left, p.win_right, fv64, lv64);
        const int last_vis = row_valid ? (int)lv64 : -1;
        const int first_vis = (int)fv64;
        const float c = p.scale_log2;
        float m_ref = -INFINITY;   // raw-score max used as the exponent reference
        float l = 0.f;
        bool ok = true;
        for (int t = 0; t < nblk && ok; ++t) {
            const int j = kb + t;
            const int sb = t & 1;
            if (!mbar_wait(&s_full[sb], (t >> 1) & 1, p.status)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            uint32_t sr[4][32];
            const uint32_t s_addr = tmem + lane_addr + (sb ? C::T_S1 : C::T_S0);
            tc::ld32(s_addr, sr[0]);
            tc::ld32(s_addr + 32, sr[1]);
            tc::ld32(s_addr + 64, sr[2]);
            tc::ld32(s_addr + 96, sr[3]);
            tc::wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);

            const int j0 = j * kBN;
            float mt = -INFINITY;
            if (j0 + kBN > mask_from || j0 < lo_max) {
#pragma unroll
                for (int h = 0; h < 4; ++h)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int key = j0 + h * 32 + e;
                        float v = __uint_as_float(sr[h][e]);
                        v = (key <= last_vis && key >= first_vis) ? v : -INFINITY;
                        sr[h][e] = __float_as_uint(v);
                        mt = fmaxf(mt, v);
                    }
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h)
#pragma unroll
                    for (int e = 0; e < 32; ++e) mt = fmaxf(mt, __uint_as_float(sr[h][e]));
            }
            // lazy rescale: move the reference only when the max grows by > 2^8
            float alpha = 1.f;
            bool rescale = false;
            if (mt > m_ref && (m_ref == -INFINITY || (mt - m_ref) * c > 8.f)) {
                alpha = m_ref == -INFINITY ? 0.f : ex2((m_ref - mt) * c);
                rescale = m_ref != -INFINITY;
                m_ref = mt;
            }
            const float mc = m_ref == -INFINITY ? 0.f : m_ref * c;
            uint32_t pk[2][32];
            float rs = 0.f;
#pragma unroll
            for (int h = 0; h < 4; ++h)
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float p0 = ex2(fmaf(__uint_as_float(sr[h][e]), c, -mc));
                    const float p1 = ex2(fmaf(__uint_as_float(sr[h][e + 1]), c, -mc));
                    rs += p0 + p1;
                    pk[h >> 1][(h & 1) * 16 + (e >> 1)] = Elem<T>::pack2(p0, p1);
                }
            l = l * alpha + rs;

            if (t > 0) {
                // O is stable and the P buffer free once PV_{j-1} has completed
                if (!mbar_wait(pv_done, (t - 1) & 1, p.status)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                    for (int h = 0; h < D_V / 32; ++h) {
                        uint32_t orr[32];
                        const uint32_t o_addr = tmem + lane_addr + C::T_O + h * 32;
                        tc::ld32(o_addr, orr);
                        tc::wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                        tc::st32(o_addr, orr);
                    }
                }
            }
            tc::st32(tmem + lane_addr + C::T_P, pk[0]);
            tc::st32(tmem + lane_addr + C::T_P + 32, pk[1]);
            tc::wait_st();
            if (p.kvcache && t == nblk - 1 && j0 + kBN > N) {
                // cache rows past N_b may hold anything: zero them in the V tile
                const int st = t % C::KST;
                if (!mbar_wait(&v_full[st], (t / C::KST) & 1, p.status)) {
                    ok = false;
                    break;
                }
                uint8_t *vt = sV + st * C::VBYTES;
                const int first = N - j0;
                const int n16 = (kBN - first) * 8 * (D_V / 64);
                for (int idx = threadIdx.x - 128; idx < n16; idx += 128) {
                    const int box = idx / ((kBN - first) * 8);
                    const int rem = idx % ((kBN - first) * 8);
                    *reinterpret_cast<uint4 *>(vt + box * C::VBOX + (first + rem / 8) * 128 + (rem % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ------------------------------------------------ epilogue
        if (ok && nblk > 0 && !mbar_wait(pv_done, (nblk - 1) & 1, p.status)) ok = false;
        tc::fence_after_sync();
        // every lane takes part in the (warp-collective) TMEM loads; only rows
        // inside the sequence are stored
        T *orow = static_cast<T *>(p.out) + tb * p.os.b + (int64_t)(qoff + i) * p.os.s + hq * p.os.h;
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int h = 0; h < D_V / 32; ++h) {
            uint32_t orr[32];
            if (nblk > 0) {
                tc::ld32(tmem + lane_addr + C::T_O + h * 32, orr);
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
                    for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(orr[e + u]) * inv;
                    reinterpret_cast<uint4 *>(orow + h * 32 + e)[0] = pack8<T>(f);
                }
            }
        }
        if (row_valid && p.lse)
            p.lse[p.cu_q ? (int64_t)hq * p.total_q + qoff + i : ((int64_t)b * p.h_q + hq) * sq + i] = l > 0.f ? (m_ref * c + log2f(l)) * kLn2 : -INFINITY;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ============================================================================
// Two query tiles per CTA (256 query rows), two softmax warpgroups.
//
// Each tile x has its own S buffer, its own P buffer and its own O
// accumulator in TMEM, so the tensor core never waits for a softmax to hand
// back S: as soon as softmax warpgroup x has loaded S_x(j) into registers
// (s_free), the MMA warp issues QK_x(j+1) into the same S buffer, and the
// tensor core computes the next scores while the softmax turns the current
// ones into P.  Per key tile j the MMA warp issues, in order,
//   QK_0(j+1)  QK_1(j+1)  PV_0(j)  PV_1(j)
// each after its operands are ready (K(j+1) loaded and S_x(j) consumed; V(j)
// loaded and P_x(j) written).  PV_x(j) commits pv_done[x]; the softmax waits
// for it before writing P_x(j+1) over P_x(j) or rescaling O_x, and before the
// epilogue reads O_x.
//
// TMEM columns (512): S_x at x BN, P_x (16-bit pairs, BN/2 columns) after
// both S buffers, O_x in the last 2 d_v columns.  That fits with BN = 128
// key rows when d_v <= 64 and with BN = 80 otherwise (3 BN + 2 d_v <= 512).
//
// Warps: 0 TMA, 1 MMA, 2-3 idle (warpgroup 0), 4-7 softmax of tile 0
// (warpgroup 1), 8-11 softmax of tile 1 (warpgroup 2); warp w reaches TMEM
// lanes 32 (w % 4) .. 32 (w % 4) + 31.
//
// KSPLIT: on grids too small for two tiles per CTA, the two "tiles" of a CTA
// are the same 128 query rows with the key range cut in two: softmax
// warpgroup 0 takes the first half of the visible key tiles, warpgroup 1
// the second, each with its own S, P, O, running max and sum, over one Q
// tile.  Per step u the K tiles of both halves are loaded, then their V
// tiles, and the MMA warp keeps the order QK_0(u+1) QK_1(u+1) PV_0(u) PV_1(u).
// At the end the two warpgroups exchange (max, sum) per row through shared
// memory (the unused second Q buffer) and each merges half of the output
// columns from both O accumulators:
//   out = (2^(m0 - m) O_0 + 2^(m1 - m) O_1) / (2^(m0 - m) l0 + 2^(m1 - m) l1).
// The CTA count doubles against pairs of tiles, and both warpgroups stay
// busy on every step, which pairs of causal tiles of unequal length do not.
//
// The register file is split with setmaxnreg: warpgroup 0 drops to 56
// registers per thread (enough for the TMA and MMA issue loops), the two
// softmax warpgroups rise to 224 so that a whole S row stays in registers
// (128 x 56 + 256 x 224 = 64512, exactly the 384 x 168 the block is launched
// with; against 64 / 216: MLA prefill 3 % faster, d 128 prefill 1-2 %).
// ============================================================================
template <int D_QK, int D_V>
struct Prefill2Cfg {
    static constexpr int BN = D_V <= 64 ? 128 : 80;  // key rows per tile
    static constexpr int QBYTES = kBM * D_QK * 2;   // per tile
    static constexpr int KBYTES = BN * D_QK * 2;
    static constexpr int VBYTES = BN * D_V * 2;
    static constexpr int QBOX = kBM * 128;           // bytes of one 64-column box of a Q tile
    static constexpr int KBOX = BN * 128;            // ... of a K or V tile
    static constexpr int BUDGET = 224 * 1024;
    static constexpr int AVAIL = BUDGET - 2 * QBYTES;
    static constexpr bool EVEN = AVAIL >= 2 * (KBYTES + VBYTES);
    static constexpr int KS_RAW = AVAIL / (KBYTES + VBYTES);
    static constexpr int KST = EVEN ? (KS_RAW > 3 ? 3 : KS_RAW) : 2;
    static constexpr int VST = EVEN ? KST : (AVAIL - 2 * KBYTES) / VBYTES;
    static constexpr int SMEM = 1024 + 2 * QBYTES + KST * KBYTES + VST * VBYTES + 256;
    static constexpr int PCOLS = ((BN / 2) + 15) / 16 * 16;   // P columns per tile, 16-aligned
    static __device__ __forceinline__ uint32_t t_s(int x) { return (uint32_t)(x * BN); }
    static __device__ __forceinline__ uint32_t t_p(int x) { return (uint32_t)(2 * BN + x * PCOLS); }
    static __device__ __forceinline__ uint32_t t_o(int x) { return (uint32_t)(512 - 2 * D_V + x * D_V); }
    static_assert(2 * BN + 2 * PCOLS <= 512 - 2 * D_V, "TMEM: S, P and O of both tiles");
    static_assert(BN % 16 == 0 && KBOX % 1024 == 0, "key tile rows");
    static_assert(VST >= 1 && KST >= 2, "K/V ring");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(D_QK % 64 == 0 && D_V % 64 == 0 && D_V <= 128, "head dims");
};

template <typename T, int D_QK, int D_V, bool KSPLIT>
__global__ void __launch_bounds__(384, 1) prefill2_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                          const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const PrefillParams p) {
    using C = Prefill2Cfg<D_QK, D_V>;
    constexpr int KST = C::KST, VST = C::VST, BN = C::BN;
    // the split order loads two K tiles ahead of the V tiles they pair with
    static_assert(!KSPLIT || (KST >= 2 && VST >= 2), "key-split rings");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                              // 2 tiles
    uint8_t *sK = sQ + 2 * C::QBYTES;
    uint8_t *sV = sK + KST * C::KBYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sV + VST * C::VBYTES);
    uint64_t *q_full = bars;                // 1
    uint64_t *k_full = bars + 1;            // KST
    uint64_t *k_empty = k_full + KST;       // KST
    uint64_t *v_full = k_empty + KST;       // VST
    uint64_t *v_empty = v_full + VST;       // VST
    uint64_t *s_full = v_empty + VST;       // 2: QK_x(j) complete
    uint64_t *s_free = s_full + 2;          // 2: softmax x holds S_x(j) in registers
    uint64_t *p_full = s_free + 2;          // 2: P_x(j) written
    uint64_t *pv_done = p_full + 2;         // 2: PV_x(j) complete
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pv_done + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // heaviest causal blocks first across every head and batch entry
    int blk, hgrp, b;
    if (KSPLIT && p.work_order)
        work_order(p, reinterpret_cast<int *>(sK), blk, hgrp, b);
    else
        grid_order(p, blk, hgrp, b);
    const int pack = p.pack;
    const int hq0 = hgrp * pack;
    const int hk = hq0 / p.g;
    const int rows_per_tile = kBM / pack;                   // query positions per tile

    // keys N, query rows sq of this CTA's sequence, and the row offsets of a
    // packed (varlen) sequence: b is then the sequence, whose rows
    // qoff .. and koff .. sit in batch entry 0 of the packed tensors
    int N, sq = p.s_q, qoff = 0, koff = 0, tb = b;
    if (p.cu_q) {
        qoff = __ldg(p.cu_q + b);
        sq = __ldg(p.cu_q + b + 1) - qoff;
        koff = __ldg(p.cu_k + b);
        N = __ldg(p.cu_k + b + 1) - koff;
        tb = 0;
        // device-side preconditions: the sequence lies inside the packed rows
        if (qoff < 0 || sq < 0 || (int64_t)qoff + sq > p.total_q || koff < 0 || N < 0 ||
            (int64_t)koff + N > p.total_k) {
            if (threadIdx.x == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
            return;
        }
    } else if (p.kvcache) {
        const int L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
        if (L < 0 || (int64_t)L + p.s_new > p.cap) {
            if (threadIdx.x == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
            return;
        }
        N = L + p.s_new;
    } else {
        N = (int)p.s_k;
    }
    // the CTA's two query tiles: 2 blk and 2 blk + 1, or blk and
    // n_q_tiles - 1 - blk (the middle tile of an odd count pairs with an
    // empty tile past the rows); every tile index is taken exactly once
    int tile[2];
    if (KSPLIT) {
        tile[0] = tile[1] = blk;                           // one query tile, two key halves
    } else if (p.pair_ends) {
        tile[0] = blk;
        tile[1] = p.n_q_tiles - 1 - blk > blk ? p.n_q_tiles - 1 - blk : p.n_q_tiles;
    } else {
        tile[0] = 2 * blk;
        tile[1] = 2 * blk + 1;
    }
    if (tile[0] * rows_per_tile >= sq) return;             // past this sequence's rows (tile[1] > tile[0])
    // per tile: key tiles kb[x] .. n_kv[x] - 1 (causal, window), and the
    // bounds past which a key tile needs an element mask (see prefill_kernel)
    int i0[2], n_kv[2], kb[2], mask_from[2], lo_max[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        i0[x] = tile[x] * rows_per_tile;
        const int i_last = min(sq, i0[x] + rows_per_tile) - 1;
        int64_t f_first, l_first, f_last, l_last;
        visible_keys(i0[x], N, sq, p.causal, p.win_left, p.win_right, f_first, l_first);
        visible_keys(i_last, N, sq, p.causal, p.win_left, p.win_right, f_last, l_last);
        const int kv_end = i0[x] >= sq ? 0 : (int)max((int64_t)0, min((int64_t)N, l_last + 1));
        n_kv[x] = (kv_end + BN - 1) / BN;
        kb[x] = min((int)(f_first / BN), n_kv[x]);
        mask_from[x] = (int)max((int64_t)0, min((int64_t)N, l_first + 1));
        lo_max[x] = (int)f_last;
    }
    if (KSPLIT) {
        // halves kb .. mid - 1 and mid .. end - 1 (the first half holds the odd tile)
        const int mid = kb[0] + (n_kv[0] - kb[0] + 1) / 2;
        kb[1] = mid;
        n_kv[0] = mid;
    }
    // tiles of each half (key-split mode)
    const int n_x[2] = {n_kv[0] - kb[0], n_kv[1] - kb[1]};
    // key tiles loaded: kb0 .. n_all - 1 (the union of both tiles' ranges)
    const bool any0 = kb[0] < n_kv[0], any1 = kb[1] < n_kv[1];
    const int kb0 = any0 && any1 ? min(kb[0], kb[1]) : (any0 ? kb[0] : (any1 ? kb[1] : 0));
    const int n_all = max(any0 ? n_kv[0] : 0, any1 ? n_kv[1] : 0);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s_full[x], 1);
            mbar_init(&s_free[x], 4);
            mbar_init(&p_full[x], 4);
            mbar_init(&pv_done[x], 1);
        }
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

    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (KSPLIT && lane == 0 && n_x[0] > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(q_full, C::QBYTES);
#pragma unroll
            for (int c = 0; c < D_QK / 64; ++c)
                tma_load_4d(sQ + c * C::QBOX, &tmQ, q_full, c * 64, hq0, qoff + i0[0], tb);
            // load index 2u + x for step u of half x: the K tiles of a step,
            // then its V tiles
            bool ok = true;
            for (int u = 0; u < n_x[0] && ok; ++u) {
#pragma unroll 1
                for (int x = 0; x < 2; ++x) {
                    if (u >= n_x[x] || !ok) continue;
                    const int li = 2 * u + x, ks = li % KST;
                    if (li >= KST && !(ok = mbar_wait(&k_empty[ks], ((li / KST) - 1) & 1, p.status))) break;
                    mbar_arrive_expect_tx(&k_full[ks], C::KBYTES);
#pragma unroll
                    for (int c = 0; c < D_QK / 64; ++c)
                        tma_load_4d(sK + ks * C::KBYTES + c * C::KBOX, &tmK, &k_full[ks], c * 64, hk,
                                    koff + (kb[x] + u) * BN, tb);
                }
#pragma unroll 1
                for (int x = 0; x < 2; ++x) {
                    if (u >= n_x[x] || !ok) continue;
                    const int li = 2 * u + x, vs = li % VST;
                    if (li >= VST && !(ok = mbar_wait(&v_empty[vs], ((li / VST) - 1) & 1, p.status))) break;
                    mbar_arrive_expect_tx(&v_full[vs], C::VBYTES);
#pragma unroll
                    for (int c = 0; c < D_V / 64; ++c)
                        tma_load_4d(sV + vs * C::VBYTES + c * C::KBOX, &tmV, &v_full[vs], c * 64, hk,
                                    koff + (kb[x] + u) * BN, tb);
                }
            }
        } else if (!KSPLIT && lane == 0 && n_all > kb0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(q_full, 2 * C::QBYTES);
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int c = 0; c < D_QK / 64; ++c)
                    tma_load_4d(sQ + x * C::QBYTES + c * C::QBOX, &tmQ, q_full, c * 64, hq0, qoff + i0[x], tb);
            for (int j = kb0; j < n_all; ++j) {
                const int u = j - kb0;   // loaded tile index (stages, parities)
                const int ks = u % KST, vs = u % VST;
                if (u >= KST && !mbar_wait(&k_empty[ks], ((u / KST) - 1) & 1, p.status)) break;
                mbar_arrive_expect_tx(&k_full[ks], C::KBYTES);
#pragma unroll
                for (int c = 0; c < D_QK / 64; ++c)
                    tma_load_4d(sK + ks * C::KBYTES + c * C::KBOX, &tmK, &k_full[ks], c * 64, hk, koff + j * BN, tb);
                if (u >= VST && !mbar_wait(&v_empty[vs], ((u / VST) - 1) & 1, p.status)) break;
                mbar_arrive_expect_tx(&v_full[vs], C::VBYTES);
#pragma unroll
                for (int c = 0; c < D_V / 64; ++c)
                    tma_load_4d(sV + vs * C::VBYTES + c * C::KBOX, &tmV, &v_full[vs], c * 64, hk, koff + j * BN, tb);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // The whole warp runs the loop (waits, warp-uniform descriptors); one
        // elected lane issues the MMAs and the commits that track them.
        if (KSPLIT ? n_x[0] > 0 : n_all > kb0) {
            const bool leader = tc::elect_one();
            const uint32_t idesc_qk = tc::idesc_f16(bf16, kBM, BN, false);
            const uint32_t idesc_pv = tc::idesc_f16(bf16, kBM, D_V, true);
            // Descriptors of the first k-step of every operand buffer; a k-step
            // only moves the start address (low 14 bits, 16-byte units), so the
            // issue loop adds a compile-time constant per MMA.
            const uint64_t dQ0 = tc::smem_desc(smem_addr(sQ), 16, 1024);
            const uint64_t dK0 = tc::smem_desc(smem_addr(sK), 16, 1024);
            const uint64_t dV0 = tc::smem_desc(smem_addr(sV), C::KBOX, 1024);
            bool ok = mbar_wait(q_full, 0, p.status);
            auto in_range = [&](int x, int j) { return j >= kb[x] && j < n_kv[x]; };
            // K tile in stage ks (key-split mode: both halves read the one Q tile)
            auto issue_qk_s = [&](int x, int ks) {
                const uint64_t dq = dQ0 + (uint64_t)(((KSPLIT ? 0 : x) * C::QBYTES) >> 4);
                const uint64_t dk = dK0 + (uint64_t)((ks * C::KBYTES) >> 4);
                const uint32_t ts = tmem + C::t_s(x);
                if (leader) {
#pragma unroll
                    for (int k = 0; k < D_QK / 16; ++k) {
                        const uint64_t qoff = (uint64_t)((((k >> 2) * C::QBOX) + (k & 3) * 32) >> 4);
                        const uint64_t koff = (uint64_t)((((k >> 2) * C::KBOX) + (k & 3) * 32) >> 4);
                        tc::mma_ss(ts, dq + qoff, dk + koff, idesc_qk, k > 0 ? 1u : 0u);
                    }
                    tc::commit(&s_full[x]);
                }
                __syncwarp();
            };
            // key tile j sits in stage (j - kb0) % KST / VST
            auto issue_qk = [&](int x, int j) { issue_qk_s(x, (j - kb0) % KST); };
            auto issue_pv_s = [&](int x, int vs, bool first) {
                const uint64_t dv = dV0 + (uint64_t)((vs * C::VBYTES) >> 4);
                const uint32_t to = tmem + C::t_o(x), tp = tmem + C::t_p(x);
                const uint32_t acc0 = first ? 0u : 1u;
                if (leader) {
#pragma unroll
                    for (int k = 0; k < BN / 16; ++k)
                        tc::mma_ts(to, tp + k * 8, dv + (uint64_t)(k * 16 * 128 / 16), idesc_pv, k > 0 ? 1u : acc0);
                    tc::commit(&pv_done[x]);
                }
                __syncwarp();
            };
            auto issue_pv = [&](int x, int j) { issue_pv_s(x, (j - kb0) % VST, j == kb[x]); };
            auto commit = [&](uint64_t *bar) {
                if (leader) tc::commit(bar);
                __syncwarp();
            };
            if (KSPLIT) {
                // step u of half x: load index 2u + x (see the producer)
                for (int x = 0; x < 2 && ok; ++x) {
                    if (n_x[x] <= 0) continue;
                    const int ks = x % KST;
                    if (!(ok = mbar_wait(&k_full[ks], (x / KST) & 1, p.status))) break;
                    tc::fence_after_sync();
                    issue_qk_s(x, ks);
                    commit(&k_empty[ks]);
                }
                for (int u = 0; u < n_x[0] && ok; ++u) {
                    // the next scores of both halves, once S_x(u) is consumed
#pragma unroll 1
                    for (int x = 0; x < 2; ++x) {
                        if (u + 1 >= n_x[x] || !ok) continue;
                        const int li = 2 * (u + 1) + x, ks = li % KST;
                        if (!(ok = mbar_wait(&k_full[ks], (li / KST) & 1, p.status))) break;
                        if (!(ok = mbar_wait(&s_free[x], u & 1, p.status))) break;
                        tc::fence_after_sync();
                        issue_qk_s(x, ks);
                        commit(&k_empty[ks]);
                    }
                    // this step's PV of both halves
#pragma unroll 1
                    for (int x = 0; x < 2; ++x) {
                        if (u >= n_x[x] || !ok) continue;
                        const int li = 2 * u + x, vs = li % VST;
                        if (!(ok = mbar_wait(&v_full[vs], (li / VST) & 1, p.status))) break;
                        if (!(ok = mbar_wait(&p_full[x], u & 1, p.status))) break;
                        tc::fence_after_sync();
                        issue_pv_s(x, vs, u == 0);
                        commit(&v_empty[vs]);
                    }
                }
            } else {
            // prologue: QK of the tiles whose range starts at the first loaded key tile
            if (ok && (ok = mbar_wait(&k_full[0], 0, p.status))) {
                tc::fence_after_sync();
                if (in_range(0, kb0)) issue_qk(0, kb0);
                if (in_range(1, kb0)) issue_qk(1, kb0);
                commit(&k_empty[0]);
            }
            for (int j = kb0; j < n_all && ok; ++j) {
                const int u = j - kb0;
                const bool next = j + 1 < n_all;
                // the next scores: QK_x(j+1) once K(j+1) is in and S_x(j) is consumed
                if (next) {
                    const int ks1 = (u + 1) % KST;
                    if (!(ok = mbar_wait(&k_full[ks1], ((u + 1) / KST) & 1, p.status))) break;
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        if (!in_range(x, j + 1)) continue;
                        if (in_range(x, j) && !(ok = mbar_wait(&s_free[x], (j - kb[x]) & 1, p.status))) break;
                        tc::fence_after_sync();
                        issue_qk(x, j + 1);
                    }
                    if (!ok) break;
                    commit(&k_empty[ks1]);
                }
                // this tile's PV: P_x(j) V(j) once V(j) is in and P_x(j) is written
                const int vs = u % VST;
                if (!(ok = mbar_wait(&v_full[vs], (u / VST) & 1, p.status))) break;
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (!in_range(x, j)) continue;
                    if (!(ok = mbar_wait(&p_full[x], (j - kb[x]) & 1, p.status))) break;
                    tc::fence_after_sync();
                    issue_pv(x, j);
                }
                if (!ok) break;
                commit(&v_empty[vs]);
            }
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax warpgroups
        asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
        const int x = (warp - 4) >> 2;                 // tile of this warpgroup
        const int q4 = warp & 3;                       // TMEM lane quadrant this warp may access
        const int r = q4 * 32 + lane;                  // tile row = TMEM lane
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int prow = tile[x] * kBM + r;            // packed row
        const int i = prow / pack;
        const int hq = hq0 + (prow % pack);
        const bool row_valid = i < sq;
        int64_t fv64, lv64;
        visible_keys(i, N, sq, p.causal, p.win_left, p.win_right, fv64, lv64);
        const int last_vis = row_valid ? (int)lv64 : -1;
        const int first_vis = (int)fv64;
        const float c = p.scale_log2;
        const uint64_t c2 = f2_pack(c, c);
        const uint32_t s_addr = tmem + lane_addr + C::t_s(x);
        const uint32_t p_addr = tmem + lane_addr + C::t_p(x);
        const uint32_t o_addr = tmem + lane_addr + C::t_o(x);
        const int nk = n_kv[x], jb = kb[x], mfrom = mask_from[x], lmax = lo_max[x];
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = jb; j < nk && ok; ++j) {
            if (!(ok = mbar_wait(&s_full[x], (j - jb) & 1, p.status))) break;
            tc::fence_after_sync();
            const int j0 = j * BN;
            // the S row: NCH chunks of 32 columns and, when BN % 32 = 16, a
            // 16-column tail (every index below is a compile-time constant)
            constexpr int NCH = BN / 32, TAIL = BN % 32;
            uint32_t sr[NCH][32];
            uint32_t st[TAIL > 0 ? TAIL : 2];
#pragma unroll
            for (int h = 0; h < NCH; ++h) tc::ld32(s_addr + h * 32, sr[h]);
            if constexpr (TAIL == 16) tc::ld16(s_addr + NCH * 32, st);
            tc::wait_ld();
            // S_x(j) is in registers: the MMA warp may compute S_x(j+1) over it
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[x]);
            const bool masked = j0 + BN > mfrom || j0 < lmax;
            if (masked) {
                // diagonal band, window edge or sequence end: -inf outside the
                // visible keys (only these tiles pay for the comparisons)
#pragma unroll
                for (int h = 0; h < NCH; ++h)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int key = j0 + 32 * h + e;
                        if (key > last_vis || key < first_vis) sr[h][e] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                for (int e = 0; e < TAIL; ++e) {
                    const int key = j0 + 32 * NCH + e;
                    if (key > last_vis || key < first_vis) st[e] = __float_as_uint(-INFINITY);
                }
            }
            // row max: four independent three-input chains
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int h = 0; h < NCH; ++h)
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(sr[h][e]), __uint_as_float(sr[h][e + 1]));
#pragma unroll
            for (int e = 0; e < TAIL; e += 2)
                mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(st[e]), __uint_as_float(st[e + 1]));
            const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            float alpha = 1.f;
            bool rescale = false;
            if (mt > m_ref && (m_ref == -INFINITY || (mt - m_ref) * c > 8.f)) {
                alpha = m_ref == -INFINITY ? 0.f : ex2((m_ref - mt) * c);
                rescale = m_ref != -INFINITY;
                m_ref = mt;
            }
            const float mc = m_ref == -INFINITY ? 0.f : m_ref * c;
            const uint64_t nmc2 = f2_pack(-mc, -mc);
            // P_x(j-1) has been read and O_x updated by PV_x(j-1)
            if (j > jb) {
                if (!(ok = mbar_wait(&pv_done[x], (j - 1 - jb) & 1, p.status))) break;
                tc::fence_after_sync();
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int h = 0; h < D_V / 32; ++h) {
                    uint32_t orr[32];
                    tc::ld32(o_addr + h * 32, orr);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                    tc::st32(o_addr + h * 32, orr);
                }
            }
            // P = 2^(s c - m c) as 16-bit pairs into the P buffer (keys
            // [2k, 2k+2) -> column k).  In tiles without masked keys and at
            // d_qk <= 64, exp2_emu_pairs() of every 8 pairs (2) take 2^x on
            // the FMA pipe (ex2_poly2) and the rest on the special function
            // unit; masked tiles need exact zeros and use the special
            // function unit throughout.  The fp32 P values overwrite S
            // in registers; the row sum is taken after P has been handed to
            // the MMA warp (off the critical path).
            // one pair of scores (a, b) -> P values in place, packed 16-bit pair returned
            auto exp_pair = [&](auto split, uint32_t &a, uint32_t &b, int q) -> uint32_t {
                const uint64_t t = f2_fma(f2_pack(__uint_as_float(a), __uint_as_float(b)), c2, nmc2);
                float t0, t1, p0, p1;
                f2_unpack(t, t0, t1);
                if (decltype(split)::value && (q & 7) < exp2_emu_pairs<D_QK>()) {
                    f2_unpack(ex2_poly2(t0, t1), p0, p1);
                } else {
                    p0 = ex2(t0);
                    p1 = ex2(t1);
                }
                a = __float_as_uint(p0);
                b = __float_as_uint(p1);
                return Elem<T>::pack2(p0, p1);
            };
            auto exp_row = [&](auto split) {
#pragma unroll
                for (int h = 0; h < NCH; ++h) {
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) pk[q] = exp_pair(split, sr[h][2 * q], sr[h][2 * q + 1], q);
                    tc::st16(p_addr + 16 * h, pk);
                }
                if constexpr (TAIL == 16) {
                    uint32_t pk8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) pk8[q] = exp_pair(split, st[2 * q], st[2 * q + 1], q);
                    tc::st8(p_addr + 16 * NCH, pk8);
                }
            };
            if (masked)
                exp_row(std::integral_constant<bool, false>());
            else
                exp_row(std::integral_constant<bool, true>());
            tc::wait_st();
            if (p.kvcache && j == nk - 1 && j0 + BN > N) {
                // cache rows past N_b may hold anything: zero them in the V tile
                // (pairs: both tiles' warpgroups do it; the writes are identical;
                // key split: only the half that holds the last tile)
                const int li = KSPLIT ? 2 * (j - jb) + x : j - kb0;   // load index of V(j)
                const int vs = li % VST;
                if (!(ok = mbar_wait(&v_full[vs], (li / VST) & 1, p.status))) break;
                uint8_t *vt = sV + vs * C::VBYTES;
                const int first = N - j0;
                const int n16 = (BN - first) * 8 * (D_V / 64);
                for (int idx = threadIdx.x - 128 - 128 * x; idx < n16; idx += 128) {
                    const int box = idx / ((BN - first) * 8);
                    const int rem = idx % ((BN - first) * 8);
                    *reinterpret_cast<uint4 *>(vt + box * C::KBOX + (first + rem / 8) * 128 + (rem % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[x]);
            // row sum of the fp32 P values (four independent packed chains)
            uint64_t rs2[4] = {0, 0, 0, 0};
#pragma unroll
            for (int h = 0; h < NCH; ++h)
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    rs2[(e >> 1) & 3] = f2_add(rs2[(e >> 1) & 3], f2_pack(__uint_as_float(sr[h][e]), __uint_as_float(sr[h][e + 1])));
#pragma unroll
            for (int e = 0; e < TAIL; e += 2)
                rs2[(e >> 1) & 3] = f2_add(rs2[(e >> 1) & 3], f2_pack(__uint_as_float(st[e]), __uint_as_float(st[e + 1])));
            float r0, r1, r2, r3, r4, r5, r6, r7;
            f2_unpack(rs2[0], r0, r1);
            f2_unpack(rs2[1], r2, r3);
            f2_unpack(rs2[2], r4, r5);
            f2_unpack(rs2[3], r6, r7);
            l = l * alpha + (((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7)));
        }
        // ------------------------------------------------ epilogue
        if (ok && nk > jb && !mbar_wait(&pv_done[x], (nk - 1 - jb) & 1, p.status)) ok = false;
        tc::fence_after_sync();
        T *orow = static_cast<T *>(p.out) + tb * p.os.b + (int64_t)(qoff + i) * p.os.s + hq * p.os.h;
        if (KSPLIT) {
            // exchange (max, sum) of the two key halves per row through the
            // unused second Q buffer; both warpgroups reach the barrier once
            float *mls = reinterpret_cast<float *>(sQ + C::QBYTES);   // [m_0 | m_1 | l_0 | l_1][128]
            mls[x * kBM + r] = (nk > jb && l > 0.f) ? m_ref * c : -INFINITY;
            mls[(2 + x) * kBM + r] = nk > jb ? l : 0.f;
            tc::fence_before_sync();
            asm volatile("bar.sync 1, 256;" ::: "memory");
            tc::fence_after_sync();
            const float m0 = mls[r], m1 = mls[kBM + r], l0 = mls[2 * kBM + r], l1 = mls[3 * kBM + r];
            const float mx = fmaxf(m0, m1);
            const float a0 = l0 > 0.f ? ex2(m0 - mx) : 0.f, a1 = l1 > 0.f ? ex2(m1 - mx) : 0.f;
            const float lt = a0 * l0 + a1 * l1;
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const float w0 = a0 * inv, w1 = a1 * inv;
            // this warpgroup merges columns x d_v/2 .. (x+1) d_v/2 - 1 of both O
            const uint32_t o_base = tmem + lane_addr;
#pragma unroll
            for (int h = 0; h < D_V / 64; ++h) {
                const int col = x * (D_V / 2) + h * 32;
                uint32_t o0[32], o1[32];
                if (n_x[0] > 0) tc::ld32(o_base + C::t_o(0) + col, o0);
                if (n_x[1] > 0) tc::ld32(o_base + C::t_o(1) + col, o1);
                tc::wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        float f[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const float v0 = n_x[0] > 0 ? __uint_as_float(o0[e + u]) * w0 : 0.f;
                            const float v1 = n_x[1] > 0 ? __uint_as_float(o1[e + u]) * w1 : 0.f;
                            f[u] = v0 + v1;
                        }
                        reinterpret_cast<uint4 *>(orow + col + e)[0] = pack8<T>(f);
                    }
                }
            }
            if (x == 0 && row_valid && p.lse)
                p.lse[p.cu_q ? (int64_t)hq * p.total_q + qoff + i : ((int64_t)b * p.h_q + hq) * sq + i] =
                    lt > 0.f ? (mx + log2f(lt)) * kLn2 : -INFINITY;
        } else {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int h = 0; h < D_V / 32; ++h) {
            uint32_t orr[32];
            if (nk > jb) {
                tc::ld32(o_addr + h * 32, orr);
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
                    for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(orr[e + u]) * inv;
                    reinterpret_cast<uint4 *>(orow + h * 32 + e)[0] = pack8<T>(f);
                }
            }
        }
        if (row_valid && p.lse)
            p.lse[p.cu_q ? (int64_t)hq * p.total_q + qoff + i : ((int64_t)b * p.h_q + hq) * sq + i] = l > 0.f ? (m_ref * c + log2f(l)) * kLn2 : -INFINITY;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// The kernel's setmaxnreg split (128 x 56 + 256 x 224 registers) must fit in
// what the block is launched with, or the increase never returns.
template <typename K>
static cudaError_t check_regs(K kernel, int *cached) {
    if (*cached < 0) {
        cudaFuncAttributes fa_attr;
        const cudaError_t e = cudaFuncGetAttributes(&fa_attr, kernel);
        if (e != cudaSuccess) return e;
        *cached = fa_attr.numRegs;
    }
    return *cached * 384 < 128 * 56 + 256 * 224 ? cudaErrorInvalidConfiguration : cudaSuccess;
}

template <typename T, int D_QK, int D_V>
static cudaError_t run_prefill(const PrefillParams &p, const CUtensorMap &tmQ, const CUtensorMap &tmK,
                               const CUtensorMap &tmV, cudaStream_t st) {
    if (p.tiles_per_cta == 2) {
        using C2 = Prefill2Cfg<D_QK, D_V>;
        auto kern = p.key_split ? prefill2_kernel<T, D_QK, D_V, true> : prefill2_kernel<T, D_QK, D_V, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C2::SMEM);
        if (e != cudaSuccess) return e;
        static int regs_pair = -1, regs_split = -1;
        if ((e = check_regs(kern, p.key_split ? &regs_split : &regs_pair)) != cudaSuccess) return e;
        // key split: one CTA per query tile; pairs: one per two tiles
        const int64_t units = p.key_split ? p.n_q_tiles : (p.n_q_tiles + 1) / 2;
        const int64_t nblk = units * (p.h_q / p.pack) * p.b;
        if (nblk > 0x7fffffff) return cudaErrorInvalidConfiguration;
        dim3 grid((unsigned)nblk);
        kernel_event(0, st);
        kern<<<grid, 384, C2::SMEM, st>>>(tmQ, tmK, tmV, p);
        e = cudaGetLastError();
        kernel_event(1, st);
        return e;
    }
    using C = PrefillCfg<D_QK, D_V>;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<T, D_QK, D_V>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int64_t nblk = (int64_t)p.n_q_tiles * (p.h_q / p.pack) * p.b;
    if (nblk > 0x7fffffff) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)nblk);
    kernel_event(0, st);
    prefill_kernel<T, D_QK, D_V><<<grid, 256, C::SMEM, st>>>(tmQ, tmK, tmV, p);
    e = cudaGetLastError();
    kernel_event(1, st);
    return e;
}

#define FA_PREFILL_DIMS(X) X(64, 64) X(128, 128) X(192, 128) X(128, 64) X(64, 128) X(192, 64)

int prefill_block_n(int d_qk, int d_v, int tiles_per_cta) {
    (void)d_qk;
    return (tiles_per_cta == 2 && d_v > 64) ? 80 : kBN;
}

bool prefill_supported(int d_qk, int d_v) {
#define FA_CASE(DQ, DV) if (d_qk == DQ && d_v == DV) return true;
    FA_PREFILL_DIMS(FA_CASE)
#undef FA_CASE
    return false;
}

cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &tmQ, const CUtensorMap &tmK,
                           const CUtensorMap &tmV, int dtype, int d_qk, int d_v, cudaStream_t st) {
#define FA_CASE(DQ, DV)                                                                   \
    if (d_qk == DQ && d_v == DV) {                                                        \
        if (dtype == FA_DTYPE_F16) return run_prefill<__half, DQ, DV>(p, tmQ, tmK, tmV, st); \
        return run_prefill<__nv_bfloat16, DQ, DV>(p, tmQ, tmK, tmV, st);                  \
    }
    FA_PREFILL_DIMS(FA_CASE)
#undef FA_CASE
    return cudaErrorInvalidValue;
}

}  // namespace fa
