// decode.cu -- persistent split-KV decode attention with fused RoPE + cache
// append, and the LSE combine of the split partials.
//
// Path (the single-token / short-chunk branch of the attention-with-KV-cache
// call: s2.cpp PR #40's eval_cached decode branch, flash_attn_with_kvcache of
// flash-attention issue #1402 with a short new chunk):
//  * Work is the key rows of every (batch, kv head) segment, N_b = L_b + s_new
//    rows each, cut into 64-row items.  One CTA per SM; CTA c takes the items
//    whose first row falls in [c R / G, (c+1) R / G) of the concatenated rows
//    R (computed on the device from cache_seqlens), so every SM streams the
//    same number of bytes whatever the mix of sequence lengths.  A CTA's items
//    form runs ("pieces") of consecutive rows of one segment; each piece is one
//    online-softmax pass.
//  * All g * s_q query rows that read a kv head (grouped-query heads of the
//    "optimizing-attention-flash" page, Workflow 2 Step 3) share one 16- or
//    32-row MMA tile, so each key/value row is read from HBM once.
//  * Warp 4 streams 64-row K and V tiles with TMA (swizzled boxes) through a
//    ring of shared-memory stages across item and piece boundaries; warps 0-3
//    each take 16 keys of every tile, keep their own running max / sum /
//    output, and merge at the end of a piece while the ring keeps filling.
//  * The tile holding rows >= L_b is patched in shared memory by the warp that
//    owns those keys: new key rows are rotated (the same rotation as the
//    append kernel) and rounded, new value rows copied, both written to the
//    cache (the only writer of those rows); rows >= N_b are zeroed so garbage
//    past the sequence cannot reach the PV product.
//  * q rows are rotated at position L_b + i while being staged.
//  * A segment that fits one item writes out / lse directly.  Otherwise every
//    piece writes its normalised output and lse to the slot of its first item
//    and lse = -inf to the slots of its other items; the combine kernel merges
//    the slots: lse = log sum exp(lse_s), out = sum exp(lse_s - lse) out_s.
//
// QK^T and PV use mma.sync m16n8k16 with fp32 accumulation: at most 32 query
// rows per kv head sit far below the tensor-core roof and the kernel is bound
// by the HBM stream of the cache.
#include <algorithm>

#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

constexpr int kDecodeTile = 64;   // key rows per tile and per item
// CTAs per SM: two when the per-thread state is small enough (one row tile,
// d_v <= 128), so that one CTA's piece merge overlaps the other's stream.
template <int D_V, int MT>
struct DecodeOcc {
    static constexpr int CTAS = (MT == 1 && D_V <= 128) ? 2 : 1;
    static constexpr int BUDGET = CTAS == 2 ? 112 * 1024 : 224 * 1024;
};

constexpr int kDecodeMaxStages = 8;

// Shared memory: rotated q tile | ring of K/V stages | merge scratch for the
// M live query rows | barriers.  The stage count is chosen at launch from the
// budget left after the (runtime-sized) merge scratch.
template <int D_QK, int D_V, int MT>
struct DecodeCfg {
    static constexpr int TILE = kDecodeTile;
    static constexpr int KBYTES = TILE * D_QK * 2;
    static constexpr int VBYTES = TILE * D_V * 2;
    static constexpr int STAGE = KBYTES + VBYTES;
    static constexpr int QROWS = MT * 16;
    static constexpr int QBYTES = ((QROWS * D_QK * 2 + 1023) / 1024) * 1024;
    static_assert(D_QK % 16 == 0 && D_V % 16 == 0, "head dims are multiples of 16");
    static int merge_bytes(int M) { return 4 * M * (D_V + 2) * 4; }
    // barriers, the 4-int schedule and the per-batch (L, N, items) table
    static int tail_bytes(int B) { return 2 * kDecodeMaxStages * 8 + 16 + 12 * B + 16; }
    static int stages(int M, int B) {
        const int raw = (DecodeOcc<D_V, MT>::BUDGET - 1024 - QBYTES - merge_bytes(M) - tail_bytes(B)) / STAGE;
        return raw < 2 ? 2 : (raw > kDecodeMaxStages ? kDecodeMaxStages : raw);
    }
    static int smem(int M, int B) { return 1024 + QBYTES + stages(M, B) * STAGE + merge_bytes(M) + tail_bytes(B); }
};

// Per-batch facts every thread can recompute: rows N_b and items n_b (0 when
// the batch entry violates the device-side preconditions).
struct SegInfo {
    int L, N, n_items;
};

__device__ __forceinline__ SegInfo seg_info(const DecodeParams &p, int b) {
    SegInfo s;
    s.L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
    const int64_t N64 = (int64_t)s.L + p.s_new;
    const bool bad = s.L < 0 || N64 > p.cap ||
                     (p.r > 0 && (int64_t)s.L + (p.s_q > p.s_new ? p.s_q : p.s_new) > p.cs_rows);
    s.N = bad ? 0 : (int)N64;
    s.n_items = bad ? 0 : (s.N + kDecodeTile - 1) / kDecodeTile;
    return s;
}

// Iterator over the items (b, hk, s) in segment order.
struct ItemIter {
    int b, hk, s;
    SegInfo seg;
};

// `tab` is the per-batch SegInfo table the CTA staged in shared memory.
__device__ __forceinline__ void iter_advance(const DecodeParams &p, const SegInfo *tab, ItemIter &it) {
    if (++it.s < it.seg.n_items) return;
    it.s = 0;
    if (++it.hk < p.h_kv) return;
    it.hk = 0;
    do {
        ++it.b;
        if (it.b >= p.b) return;
        it.seg = tab[it.b];
    } while (it.seg.n_items == 0);
}

// Global index of the first item whose first row is >= X in the concatenated
// row space, and the CTA's item range [I(c R/G), I((c+1) R/G)).
__device__ void cta_item_range(const DecodeParams &p, const SegInfo *tab, int c, int G, ItemIter &first,
                               int &n_items) {
    int64_t R = 0;
    for (int b = 0; b < p.b; ++b) R += (int64_t)p.h_kv * tab[b].N;
    const int64_t X0 = R * c / G, X1 = R * (c + 1) / G;
    int64_t I0 = -1, I1 = -1, items_before = 0, rows_before = 0;
    first.b = p.b;
    for (int b = 0; b < p.b && I1 < 0; ++b) {
        const SegInfo sg = tab[b];
        const int64_t seg_rows = (int64_t)p.h_kv * sg.N;
        for (int which = 0; which < 2; ++which) {
            const int64_t X = which ? X1 : X0;
            int64_t &I = which ? I1 : I0;
            if (I >= 0 || X >= rows_before + seg_rows) continue;
            const int64_t off = X - rows_before;
            const int64_t hk = off / sg.N, within = off - hk * sg.N;
            I = items_before + hk * sg.n_items + (within + kDecodeTile - 1) / kDecodeTile;
            if (which == 0) {
                // decode I0 into (b, hk, s), rolling over to the next item if needed
                first.b = b;
                first.hk = (int)hk;
                first.s = (int)((within + kDecodeTile - 1) / kDecodeTile);
                first.seg = sg;
                if (first.s >= sg.n_items) {
                    first.s = sg.n_items - 1;
                    iter_advance(p, tab, first);
                }
            }
        }
        items_before += (int64_t)p.h_kv * sg.n_items;
        rows_before += seg_rows;
    }
    if (I0 < 0) I0 = items_before;
    if (I1 < 0) I1 = items_before;
    n_items = (int)(I1 - I0);
}

template <typename T, int D_QK, int D_V, int MT>
__global__ void __launch_bounds__(160, DecodeOcc<D_V, MT>::CTAS) decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                        const __grid_constant__ CUtensorMap tmV,
                                                        const DecodeParams p) {
    using C = DecodeCfg<D_QK, D_V, MT>;
    constexpr int CHK = box_cols(D_QK), RBK = box_row_bytes(D_QK);
    constexpr int CHV = box_cols(D_V), RBV = box_row_bytes(D_V);
    constexpr int CK = D_QK / 8, CV = D_V / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int M = p.g * p.s_q;
    const int NST = p.n_stages;
    uint8_t *sQ = smem;
    uint8_t *sStage = smem + C::QBYTES;
    float *red_o = reinterpret_cast<float *>(sStage + NST * C::STAGE);   // [4][M][D_V]
    float *red_m = red_o + 4 * M * D_V;                                   // [4][M]
    float *red_l = red_m + 4 * M;                                         // [4][M]
    uint64_t *full = reinterpret_cast<uint64_t *>(red_l + 4 * M);
    uint64_t *empty = full + kDecodeMaxStages;
    int *sched = reinterpret_cast<int *>(empty + kDecodeMaxStages);   // b, hk, s, n_items
    SegInfo *tab = reinterpret_cast<SegInfo *>(sched + 4);             // [b]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool inter = p.interleaved != 0;

    // allow the combine kernel (launched as a programmatic dependent) to get scheduled
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // stage every batch entry's (L, N, items) once, with parallel loads
    for (int b = threadIdx.x; b < p.b; b += blockDim.x) tab[b] = seg_info(p, b);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        fence_barrier_init();
        ItemIter first;
        int n_items;
        cta_item_range(p, tab, blockIdx.x, gridDim.x, first, n_items);
        sched[0] = first.b;
        sched[1] = first.hk;
        sched[2] = first.s;
        sched[3] = n_items;
    }
    if (blockIdx.x == 0) {
        // batch entries with no key at all: out = 0, lse = -inf; bad entries: record
        for (int b = 0; b < p.b; ++b) {
            const SegInfo sg = tab[b];
            if (sg.n_items > 0) continue;
            const int L = sg.L;
            const bool bad = L < 0 || (int64_t)L + p.s_new > p.cap ||
                             (p.r > 0 && (int64_t)L + (p.s_q > p.s_new ? p.s_q : p.s_new) > p.cs_rows);
            if (bad) {
                if (threadIdx.x == 0) record_status(p.status, FA_ERR_DEVICE_PRECONDITION);
                continue;
            }
            for (int idx = threadIdx.x; idx < p.h_q * p.s_q * CV; idx += blockDim.x) {
                const int c = idx % CV, row = idx / CV;
                const int hq = row / p.s_q, i = row % p.s_q;
                T *dst = static_cast<T *>(p.out) + b * p.os.b + i * p.os.s + hq * p.os.h;
                reinterpret_cast<uint4 *>(dst)[c] = make_uint4(0, 0, 0, 0);
                if (c == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = -INFINITY;
            }
        }
    }
    __syncthreads();
    const int n_items = sched[3];
    if (n_items == 0) return;
    ItemIter it0;
    it0.b = sched[0];
    it0.hk = sched[1];
    it0.s = sched[2];
    it0.seg = tab[it0.b];

    if (warp == 4) {
        // ---------------- producer: TMA stream of K/V tiles over all items ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            ItemIter it = it0;
            int t = 0;
            bool ok = true;
            for (int k = 0; k < n_items && ok; ++k) {
                const int row0 = it.s * C::TILE;
                const int s = t % NST;
                if (t >= NST && !mbar_wait(&empty[s], ((t / NST) - 1) & 1, p.status)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                uint8_t *kd = sStage + s * C::STAGE;
                uint8_t *vd = kd + C::KBYTES;
#pragma unroll
                for (int c = 0; c < D_QK / CHK; ++c)
                    tma_load_4d(kd + c * C::TILE * RBK, &tmK, &full[s], c * CHK, it.hk, row0, it.b);
#pragma unroll
                for (int c = 0; c < D_V / CHV; ++c)
                    tma_load_4d(vd + c * C::TILE * RBV, &tmV, &full[s], c * CHV, it.hk, row0, it.b);
                ++t;
                iter_advance(p, tab, it);
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    const T *cos_t = static_cast<const T *>(p.cos);
    const T *sin_t = static_cast<const T *>(p.sin);
    const uint32_t sQa = smem_addr(sQ);
    float o[MT][D_V / 8][4];
    float m_r[MT][2], l_r[MT][2];
    int last_vis[MT][2];
    int s_first = 0;
    bool timed_out = false;
    ItemIter it = it0;
    for (int k = 0; k < n_items; ++k) {
        const int b = it.b, hk = it.hk;
        const int L = it.seg.L, N = it.seg.N;
        const int hq0 = hk * p.g;
        const bool piece_start = (k == 0) || it.s == 0;
        if (piece_start) {
            s_first = it.s;
            // stage the rotated q rows of this (batch, kv head)
            for (int idx = threadIdx.x; idx < C::QROWS * CK; idx += 128) {
                const int r = idx / CK, c = idx % CK;
                float f[8];
                if (r < M) {
                    const int i = r / p.g, hq = hq0 + r % p.g;
                    const T *src = static_cast<const T *>(p.q) + b * p.qs.b + i * p.qs.s + hq * p.qs.h;
                    const int64_t pos = (int64_t)L + i;
                    load_rotated_chunk<T>(src, c, p.r, inter, p.r ? cos_t + pos * p.cs_row : nullptr,
                                          p.r ? sin_t + pos * p.cs_row : nullptr, f);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = 0.f;
                }
                *reinterpret_cast<uint4 *>(sQ + swz_offset<D_QK>(r, c * 8, C::QROWS)) = pack8<T>(f);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int n = 0; n < D_V / 8; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[mt][n][e] = 0.f;
                m_r[mt][0] = m_r[mt][1] = -INFINITY;
                l_r[mt][0] = l_r[mt][1] = 0.f;
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = mt * 16 + (lane >> 2) + hr * 8;
                    last_vis[mt][hr] = r < M ? (p.causal ? min(N - 1, r / p.g + N - p.s_q) : N - 1) : -1;
                }
            }
            consumer_sync();
        }

        // ---- one 64-row tile = one item ----
        const int t = k;
        const int s = t % NST;
        if (!timed_out && !mbar_wait(&full[s], (t / NST) & 1, p.status)) timed_out = true;
        if (!timed_out) {
            uint8_t *sK = sStage + s * C::STAGE;
            uint8_t *sV = sK + C::KBYTES;
            const int tile_row0 = it.s * C::TILE;
            const int key0 = tile_row0 + warp * 16;
            if (key0 + 16 > L) {
                for (int item = lane; item < 16 * (CK + CV); item += 32) {
                    const int rr = item / (CK + CV), c = item % (CK + CV);
                    const int j = key0 + rr;
                    if (j < L) continue;
                    const int tr = warp * 16 + rr;
                    if (j < N) {
                        const int i = j - L;
                        if (c < CK) {
                            const T *src = static_cast<const T *>(p.k_new) + b * p.kn.b + i * p.kn.s + hk * p.kn.h;
                            float f[8];
                            load_rotated_chunk<T>(src, c, p.r, inter,
                                                  p.r ? cos_t + (int64_t)j * p.cs_row : nullptr,
                                                  p.r ? sin_t + (int64_t)j * p.cs_row : nullptr, f);
                            const uint4 v = pack8<T>(f);
                            *reinterpret_cast<uint4 *>(sK + swz_offset<D_QK>(tr, c * 8, C::TILE)) = v;
                            T *dst = static_cast<T *>(p.k_cache) + b * p.kc.b + (int64_t)j * p.kc.s + hk * p.kc.h;
                            reinterpret_cast<uint4 *>(dst)[c] = v;
                        } else {
                            const int cv = c - CK;
                            const T *src = static_cast<const T *>(p.v_new) + b * p.vn.b + i * p.vn.s + hk * p.vn.h;
                            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + cv);
                            *reinterpret_cast<uint4 *>(sV + swz_offset<D_V>(tr, cv * 8, C::TILE)) = v;
                            T *dst = static_cast<T *>(p.v_cache) + b * p.vc.b + (int64_t)j * p.vc.s + hk * p.vc.h;
                            reinterpret_cast<uint4 *>(dst)[cv] = v;
                        }
                    } else {
                        const uint4 z = make_uint4(0, 0, 0, 0);
                        if (c < CK)
                            *reinterpret_cast<uint4 *>(sK + swz_offset<D_QK>(tr, c * 8, C::TILE)) = z;
                        else
                            *reinterpret_cast<uint4 *>(sV + swz_offset<D_V>(tr, (c - CK) * 8, C::TILE)) = z;
                    }
                }
                fence_proxy_async();
                __syncwarp();
            }

            // S = Q K^T over this warp's 16 keys
            float sacc[MT][2][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc[mt][nt][e] = 0.f;
            const uint32_t sKa = smem_addr(sK), sVa = smem_addr(sV);
#pragma unroll
            for (int kk = 0; kk < D_QK / 16; ++kk) {
                uint32_t kb[4];
                ldmatrix_x4(sKa + swz_offset<D_QK>(warp * 16 + (lane & 7) + ((lane >> 4) << 3),
                                                   kk * 16 + (((lane >> 3) & 1) << 3), C::TILE),
                            kb[0], kb[1], kb[2], kb[3]);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t a[4];
                    ldmatrix_x4(sQa + swz_offset<D_QK>(mt * 16 + (lane & 15), kk * 16 + ((lane >> 4) << 3),
                                                       C::QROWS),
                                a[0], a[1], a[2], a[3]);
                    Mma<T>::run(sacc[mt][0], a, kb[0], kb[1]);
                    Mma<T>::run(sacc[mt][1], a, kb[2], kb[3]);
                }
            }

            // mask + online softmax (base 2, scale folded in)
            uint32_t pa[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                float pv[2][2][2];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    float vals[2][2];
                    float mx = -INFINITY;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = key0 + nt * 8 + ((lane & 3) << 1) + e;
                            float v = sacc[mt][nt][hr * 2 + e] * p.scale_log2;
                            if (j > last_vis[mt][hr]) v = -INFINITY;
                            vals[nt][e] = v;
                            mx = fmaxf(mx, v);
                        }
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    const float m_new = fmaxf(m_r[mt][hr], mx);
                    const float m_use = m_new == -INFINITY ? 0.f : m_new;
                    const float corr = ex2(m_r[mt][hr] - m_use);
                    float sum = 0.f;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            pv[hr][nt][e] = ex2(vals[nt][e] - m_use);
                            sum += pv[hr][nt][e];
                        }
                    l_r[mt][hr] = l_r[mt][hr] * corr + sum;
                    m_r[mt][hr] = m_new;
                    if (corr != 1.f) {
#pragma unroll
                        for (int n = 0; n < D_V / 8; ++n) {
                            o[mt][n][hr * 2] *= corr;
                            o[mt][n][hr * 2 + 1] *= corr;
                        }
                    }
                }
                pa[mt][0] = Elem<T>::pack2(pv[0][0][0], pv[0][0][1]);
                pa[mt][1] = Elem<T>::pack2(pv[1][0][0], pv[1][0][1]);
                pa[mt][2] = Elem<T>::pack2(pv[0][1][0], pv[0][1][1]);
                pa[mt][3] = Elem<T>::pack2(pv[1][1][0], pv[1][1][1]);
            }

            // O += P V over this warp's 16 keys
#pragma unroll
            for (int nn = 0; nn < D_V / 16; ++nn) {
                uint32_t vb[4];
                ldmatrix_x4_trans(sVa + swz_offset<D_V>(warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                                                        nn * 16 + ((lane >> 4) << 3), C::TILE),
                                  vb[0], vb[1], vb[2], vb[3]);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    Mma<T>::run(o[mt][2 * nn], pa[mt], vb[0], vb[1]);
                    Mma<T>::run(o[mt][2 * nn + 1], pa[mt], vb[2], vb[3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }

        // ---- end of piece: merge the four warps and write ----
        const bool piece_end = (k == n_items - 1) || (it.s + 1 >= it.seg.n_items);
        if (piece_end) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    l_r[mt][hr] += __shfl_xor_sync(0xffffffffu, l_r[mt][hr], 1);
                    l_r[mt][hr] += __shfl_xor_sync(0xffffffffu, l_r[mt][hr], 2);
                }
            consumer_sync();
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int row = mt * 16 + (lane >> 2) + hr * 8;
                    if (row < M) {
                        if ((lane & 3) == 0) {
                            red_m[warp * M + row] = m_r[mt][hr];
                            red_l[warp * M + row] = l_r[mt][hr];
                        }
                        float *dst = red_o + (warp * M + row) * D_V + ((lane & 3) << 1);
#pragma unroll
                        for (int n = 0; n < D_V / 8; ++n)
                            *reinterpret_cast<float2 *>(dst + n * 8) =
                                make_float2(o[mt][n][hr * 2], o[mt][n][hr * 2 + 1]);
                    }
                }
            consumer_sync();
            const bool single = it.seg.n_items == 1;
            for (int idx = threadIdx.x; idx < M * CV; idx += 128) {
                const int row = idx / CV, c = idx % CV;
                float mw[4], mx = -INFINITY;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    mw[w] = red_m[w * M + row];
                    mx = fmaxf(mx, mw[w]);
                }
                const float mu = mx == -INFINITY ? 0.f : mx;
                float ltot = 0.f, acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float sc = ex2(mw[w] - mu);
                    ltot += red_l[w * M + row] * sc;
                    const float *src = red_o + (w * M + row) * D_V + c * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] += src[e] * sc;
                }
                const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] *= inv;
                const float lse_v = ltot > 0.f ? (mx + log2f(ltot)) * kLn2 : -INFINITY;
                const int i = row / p.g, hq = hq0 + row % p.g;
                if (single) {
                    T *dst = static_cast<T *>(p.out) + b * p.os.b + i * p.os.s + hq * p.os.h;
                    reinterpret_cast<uint4 *>(dst)[c] = pack8<T>(acc);
                    if (c == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = lse_v;
                } else {
                    // slots of one output row are contiguous: [b][h_q][s_q][n_splits]
                    const int64_t row_slot0 = (((int64_t)b * p.h_q + hq) * p.s_q + i) * p.n_splits;
                    float4 *dst = reinterpret_cast<float4 *>(p.o_part + (row_slot0 + s_first) * D_V + c * 8);
                    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
                    if (c == 0) {
                        p.lse_part[row_slot0 + s_first] = lse_v;
                        for (int s2 = s_first + 1; s2 <= it.s; ++s2) p.lse_part[row_slot0 + s2] = -INFINITY;
                    }
                }
            }
        }
        iter_advance(p, tab, it);
    }
}

// One warp per (batch, query head, query row): merge the split slots.
template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(const DecodeParams p, int d_v) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t total = (int64_t)p.b * p.h_q * p.s_q;
    if (w >= total) return;
    const int i = (int)(w % p.s_q);
    const int hq = (int)((w / p.s_q) % p.h_q);
    const int b = (int)(w / ((int64_t)p.s_q * p.h_q));
    const SegInfo sg = seg_info(p, b);
    const int n = sg.n_items;
    if (n <= 1) return;
    // the row's slots are contiguous: read their lse values coalesced, keep
    // them in registers (lane l holds slots l, l + 32, ...)
    const int64_t row_slot0 = (((int64_t)b * p.h_q + hq) * p.s_q + i) * p.n_splits;
    constexpr int MAXS = 16;  // up to 512 slots per row
    float ls[MAXS];
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < MAXS; ++k) {
        const int s = lane + 32 * k;
        ls[k] = s < n ? p.lse_part[row_slot0 + s] : -INFINITY;
        mx = fmaxf(mx, ls[k]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    T *dst = static_cast<T *>(p.out) + b * p.os.b + i * p.os.s + hq * p.os.h;
    if (mx == -INFINITY) {
        for (int c = lane * 2; c < d_v; c += 64) *reinterpret_cast<uint32_t *>(dst + c) = 0u;
        if (lane == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = -INFINITY;
        return;
    }
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < MAXS; ++k) sum += ex2((ls[k] - mx) * kLog2e);
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse = mx + logf(sum);
    float a[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
    // Only the first slot of every piece holds an output.  Compact the live
    // slots and their weights into this warp's shared-memory list, then read
    // their outputs with independent (overlapping) loads.
    constexpr int LIST = 64;
    __shared__ int live_slot[8][LIST];
    __shared__ float live_w[8][LIST];
    const int wib = threadIdx.x >> 5;
    int n_total = 0;
#pragma unroll
    for (int k = 0; k < MAXS; ++k) n_total += __popc(__ballot_sync(0xffffffffu, ls[k] != -INFINITY));
    for (int base = 0; base < n_total; base += LIST) {
        int n_live = 0;
#pragma unroll
        for (int k = 0; k < MAXS; ++k) {
            const bool is_live = ls[k] != -INFINITY;
            const unsigned live = __ballot_sync(0xffffffffu, is_live);
            const int pos = n_live + __popc(live & ((1u << lane) - 1u)) - base;
            if (is_live && pos >= 0 && pos < LIST) {
                live_slot[wib][pos] = lane + 32 * k;
                live_w[wib][pos] = ex2((ls[k] - lse) * kLog2e);
            }
            n_live += __popc(live);
        }
        __syncwarp();
        const int cnt = min(LIST, n_total - base);
#pragma unroll 4
        for (int t = 0; t < cnt; ++t) {
            const float wgt = live_w[wib][t];
            const float *src = p.o_part + (row_slot0 + live_slot[wib][t]) * d_v;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = lane * 2 + e * 64;
                if (c < d_v) {
                    const float2 v = *reinterpret_cast<const float2 *>(src + c);
                    a[2 * e] = fmaf(wgt, v.x, a[2 * e]);
                    a[2 * e + 1] = fmaf(wgt, v.y, a[2 * e + 1]);
                }
            }
        }
        __syncwarp();
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int c = lane * 2 + e * 64;
        if (c < d_v) *reinterpret_cast<uint32_t *>(dst + c) = Elem<T>::pack2(a[2 * e], a[2 * e + 1]);
    }
    if (lane == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = lse;
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <typename T, int D_QK, int D_V, int MT>
static cudaError_t run_decode(const DecodeParams &p_in, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              cudaStream_t st) {
    using C = DecodeCfg<D_QK, D_V, MT>;
    DecodeParams p = p_in;
    const int M = p.g * p.s_q;
    p.n_stages = C::stages(M, p.b);
    const int smem = C::smem(M, p.b);
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D_QK, D_V, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kernel_event(0, st);
    decode_kernel<T, D_QK, D_V, MT><<<sm_count() * DecodeOcc<D_V, MT>::CTAS, 160, smem, st>>>(tmK, tmV, p);
    e = cudaGetLastError();
    kernel_event(1, st);
    if (e != cudaSuccess) return e;
    if (p.n_splits > 1) {
        const int64_t warps = (int64_t)p.b * p.h_q * p.s_q;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((warps * 32 + 255) / 256));
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, combine_kernel<T>, p, D_V);
    }
    return e;
}

#define FA_DECODE_DIMS(X) \
    X(16, 16, 1) X(16, 16, 2) X(32, 32, 1) X(32, 32, 2) X(64, 64, 1) X(64, 64, 2) \
    X(128, 128, 1) X(128, 128, 2) X(192, 128, 1) X(192, 128, 2) X(256, 256, 1)

bool decode_supported(int d_qk, int d_v, int mt) {
#define FA_CASE(DQ, DV, MT) if (d_qk == DQ && d_v == DV && mt == MT) return true;
    FA_DECODE_DIMS(FA_CASE)
#undef FA_CASE
    return false;
}

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmK, const CUtensorMap &tmV,
                          int dtype, int d_qk, int d_v, int mt, cudaStream_t st) {
#define FA_CASE(DQ, DV, MT)                                                                \
    if (d_qk == DQ && d_v == DV && mt == MT) {                                             \
        if (dtype == FA_DTYPE_F16) return run_decode<__half, DQ, DV, MT>(p, tmK, tmV, st); \
        return run_decode<__nv_bfloat16, DQ, DV, MT>(p, tmK, tmV, st);                     \
    }
    FA_DECODE_DIMS(FA_CASE)
#undef FA_CASE
    return cudaErrorInvalidValue;
}

}  // namespace fa
