// decode.cu -- persistent split-KV decode attention over the KV cache, and
// the LSE combine of the split partials.
//
// Path (the single-token / short-chunk branch of the attention-with-KV-cache
// call: s2.cpp PR #40's eval_cached decode branch, flash_attn_with_kvcache of
// flash-attention issue #1402 with a short new chunk).  The RoPE/append
// kernel runs first on the same stream: it rotates q into the workspace,
// writes the rotated new key rows and the new value rows into the cache, and
// zeroes the work-pool counter.  This kernel is launched as its programmatic
// dependent, so its CTAs start while that kernel is still running; the
// producer waits for it (griddepcontrol) only before loading q or a tile that
// holds new rows, and before touching the pool counter.
//  * Work is the key rows of every (batch, kv head) segment, N_b = L_b + s_new
//    rows each, cut into n_b 64-row items.  The last floor(n_b / 4) items of
//    every segment form the pool; the rest is split statically: CTA c takes
//    the static items whose first row falls in [c R_s / G, (c+1) R_s / G) of
//    the concatenated static rows R_s (computed on the device from
//    cache_seqlens).  When its static share is done a CTA claims 2-item chunks
//    of the pool (segment tails, in segment order) with an atomic counter, so
//    SMs that stream faster take more of the tail.  A CTA's items form runs
//    ("pieces") of consecutive rows of one segment; a piece ends where the
//    segment, the segment's static part, the static share or a chunk ends,
//    and each piece is one online-softmax pass.
//  * All g * s_q query rows that read a kv head (grouped-query heads of the
//    "optimizing-attention-flash" page, Workflow 2 Step 3) share one 16- or
//    32-row MMA tile, so each key/value row is read from HBM once.
//  * Warp 4 is the only warp that touches global memory while the stream
//    runs: it loads every piece's rotated q rows (a two-buffer ring) and the
//    64-row K and V tiles (a ring of stages) with TMA, and posts each stage's
//    item in shared memory.  Warps 0-3 each take 16 keys of every tile, keep
//    their own running max / sum / output, and merge at the end of a piece.
//    (With HBM saturated by the stream, an ordinary load or store issued by a
//    consumer warp waits behind the queued tile requests for microseconds, so
//    consumers issue none until a piece ends.)
//  * Rows >= N_b of a segment's last tile are zeroed in shared memory by the
//    warp that owns them, so whatever the cache holds past the sequence
//    cannot reach the PV product (their scores are masked to -inf).
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

constexpr int kDecodeTile = 64;        // key rows per tile and per item
constexpr int kPoolChunk = 2;          // items per claim from the pool
constexpr int kPoolDen = 4;            // the pool holds floor(n_b / 4) items of each segment

// CTAs per SM: two when the per-thread state is small enough (one row tile,
// d_v <= 128), so that one CTA's piece merge overlaps the other's stream.
template <int D_V, int MT>
struct DecodeOcc {
    static constexpr int CTAS = (MT == 1 && D_V <= 128) ? 2 : 1;
    static constexpr int BUDGET = CTAS == 2 ? 112 * 1024 : 224 * 1024;
};

constexpr int kDecodeMaxStages = 8;

// The item of one stage, posted by the producer before the stage's TMA.
struct StageItem {
    int b, hk, s, flags;
};
constexpr int kPieceStart = 1, kPieceEnd = 2, kEndOfStream = 4;

// Shared memory: two q buffers | ring of K/V stages | merge scratch for the
// M live query rows | barriers, stage items, schedule, per-batch table.  A q
// buffer holds QT = M rounded up to 8 rows per 64-column box (the TMA writes
// the M live rows; the MMA tile reads up to 16 * MT rows, and rows >= M only
// feed output rows that are never written).  The stage count is chosen at
// launch from the budget left.
template <int D_QK, int D_V, int MT>
struct DecodeCfg {
    static constexpr int TILE = kDecodeTile;
    static constexpr int KBYTES = TILE * D_QK * 2;
    static constexpr int VBYTES = TILE * D_V * 2;
    static constexpr int STAGE = KBYTES + VBYTES;
    static constexpr int QROWS = MT * 16;
    static_assert(D_QK % 16 == 0 && D_V % 16 == 0, "head dims are multiples of 16");
    __host__ __device__ static int qt(int M) { return (M + 7) / 8 * 8; }
    __host__ __device__ static int qbuf_bytes(int M) { return (qt(M) * D_QK * 2 + 1023) / 1024 * 1024; }
    static int merge_bytes(int M) { return 4 * M * (D_V + 2) * 4; }
    // ring and q barriers, stage items, the 4-int64 schedule, the 16-byte per-batch table
    static int tail_bytes(int B) {
        return (2 * kDecodeMaxStages + 4) * 8 + kDecodeMaxStages * 16 + 32 + 16 * B + 16;
    }
    static int stages(int M, int B) {
        const int raw =
            (DecodeOcc<D_V, MT>::BUDGET - 1024 - 2 * qbuf_bytes(M) - merge_bytes(M) - tail_bytes(B)) / STAGE;
        return raw < 2 ? 2 : (raw > kDecodeMaxStages ? kDecodeMaxStages : raw);
    }
    static int smem(int M, int B) {
        return 1024 + 2 * qbuf_bytes(M) + stages(M, B) * STAGE + merge_bytes(M) + tail_bytes(B);
    }
};

// Per-batch facts every thread can recompute: rows N_b, the first row `base`
// of item 0 (0, or with a left window the first visible row of the first
// query row rounded down to 64) and items n_b covering rows base .. N_b - 1
// (0 when the batch entry violates the device-side preconditions, which the
// RoPE/append kernel records and skips in the same way).
struct SegInfo {
    int L, N, base, n_items;
};

__device__ __forceinline__ SegInfo seg_info(const DecodeParams &p, int b) {
    SegInfo s;
    s.L = seqlen_of(p.seqlens, p.seqlen_scalar, b);
    const int64_t N64 = (int64_t)s.L + p.s_new;
    const bool bad = s.L < 0 || N64 > p.cap ||
                     (p.r > 0 && (int64_t)s.L + (p.s_q > p.s_new ? p.s_q : p.s_new) > p.cs_rows);
    s.N = bad ? 0 : (int)N64;
    int64_t first = 0, last = -1;
    visible_keys(0, s.N, p.s_q, p.causal, p.win_left, p.win_right, first, last);
    s.base = (int)(first < s.N ? first : s.N) & ~(kDecodeTile - 1);
    s.n_items = bad ? 0 : (s.N - s.base + kDecodeTile - 1) / kDecodeTile;
    return s;
}

// Items [0, ns) of a segment are split statically, [ns, n) are in the pool.
__device__ __forceinline__ int pool_items(int n) { return n / kPoolDen; }
__device__ __forceinline__ int static_items(int n) { return n - pool_items(n); }
// Rows of a segment's static part (all of it when the pool holds none).
__device__ __forceinline__ int static_rows(const SegInfo &sg) {
    return pool_items(sg.n_items) > 0 ? static_items(sg.n_items) * kDecodeTile : sg.N - sg.base;
}

// An item (b, hk, s) and its segment; POOL selects which items of a segment
// the iteration visits ([0, ns) or [ns, n)).
struct ItemIter {
    int b, hk, s;
    SegInfo seg;
};

template <bool POOL>
__device__ __forceinline__ int part_first(const SegInfo &sg) { return POOL ? static_items(sg.n_items) : 0; }
template <bool POOL>
__device__ __forceinline__ int part_end(const SegInfo &sg) { return POOL ? sg.n_items : static_items(sg.n_items); }
template <bool POOL>
__device__ __forceinline__ int part_count(const SegInfo &sg) { return part_end<POOL>(sg) - part_first<POOL>(sg); }

// Next item of the same part, in (batch, kv head, item) order.
template <bool POOL>
__device__ __forceinline__ void iter_advance(const DecodeParams &p, const SegInfo *tab, ItemIter &it) {
    if (++it.s < part_end<POOL>(it.seg)) return;
    if (++it.hk < p.h_kv) {
        it.s = part_first<POOL>(it.seg);
        return;
    }
    it.hk = 0;
    do {
        ++it.b;
        if (it.b >= p.b) return;
        it.seg = tab[it.b];
    } while (part_count<POOL>(it.seg) == 0);
    it.s = part_first<POOL>(it.seg);
}

// Index (among all static items) of the first static item whose first row is
// >= X in the concatenated static rows (the static item count if none).
__device__ int64_t static_item_at_row(const DecodeParams &p, const SegInfo *tab, int64_t X) {
    int64_t items_before = 0, rows_before = 0;
    for (int b = 0; b < p.b; ++b) {
        const SegInfo sg = tab[b];
        const int rs = static_rows(sg), ns = static_items(sg.n_items);
        const int64_t seg_rows = (int64_t)p.h_kv * rs;
        if (X < rows_before + seg_rows) {
            const int64_t off = X - rows_before;
            const int64_t hk = off / rs, within = off - hk * rs;
            return items_before + hk * ns + (within + kDecodeTile - 1) / kDecodeTile;
        }
        items_before += (int64_t)p.h_kv * ns;
        rows_before += seg_rows;
    }
    return items_before;
}

// Position of the I-th item of a part, advancing a batch cursor (cb, items of
// the part before batch cb) that only moves forward.
template <bool POOL>
__device__ __forceinline__ ItemIter part_item(const DecodeParams &p, const SegInfo *tab, int64_t I, int &cb,
                                              int64_t &cb_items) {
    while (cb < p.b && cb_items + (int64_t)p.h_kv * part_count<POOL>(tab[cb]) <= I) {
        cb_items += (int64_t)p.h_kv * part_count<POOL>(tab[cb]);
        ++cb;
    }
    ItemIter it;
    it.b = cb;
    it.seg = tab[cb];
    const int cnt = part_count<POOL>(it.seg);
    const int64_t off = I - cb_items;
    it.hk = (int)(off / cnt);
    it.s = part_first<POOL>(it.seg) + (int)(off - (int64_t)it.hk * cnt);
    return it;
}

// Wait until the grid this kernel depends on (the RoPE/append kernel) has
// completed and its writes are visible; returns at once without one.
__device__ __forceinline__ void wait_prerequisite_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename T, int D_QK, int D_V, int MT>
__global__ void __launch_bounds__(160, DecodeOcc<D_V, MT>::CTAS)
    decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
    using C = DecodeCfg<D_QK, D_V, MT>;
    constexpr int CHK = box_cols(D_QK), RBK = box_row_bytes(D_QK);
    constexpr int CHV = box_cols(D_V), RBV = box_row_bytes(D_V);
    constexpr int CV = D_V / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int M = p.g * p.s_q;
    const int QT = C::qt(M);
    const int QBUF = C::qbuf_bytes(M);
    const int NST = p.n_stages;
    uint8_t *sQ = smem;                       // [2][QBUF]
    uint8_t *sStage = smem + 2 * QBUF;
    float *red_o = reinterpret_cast<float *>(sStage + NST * C::STAGE);   // [4][M][D_V]
    float *red_m = red_o + 4 * M * D_V;                                   // [4][M]
    float *red_l = red_m + 4 * M;                                         // [4][M]
    uint64_t *full = reinterpret_cast<uint64_t *>(red_l + 4 * M);
    uint64_t *empty = full + kDecodeMaxStages;
    uint64_t *q_full = empty + kDecodeMaxStages;   // [2]
    uint64_t *q_empty = q_full + 2;                // [2]
    StageItem *items = reinterpret_cast<StageItem *>(q_empty + 2);            // [kDecodeMaxStages]
    int64_t *sched = reinterpret_cast<int64_t *>(items + kDecodeMaxStages);   // I0, n_static, pool, total
    SegInfo *tab = reinterpret_cast<SegInfo *>(sched + 4);                    // [b]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // allow the combine kernel (launched as a programmatic dependent) to get scheduled
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 128) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }

    // stage every batch entry's (L, N, items) once, with parallel loads
    for (int b = threadIdx.x; b < p.b; b += blockDim.x) tab[b] = seg_info(p, b);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&q_full[q], 1);
            mbar_init(&q_empty[q], 4);
        }
        fence_barrier_init();
        int64_t Rs = 0, n_pool = 0, n_all = 0;
        for (int b = 0; b < p.b; ++b) {
            Rs += (int64_t)p.h_kv * static_rows(tab[b]);
            n_pool += (int64_t)p.h_kv * pool_items(tab[b].n_items);
            n_all += (int64_t)p.h_kv * tab[b].n_items;
        }
        const int c = blockIdx.x, G = gridDim.x;
        const int64_t I0 = static_item_at_row(p, tab, Rs * c / G);
        sched[0] = I0;
        sched[1] = static_item_at_row(p, tab, Rs * (c + 1) / G) - I0;
        sched[2] = n_pool;
        sched[3] = n_all;
    }
    __syncthreads();
    const int64_t I_static = sched[0];
    const int n_static = (int)sched[1];
    const int64_t n_pool = sched[2], T_items = sched[3];
    if (blockIdx.x == 0 && threadIdx.x < 128) {
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
            for (int idx = threadIdx.x; idx < p.h_q * p.s_q * CV; idx += 128) {
                const int c = idx % CV, row = idx / CV;
                const int hq = row / p.s_q, i = row % p.s_q;
                T *dst = static_cast<T *>(p.out) + b * p.os.b + i * p.os.s + hq * p.os.h;
                reinterpret_cast<uint4 *>(dst)[c] = make_uint4(0, 0, 0, 0);
                if (c == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = -INFINITY;
            }
        }
    }
    if (T_items == 0) return;

    if (warp == 4) {
        // ---------------- producer: TMA stream of q rows and K/V tiles ----------------
        if (lane == 0) {
            // the cache is read once: evict its lines first, keeping the
            // partial results (and everything else) in L2
            const uint64_t stream_policy = l2_evict_first_policy();
            bool waited = false;   // prerequisite grid (RoPE/append) known complete
            auto ensure_waited = [&]() {
                if (!waited) {
                    wait_prerequisite_grid();
                    waited = true;
                }
            };
            int qi = 0;            // q tiles issued
            // q rows of the piece that starts at `pc`, into buffer qi % 2
            auto issue_q = [&](const ItemIter &pc) {
                const int qb = qi & 1;
                if (qi >= 2 && !mbar_wait(&q_empty[qb], ((qi >> 1) - 1) & 1, p.status)) return false;
                ensure_waited();
                mbar_arrive_expect_tx(&q_full[qb], (uint32_t)(M * D_QK * 2));
                uint8_t *qd = sQ + qb * QBUF;
#pragma unroll
                for (int c = 0; c < D_QK / CHK; ++c)
                    tma_load_4d(qd + c * QT * RBK, &tmQ, &q_full[qb], c * CHK, pc.hk * p.g, 0, pc.b);
                ++qi;
                return true;
            };
            int k = 0;              // stages issued
            ItemIter first_piece;   // the first piece's q goes out after the first tiles
            first_piece.b = -1;
            bool q0_issued = false;
            auto issue_first_q = [&]() {
                if (q0_issued || first_piece.b < 0) return true;
                q0_issued = true;
                return issue_q(first_piece);
            };
            // one stage: the item's K/V tile, after the q of a new piece
            auto issue_item = [&](const ItemIter &itm, int flags) {
                if (flags & kPieceStart) {
                    if (first_piece.b < 0) {
                        first_piece = itm;
                    } else {
                        if (!issue_first_q()) return false;
                        if (!issue_q(itm)) return false;
                    }
                }
                const int row0 = itm.seg.base + itm.s * C::TILE;
                // rows >= L of this tile were written by the RoPE/append kernel
                if (p.s_new > 0 && row0 + C::TILE > itm.seg.L) ensure_waited();
                const int s = k % NST;
                if (k >= NST && !mbar_wait(&empty[s], ((k / NST) - 1) & 1, p.status)) return false;
                items[s] = StageItem{itm.b, itm.hk, itm.s, flags};
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                uint8_t *kd = sStage + s * C::STAGE;
                uint8_t *vd = kd + C::KBYTES;
#pragma unroll
                for (int c = 0; c < D_QK / CHK; ++c)
                    tma_load_4d_hint(kd + c * C::TILE * RBK, &tmK, &full[s], c * CHK, itm.hk, row0, itm.b, stream_policy);
#pragma unroll
                for (int c = 0; c < D_V / CHV; ++c)
                    tma_load_4d_hint(vd + c * C::TILE * RBV, &tmV, &full[s], c * CHV, itm.hk, row0, itm.b, stream_policy);
                ++k;
                // the old cache rows of the first stages are in flight before q
                if (k == NST && !issue_first_q()) return false;
                return true;
            };
            bool ok = true;
            int cb = 0;            // batch cursor of part_item
            int64_t cb_items = 0;
            int grab = -1;         // claimed pool chunk, or -1
            // static share
            if (n_static > 0) {
                ItemIter it = part_item<false>(p, tab, I_static, cb, cb_items);
                for (int i = 0; i < n_static && ok; ++i) {
                    // claim the first pool chunk at the last item of the share
                    if (i == n_static - 1) {
                        ensure_waited();
                        grab = atomicAdd(p.pool, 1);
                    }
                    const int flags = ((i == 0 || it.s == 0) ? kPieceStart : 0) |
                                      ((i == n_static - 1 || it.s + 1 == static_items(it.seg.n_items)) ? kPieceEnd : 0);
                    ok = issue_item(it, flags);
                    iter_advance<false>(p, tab, it);
                }
            }
            // pool chunks
            cb = 0;
            cb_items = 0;
            while (ok) {
                if (grab < 0) {
                    ensure_waited();
                    grab = atomicAdd(p.pool, 1);
                }
                const int64_t J0 = (int64_t)grab * kPoolChunk;
                if (J0 >= n_pool) break;
                const int64_t J1 = J0 + kPoolChunk < n_pool ? J0 + kPoolChunk : n_pool;
                ItemIter it = part_item<true>(p, tab, J0, cb, cb_items);
                int next = -1;
                for (int64_t J = J0; J < J1 && ok; ++J) {
                    // claim the next chunk at this chunk's last item; its index
                    // is read after the item is issued
                    if (J == J1 - 1) next = atomicAdd(p.pool, 1);
                    const int flags = ((J == J0 || it.s == static_items(it.seg.n_items)) ? kPieceStart : 0) |
                                      ((J == J1 - 1 || it.s + 1 == it.seg.n_items) ? kPieceEnd : 0);
                    ok = issue_item(it, flags);
                    iter_advance<true>(p, tab, it);
                }
                grab = next;
            }
            if (ok) ok = issue_first_q();
            if (ok) {
                // end of stream: an item-less stage
                const int s = k % NST;
                if (k < NST || mbar_wait(&empty[s], ((k / NST) - 1) & 1, p.status)) {
                    items[s] = StageItem{0, 0, 0, kEndOfStream};
                    mbar_arrive(&full[s]);
                }
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    float o[MT][D_V / 8][4];
    float m_r[MT][2], l_r[MT][2];
    int last_vis[MT][2], first_vis[MT][2];
    int s_first = 0;
    int qi = 0;            // pieces started
    uint32_t sQa = 0;
    for (int k = 0;; ++k) {
        const int s = k % NST;
        if (!mbar_wait(&full[s], (k / NST) & 1, p.status)) break;
        const StageItem itm = items[s];
        if (itm.flags & kEndOfStream) break;
        const int b = itm.b;
        const SegInfo seg = tab[b];
        const int N = seg.N;
        const int hq0 = itm.hk * p.g;
        if (itm.flags & kPieceStart) {
            s_first = itm.s;
            const int qb = qi & 1;
            sQa = smem_addr(sQ + qb * QBUF);
            if (!mbar_wait(&q_full[qb], (qi >> 1) & 1, p.status)) break;
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
                    int64_t fv, lv;
                    visible_keys(r / p.g, N, p.s_q, p.causal, p.win_left, p.win_right, fv, lv);
                    last_vis[mt][hr] = r < M ? (int)lv : -1;
                    first_vis[mt][hr] = (int)fv;
                }
            }
        }

        // ---- one 64-row tile = one item ----
        {
            uint8_t *sK = sStage + s * C::STAGE;
            uint8_t *sV = sK + C::KBYTES;
            const int key0 = seg.base + itm.s * C::TILE + warp * 16;
            const bool tail = key0 + 16 > N;
            if (tail) {
                // rows past the sequence: zero this warp's value rows
                for (int item = lane; item < 16 * CV; item += 32) {
                    const int rr = item / CV, c = item % CV;
                    if (key0 + rr >= N)
                        *reinterpret_cast<uint4 *>(sV + swz_offset<D_V>(warp * 16 + rr, c * 8, C::TILE)) =
                            make_uint4(0, 0, 0, 0);
                }
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
                    ldmatrix_x4(sQa + swz_offset<D_QK>(mt * 16 + (lane & 15), kk * 16 + ((lane >> 4) << 3), QT),
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
                            if (j > last_vis[mt][hr] || j < first_vis[mt][hr]) v = -INFINITY;
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
            // the zeroed rows were written through the generic proxy; the next
            // TMA into this stage writes through the async proxy
            if (tail) fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }

        // ---- end of piece: release q, merge the four warps and write ----
        if (itm.flags & kPieceEnd) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_empty[qi & 1]);
            ++qi;
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
            const bool single = seg.n_items == 1;
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
                        for (int s2 = s_first + 1; s2 <= itm.s; ++s2) p.lse_part[row_slot0 + s2] = -INFINITY;
                    }
                }
            }
        }
    }
}

// One 128-thread block per (batch, query head, query row): merge the split
// slots.  The row's slots are contiguous; every thread loads up to four lse
// values (slots t, t + 128, ...) at once with the batch entry's item count,
// the block reduces max and sum, compacts the live slots (the first slot of
// each piece) in slot order, and the four warps read the live partial outputs
// with independent 16-byte loads (lane l owns columns 4 l .. 4 l + 3 and
// 4 l + 128 .. 4 l + 131), summed across warps in shared memory.
constexpr int kCombineThreads = 128;
constexpr int kCombineSlots = 4 * kCombineThreads;   // slots per row the combine handles

template <typename T>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const DecodeParams p, int d_v) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i = (int)(row % p.s_q);
    const int hq = (int)((row / p.s_q) % p.h_q);
    const int b = (int)(row / ((int64_t)p.s_q * p.h_q));
    const int64_t row_slot0 = (((int64_t)b * p.h_q + hq) * p.s_q + i) * p.n_splits;
    float ls[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int s = tid + kCombineThreads * k;
        ls[k] = s < p.n_splits ? p.lse_part[row_slot0 + s] : -INFINITY;
    }
    const SegInfo sg = seg_info(p, b);
    const int n = sg.n_items;
    if (n <= 1) return;   // written by the decode kernel (or the empty-entry path)

    __shared__ float red[4];
    __shared__ int counts[4][4];           // live slots per (k, warp)
    __shared__ int live_slot[kCombineSlots];
    __shared__ float live_w[kCombineSlots];
    __shared__ __align__(16) float acc_s[4][256];

    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (tid + kCombineThreads * k >= n) ls[k] = -INFINITY;
        mx = fmaxf(mx, ls[k]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    T *dst = static_cast<T *>(p.out) + b * p.os.b + i * p.os.s + hq * p.os.h;
    if (mx == -INFINITY) {
        for (int c = tid * 2; c < d_v; c += 2 * kCombineThreads) *reinterpret_cast<uint32_t *>(dst + c) = 0u;
        if (tid == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = -INFINITY;
        return;
    }
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) sum += ex2((ls[k] - mx) * kLog2e);
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    __syncthreads();   // everyone has read red[] (max)
    if (lane == 0) red[warp] = sum;
    unsigned live[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        live[k] = __ballot_sync(0xffffffffu, ls[k] != -INFINITY);
        if (lane == 0) counts[k][warp] = __popc(live[k]);
    }
    __syncthreads();
    const float lse = mx + logf(red[0] + red[1] + red[2] + red[3]);
    // ordered compaction: slot order is (k, warp, lane)
    int n_live = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int w = 0; w < 4; ++w) n_live += counts[k][w];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        int before = 0;
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2)
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (k2 < k || (k2 == k && w < warp)) before += counts[k2][w];
        if (ls[k] != -INFINITY) {
            const int pos = before + __popc(live[k] & ((1u << lane) - 1u));
            live_slot[pos] = tid + kCombineThreads * k;
            live_w[pos] = ex2((ls[k] - lse) * kLog2e);
        }
    }
    __syncthreads();
    float a[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
    // warp w reads live slots w, w + 4, ...: a batch of up to 16 loads per
    // column group is in flight before any is used
    constexpr int BATCH = 16;
    for (int t0 = warp; t0 < n_live; t0 += 4 * BATCH) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane * 4 + h * 128;
            if (c >= d_v) continue;
            float4 v[BATCH];
            float wgt[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int t = t0 + 4 * u;
                wgt[u] = 0.f;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (t < n_live) {
                    wgt[u] = live_w[t];
                    v[u] = *reinterpret_cast<const float4 *>(p.o_part + (row_slot0 + live_slot[t]) * d_v + c);
                }
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                a[4 * h + 0] = fmaf(wgt[u], v[u].x, a[4 * h + 0]);
                a[4 * h + 1] = fmaf(wgt[u], v[u].y, a[4 * h + 1]);
                a[4 * h + 2] = fmaf(wgt[u], v[u].z, a[4 * h + 2]);
                a[4 * h + 3] = fmaf(wgt[u], v[u].w, a[4 * h + 3]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = lane * 4 + h * 128;
        if (c < d_v) *reinterpret_cast<float4 *>(&acc_s[warp][c]) = make_float4(a[4 * h], a[4 * h + 1], a[4 * h + 2], a[4 * h + 3]);
    }
    __syncthreads();
    for (int c = tid * 2; c < d_v; c += 2 * kCombineThreads) {
        const float v0 = acc_s[0][c] + acc_s[1][c] + acc_s[2][c] + acc_s[3][c];
        const float v1 = acc_s[0][c + 1] + acc_s[1][c + 1] + acc_s[2][c + 1] + acc_s[3][c + 1];
        *reinterpret_cast<uint32_t *>(dst + c) = Elem<T>::pack2(v0, v1);
    }
    if (tid == 0 && p.lse) p.lse[((int64_t)b * p.h_q + hq) * p.s_q + i] = lse;
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

// The decode kernel is a programmatic dependent of the RoPE/append kernel
// launched just before it (its CTAs start early and wait for that grid before
// reading what it wrote); the combine kernel is a programmatic dependent of
// the decode kernel.
template <typename T, int D_QK, int D_V, int MT>
static cudaError_t run_decode(const DecodeParams &p_in, const CUtensorMap &tmQ, const CUtensorMap &tmK,
                              const CUtensorMap &tmV, cudaStream_t st) {
    using C = DecodeCfg<D_QK, D_V, MT>;
    DecodeParams p = p_in;
    const int M = p.g * p.s_q;
    p.n_stages = C::stages(M, p.b);
    const int smem = C::smem(M, p.b);
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D_QK, D_V, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sm_count() * DecodeOcc<D_V, MT>::CTAS));
    cfg.blockDim = dim3(160);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    kernel_event(0, st);
    e = cudaLaunchKernelEx(&cfg, decode_kernel<T, D_QK, D_V, MT>, tmQ, tmK, tmV, p);
    kernel_event(1, st);
    if (e != cudaSuccess) return e;
    if (p.n_splits > 1) {
        const int64_t rows = (int64_t)p.b * p.h_q * p.s_q;
        cudaLaunchConfig_t ccfg = {};
        ccfg.gridDim = dim3((unsigned)rows);
        ccfg.blockDim = dim3(kCombineThreads);
        ccfg.dynamicSmemBytes = 0;
        ccfg.stream = st;
        ccfg.attrs = attr;
        ccfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&ccfg, combine_kernel<T>, p, D_V);
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

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmQ, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, int dtype, int d_qk, int d_v, int mt, cudaStream_t st) {
#define FA_CASE(DQ, DV, MT)                                                                     \
    if (d_qk == DQ && d_v == DV && mt == MT) {                                                  \
        if (dtype == FA_DTYPE_F16) return run_decode<__half, DQ, DV, MT>(p, tmQ, tmK, tmV, st); \
        return run_decode<__nv_bfloat16, DQ, DV, MT>(p, tmQ, tmK, tmV, st);                     \
    }
    FA_DECODE_DIMS(FA_CASE)
#undef FA_CASE
    return cudaErrorInvalidValue;
}

}  // namespace fa
