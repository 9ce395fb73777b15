// fa_api.cu -- the C ABI of libfa.so: argument validation, the planner that
// picks the kernels for a call, TMA descriptor set-up and the launches.
//
// Planner (one GPU, one stream, no allocation):
//  * fa_kvcache_fwd with a short new chunk (s_q <= 8 and at most 32 query
//    rows per kv head, the decode branch of s2.cpp PR #40's eval_cached):
//    the rope+append kernel (new rows into the cache, rotated q into the
//    workspace), the persistent split-KV decode kernel as its programmatic
//    dependent, then the LSE combine when a batch entry spans several items.
//  * otherwise (the prefill / concat branch): the rope+append kernel, then
//    the attention kernel over the cache, on the same stream (write before
//    read, s2.cpp PR #40 review).
//  * fa_fwd: the attention kernel over dense k/v.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"
#include "fa_testing.h"

namespace fa {

// The device status word (one per device that loads the library).
__device__ int32_t g_status_word = 0;

namespace {

thread_local char g_last_error[512] = "";

// Query tiles per CTA forced by fa_testing_set_prefill_tiles (0: the planner decides).
int g_forced_tiles = 0;

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int32_t *status_word() {
    static int32_t *ptrs[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int32_t *>(p);
    }
    return ptrs[dev];
}

// ---------------------------------------------------------------- validation
struct Dims4 {
    int64_t n[4];
    int64_t s[4];
};

int check_tensor(const fa_tensor *t, const char *name, int ndim, int dtype, Dims4 *out,
                 bool vector_rows = true) {
    if (!t) return fail(FA_ERR_INVALID_ARG, "%s is NULL", name);
    if (t->ndim != ndim) return fail(FA_ERR_INVALID_ARG, "%s must have %d dims (got %d)", name, ndim, t->ndim);
    bool empty = false;
    for (int k = 0; k < ndim; ++k) empty = empty || t->shape[k] == 0;
    if (!t->data && !empty) return fail(FA_ERR_INVALID_ARG, "%s->data is NULL", name);
    if (t->dtype != FA_DTYPE_F16 && t->dtype != FA_DTYPE_BF16)
        return fail(FA_ERR_UNSUPPORTED, "%s: dtype %d is not fp16/bf16", name, t->dtype);
    if (dtype && t->dtype != dtype)
        return fail(FA_ERR_INVALID_ARG, "%s: dtype differs from q", name);
    for (int k = 0; k < ndim; ++k)
        if (t->shape[k] < 0) return fail(FA_ERR_INVALID_ARG, "%s: negative size", name);
    if (t->stride[ndim - 1] != 1 && t->shape[ndim - 1] > 1)
        return fail(FA_ERR_LAYOUT, "%s: innermost stride must be 1", name);
    if (vector_rows) {
        if ((reinterpret_cast<uintptr_t>(t->data) & 15) != 0)
            return fail(FA_ERR_LAYOUT, "%s: base address not 16-byte aligned", name);
        for (int k = 0; k < ndim - 1; ++k)
            if (t->shape[k] > 1 && ((t->stride[k] * 2) % 16 != 0 || t->stride[k] <= 0))
                return fail(FA_ERR_LAYOUT, "%s: stride of dim %d not a positive multiple of 16 bytes", name, k);
    } else {
        // read element by element: 2-byte alignment and positive strides suffice
        if ((reinterpret_cast<uintptr_t>(t->data) & 1) != 0)
            return fail(FA_ERR_LAYOUT, "%s: base address not 2-byte aligned", name);
        for (int k = 0; k < ndim - 1; ++k)
            if (t->shape[k] > 1 && t->stride[k] <= 0)
                return fail(FA_ERR_LAYOUT, "%s: stride of dim %d must be positive", name, k);
    }
    if (out) {
        for (int k = 0; k < 4; ++k) {
            out->n[k] = k < ndim ? t->shape[k] : 1;
            out->s[k] = k < ndim ? t->stride[k] : 0;
        }
    }
    return FA_OK;
}

bool head_dim_ok(int64_t d) { return d >= 8 && d <= 256 && d % 8 == 0; }

Strides3 s3(const Dims4 &d) { return Strides3{d.s[0], d.s[1], d.s[2]}; }

// ---------------------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 4-D map over a [batch, rows, heads, dim] tensor, dims ordered (dim, heads,
// rows, batch); box = (min(d, 64), box_h, box_rows, 1) with the swizzle that
// matches the box row width.
// L2 promotion: 256 B by default; the decode kernel's K/V maps take 128 B, because a
// kv head's row there is streamed once under evict-first, and with a
// 384-byte row (d 192) a 256-byte promotion fetches the neighbouring head's
// 128 bytes, which are often evicted before that head's CTA reads them.
int make_rows_map(CUtensorMap *map, const fa_tensor *t, int box_rows, const char *name, int box_h = 1,
                  CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const int64_t d = t->shape[3];
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)t->shape[2], (cuuint64_t)t->shape[1],
                          (cuuint64_t)t->shape[0]};
    // strides of dims 1..3 in bytes; a size-1 dim gets the packed stride
    int64_t sh = t->shape[2] > 1 ? t->stride[2] : d;
    int64_t ss = t->shape[1] > 1 ? t->stride[1] : sh * t->shape[2];
    int64_t sb = t->shape[0] > 1 ? t->stride[0] : ss * t->shape[1];
    cuuint64_t strides[3] = {(cuuint64_t)(sh * 2), (cuuint64_t)(ss * 2), (cuuint64_t)(sb * 2)};
    const int bc = d < 64 ? (int)d : 64;
    cuuint32_t box[4] = {(cuuint32_t)bc, (cuuint32_t)box_h, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMapSwizzle sw = bc * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : bc * 2 == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                          : CU_TENSOR_MAP_SWIZZLE_32B;
    CUtensorMapDataType dt = t->dtype == FA_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = fn(map, dt, 4, t->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed (%d)", name, (int)r);
    return FA_OK;
}

// ---------------------------------------------------------------- planning
struct KvPlan {
    bool decode = false;
    int mt = 1;
    int chunk = 0;
    int n_splits = 1;
    size_t ws_bytes = 0;
    size_t off_pool = 0;      // decode: workspace = q_rot | pool counter | o_part | lse_part
    size_t off_o_part = 0;
    size_t off_lse_part = 0;
    bool rotate_q_to_ws = false;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch the tcgen05 attention kernel over q (any [b, s_q, h_q, d_qk] view),
// k/v (dense [b, s_k, h_kv, d] or the caches).  Grouped heads are packed into
// the 128-row tile when g divides 128.
int run_tc_attention(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, const fa_tensor *out,
                     float *lse, bool kvcache, const int32_t *seqlens, int32_t seqlen_scalar, int64_t s_new,
                     int64_t cap, int causal, int win_left, int win_right, float scale_log2, int32_t *status,
                     cudaStream_t st, const int32_t *cu_q = nullptr, const int32_t *cu_k = nullptr,
                     int64_t n_seqs = 0, int64_t max_seqlen_q = 0) {
    // packed sequences: q/k/v/out are [1, total, h, d] views, the grid runs
    // over n_seqs sequences of at most max_seqlen_q query rows
    const bool varlen = cu_q != nullptr;
    const int64_t b = varlen ? n_seqs : q->shape[0], s_q = varlen ? max_seqlen_q : q->shape[1];
    const int64_t h_q = q->shape[2], d_qk = q->shape[3];
    const int64_t h_kv = k->shape[2], d_v = v->shape[3];
    const int64_t g = h_q / h_kv;
    const int pack = (128 % g == 0) ? (int)g : 1;
    PrefillParams p{};
    p.status = status;
    p.out = out->data;
    p.os = Strides3{out->stride[0], out->stride[1], out->stride[2]};
    p.lse = lse;
    p.seqlens = seqlens;
    p.seqlen_scalar = seqlen_scalar;
    p.s_new = (int)s_new;
    p.s_k = kvcache ? 0 : k->shape[1];
    p.cap = cap;
    p.kvcache = kvcache ? 1 : 0;
    p.b = (int)b;
    p.s_q = (int)s_q;
    p.h_q = (int)h_q;
    p.h_kv = (int)h_kv;
    p.g = (int)g;
    p.pack = pack;
    p.causal = causal ? 1 : 0;
    p.win_left = win_left;
    p.win_right = win_right;
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.total_q = varlen ? q->shape[1] : 0;
    p.total_k = varlen ? k->shape[1] : 0;
    p.n_q_tiles = (int)((s_q * pack + 127) / 128);
    p.scale_log2 = scale_log2;
    // Two query tiles per CTA keep the tensor core busy during the softmax,
    // but halve the CTA count: use them when the grid still fills the SMs
    // about twice over, or, at d_qk <= 64 (where a key tile's QK^T is short
    // next to the softmax of its 128 x 128 scores, so the second softmax
    // warpgroup pays), when it fills at least half of them once.  Measured on
    // d 64 dense attention with 128 two-tile CTAs: +24 % non-causal, +5 %
    // causal; on d 128 chunked prefill with 128 two-tile CTAs: -12 %.
    const int64_t ctas2 = (int64_t)((p.n_q_tiles + 1) / 2) * (h_q / pack) * b;
    const int64_t sms = sm_count();
    p.tiles_per_cta = (ctas2 >= 2 * sms || (d_qk <= 64 && 2 * ctas2 >= sms)) ? 2 : 1;
    // The key-split mode of the two-tile kernel (one query tile per CTA, its
    // key range halved between the two softmax warpgroups) is not chosen
    // here: on the small causal grid it measured the same as pairs of tiles
    // (d 64 dense causal 29.4 against 29.3 us per call, ten calls per graph),
    // and at d 128 slower than the one-tile kernel (chunked prefill 65.7
    // against 57.3 us).  The test hook reaches it.
    p.key_split = 0;
    // a test may pin the kernel (fa_testing_set_prefill_tiles: 3 = key split)
    if (g_forced_tiles) {
        p.tiles_per_cta = g_forced_tiles == 1 ? 1 : 2;
        p.key_split = g_forced_tiles == 3 ? 1 : 0;
    }
    // Under a causal mask the work of query tile t grows with t.  When the
    // two-tile grid is one wave, the slowest CTA sets the time, so pair tile
    // k with tile n-1-k (every CTA then sees about the same number of key
    // tiles); with several waves the heaviest-first launch order balances
    // adjacent pairs, which keep both softmax warpgroups busy to the end.
    p.pair_ends = (causal && !varlen && p.tiles_per_cta == 2 && !p.key_split && ctas2 <= sms) ? 1 : 0;
    // Over a cache the batch entries' key counts differ: order one-tile CTAs
    // by their visible keys, computed on the device (chunked prefill with one
    // long entry: 71.7 -> 63.5 us per call)
    p.work_order = (kvcache && (p.tiles_per_cta == 1 || p.key_split) && b * p.n_q_tiles <= 256) ? 1 : 0;
    const int bn = prefill_block_n((int)d_qk, (int)d_v, p.tiles_per_cta);
    CUtensorMap tmQ, tmK, tmV;
    int rc;
    if ((rc = make_rows_map(&tmQ, q, 128 / pack, "q", pack))) return rc;
    if ((rc = make_rows_map(&tmK, k, bn, "k"))) return rc;
    if ((rc = make_rows_map(&tmV, v, bn, "v"))) return rc;
    cudaError_t e = launch_prefill(p, tmQ, tmK, tmV, q->dtype, (int)d_qk, (int)d_v, st);
    if (e != cudaSuccess) return cuda_fail(e, "tcgen05 attention launch");
    return FA_OK;
}

KvPlan plan_kvcache(int64_t b, int64_t s_q, int64_t h_q, int64_t h_kv, int64_t d_qk, int64_t d_v,
                    int64_t cap, int64_t s_new, bool rotary) {
    KvPlan pl;
    const int64_t g = h_q / h_kv;
    const int64_t M = g * s_q;
    const int mt = M <= 16 ? 1 : 2;
    // the combine holds up to 512 split slots per output row in registers
    // the decode kernel stages a 16-byte record per batch entry in shared memory
    if (s_q <= 8 && M <= 32 && (s_new == 0 || s_new == s_q) && decode_supported((int)d_qk, (int)d_v, mt) &&
        cap >= 1 && cap <= 512 * 64 && b <= 1024) {
        pl.decode = true;
        pl.mt = mt;
        // The persistent decode kernel balances 64-row items across the SMs;
        // each item owns one partial-result slot.
        pl.chunk = 64;
        pl.n_splits = (int)((cap + 63) / 64);
        // the decode kernel reads q through a TMA map over a contiguous rotated copy
        pl.rotate_q_to_ws = true;
        pl.off_pool = align_up((size_t)b * s_q * h_q * d_qk * 2, 256);
        pl.off_o_part = pl.off_pool + 256;
        pl.ws_bytes = pl.off_o_part;
        if (pl.n_splits > 1) {
            const size_t rows = (size_t)pl.n_splits * b * h_q * s_q;
            pl.off_lse_part = pl.off_o_part + align_up(rows * d_v * sizeof(float), 256);
            pl.ws_bytes = pl.off_lse_part + align_up(rows * sizeof(float), 256);
        }
        return pl;
    }
    pl.decode = false;
    if (rotary) {
        pl.rotate_q_to_ws = true;
        pl.ws_bytes = align_up((size_t)b * s_q * h_q * d_qk * 2, 256);
    }
    return pl;
}

struct KvArgs {
    Dims4 q, kc, vc, kn, vn;
    int dtype;
    int64_t b, s_q, h_q, h_kv, d_qk, d_v, cap, s_new, s_ro;
    int r;
    bool has_new;
};

int validate_kvcache(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                     const fa_tensor *k_new, const fa_tensor *v_new, const fa_tensor *cos,
                     const fa_tensor *sin, int32_t rotary_dim, KvArgs *a) {
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, &a->q))) return rc;
    a->dtype = q->dtype;
    if ((rc = check_tensor(k_cache, "k_cache", 4, a->dtype, &a->kc))) return rc;
    if ((rc = check_tensor(v_cache, "v_cache", 4, a->dtype, &a->vc))) return rc;
    a->b = a->q.n[0];
    a->s_q = a->q.n[1];
    a->h_q = a->q.n[2];
    a->d_qk = a->q.n[3];
    a->cap = a->kc.n[1];
    a->h_kv = a->kc.n[2];
    a->d_v = a->vc.n[3];
    if (a->kc.n[0] != a->b || a->vc.n[0] != a->b) return fail(FA_ERR_INVALID_ARG, "cache batch differs from q");
    if (a->kc.n[3] != a->d_qk) return fail(FA_ERR_INVALID_ARG, "k_cache head dim differs from q");
    if (a->vc.n[1] != a->cap || a->vc.n[2] != a->h_kv)
        return fail(FA_ERR_INVALID_ARG, "v_cache shape differs from k_cache");
    if (a->h_kv <= 0 || a->h_q % a->h_kv != 0)
        return fail(FA_ERR_INVALID_ARG, "h_q (%lld) must be a multiple of h_kv (%lld)", (long long)a->h_q,
                    (long long)a->h_kv);
    if (!head_dim_ok(a->d_qk) || !head_dim_ok(a->d_v))
        return fail(FA_ERR_UNSUPPORTED, "head dims must be multiples of 8 in 8..256 (got %lld/%lld)",
                    (long long)a->d_qk, (long long)a->d_v);
    if (a->cap > INT32_MAX || a->s_q > INT32_MAX) return fail(FA_ERR_INVALID_ARG, "sequence too long");
    a->has_new = k_new != nullptr;
    if ((k_new == nullptr) != (v_new == nullptr))
        return fail(FA_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
    a->s_new = 0;
    if (a->has_new) {
        if ((rc = check_tensor(k_new, "k_new", 4, a->dtype, &a->kn))) return rc;
        if ((rc = check_tensor(v_new, "v_new", 4, a->dtype, &a->vn))) return rc;
        a->s_new = a->kn.n[1];
        if (a->kn.n[0] != a->b || a->kn.n[2] != a->h_kv || a->kn.n[3] != a->d_qk)
            return fail(FA_ERR_INVALID_ARG, "k_new shape must be [b, s_new, h_kv, d_qk]");
        if (a->vn.n[0] != a->b || a->vn.n[1] != a->s_new || a->vn.n[2] != a->h_kv || a->vn.n[3] != a->d_v)
            return fail(FA_ERR_INVALID_ARG, "v_new shape must be [b, s_new, h_kv, d_v]");
        if (a->s_new != a->s_q)
            return fail(FA_ERR_INVALID_ARG, "s_new (%lld) must equal s_q (%lld)", (long long)a->s_new,
                        (long long)a->s_q);
        if (a->s_new > a->cap) return fail(FA_ERR_INVALID_ARG, "s_new exceeds the cache capacity");
    }
    a->r = 0;
    a->s_ro = 0;
    if ((cos == nullptr) != (sin == nullptr))
        return fail(FA_ERR_INVALID_ARG, "cos and sin must both be given or both be NULL");
    if (cos) {
        Dims4 dc, ds;
        if ((rc = check_tensor(cos, "cos", 2, a->dtype, &dc, false))) return rc;
        if ((rc = check_tensor(sin, "sin", 2, a->dtype, &ds, false))) return rc;
        if (dc.n[0] != ds.n[0] || dc.n[1] != ds.n[1] || dc.s[0] != ds.s[0])
            return fail(FA_ERR_INVALID_ARG, "cos and sin must have the same shape and strides");
        if (rotary_dim < 0 || rotary_dim % 2 || rotary_dim > a->d_qk)
            return fail(FA_ERR_INVALID_ARG, "rotary_dim must be even and <= d_qk (got %d)", rotary_dim);
        if (rotary_dim > 0 && dc.n[1] < rotary_dim / 2)
            return fail(FA_ERR_INVALID_ARG, "cos/sin need rotary_dim/2 = %d columns (got %lld)", rotary_dim / 2,
                        (long long)dc.n[1]);
        a->r = rotary_dim;
        a->s_ro = dc.n[0];
    }
    return FA_OK;
}

}  // namespace

int set_last_error(int code, const char *msg) { return fail(code, "%s", msg); }

static cudaEvent_t g_kernel_events[2] = {nullptr, nullptr};

void kernel_event(int which, cudaStream_t st) {
    cudaEvent_t ev = g_kernel_events[which];
    if (!ev) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, st);
}

}  // namespace fa

using namespace fa;

extern "C" {

int fa_version(void) { return 100; }

int fa_rotary(const fa_tensor *x, const fa_tensor *cos, const fa_tensor *sin,
              const int32_t *seqlen_offsets, int32_t seqlen_offset_scalar,
              const int32_t *cu_seqlens, int32_t n_seqs,
              int32_t rotary_dim, int32_t interleaved, int32_t conjugate,
              const fa_tensor *out, void *stream) {
    g_last_error[0] = 0;
    Dims4 xd, od;
    int rc;
    if ((rc = check_tensor(x, "x", 4, 0, &xd))) return rc;
    if ((rc = check_tensor(out, "out", 4, x->dtype, &od))) return rc;
    for (int k = 0; k < 4; ++k)
        if (xd.n[k] != od.n[k]) return fail(FA_ERR_INVALID_ARG, "out must have the shape of x");
    const int64_t d = xd.n[3];
    if (d % 8 || d > 256) return fail(FA_ERR_UNSUPPORTED, "rotary needs d a multiple of 8 and <= 256 (got %lld)",
                                      (long long)d);
    if (rotary_dim < 0 || rotary_dim % 2 || rotary_dim > d)
        return fail(FA_ERR_INVALID_ARG, "rotary_dim must be even and <= d (got %d)", rotary_dim);
    if (cu_seqlens && (xd.n[0] != 1 || n_seqs < 1))
        return fail(FA_ERR_INVALID_ARG, "packed rows need x of shape [1, total, h, d] and n_seqs >= 1");
    if (!cu_seqlens && n_seqs != 0) return fail(FA_ERR_INVALID_ARG, "n_seqs without cu_seqlens");
    int64_t s_ro = 0, cs_row = 0;
    if (rotary_dim > 0) {
        if (!cos || !sin) return fail(FA_ERR_INVALID_ARG, "cos and sin are needed when rotary_dim > 0");
        Dims4 dc, ds;
        if ((rc = check_tensor(cos, "cos", 2, x->dtype, &dc, false))) return rc;
        if ((rc = check_tensor(sin, "sin", 2, x->dtype, &ds, false))) return rc;
        if (dc.n[0] != ds.n[0] || dc.n[1] != ds.n[1] || dc.s[0] != ds.s[0])
            return fail(FA_ERR_INVALID_ARG, "cos and sin must have the same shape and strides");
        if (dc.n[1] < rotary_dim / 2)
            return fail(FA_ERR_INVALID_ARG, "cos/sin need rotary_dim/2 = %d columns (got %lld)", rotary_dim / 2,
                        (long long)dc.n[1]);
        s_ro = dc.n[0];
        cs_row = dc.n[0] > 1 ? dc.s[0] : dc.n[1];
    }
    const int64_t rows = xd.n[0] * xd.n[1];
    if (rows == 0 || xd.n[2] == 0 || d == 0) return FA_OK;
    int32_t *status = status_word();
    if (!status) return fail(FA_ERR_CUDA, "no CUDA device");
    RotaryParams p{};
    p.status = status;
    p.x = x->data;
    p.xs = s3(xd);
    p.out = out->data;
    p.os = s3(od);
    p.cos = rotary_dim > 0 ? cos->data : nullptr;
    p.sin = rotary_dim > 0 ? sin->data : nullptr;
    p.cs_row = cs_row;
    p.cs_rows = s_ro;
    p.offsets = seqlen_offsets;
    p.offset_scalar = seqlen_offset_scalar;
    p.cu_seqlens = cu_seqlens;
    p.n_seqs = cu_seqlens ? n_seqs : 0;
    p.rows = rows;
    p.s = (int)xd.n[1];
    p.h = (int)xd.n[2];
    p.d = (int)d;
    p.r = rotary_dim;
    p.interleaved = interleaved ? 1 : 0;
    p.conjugate = conjugate ? 1 : 0;
    cudaError_t e = launch_rotary(p, x->dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rotary launch");
    return FA_OK;
}

int fa_testing_set_prefill_tiles(int32_t tiles) {
    if (tiles < 0 || tiles > 3) return fail(FA_ERR_INVALID_ARG, "prefill kernel choice must be 0, 1, 2 or 3");
    g_forced_tiles = tiles;
    return FA_OK;
}

int fa_set_kernel_events(void *start, void *stop) {
    if ((start == nullptr) != (stop == nullptr))
        return fail(FA_ERR_INVALID_ARG, "fa_set_kernel_events: pass both events or neither");
    g_kernel_events[0] = static_cast<cudaEvent_t>(start);
    g_kernel_events[1] = static_cast<cudaEvent_t>(stop);
    return FA_OK;
}

const char *fa_last_error(void) { return g_last_error; }

const char *fa_status_string(int s) {
    switch (s) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG: return "invalid argument";
        case FA_ERR_UNSUPPORTED: return "unsupported dtype or head dim";
        case FA_ERR_LAYOUT: return "unsupported memory layout";
        case FA_ERR_WORKSPACE: return "workspace missing or too small";
        case FA_ERR_CUDA: return "CUDA error";
        case FA_ERR_DEVICE_PRECONDITION: return "cache_seqlens out of range (recorded on the device)";
        case FA_ERR_DEVICE_TIMEOUT: return "bounded wait timed out on the device";
        default: return "unknown status";
    }
}

int fa_kvcache_workspace_size(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                              const fa_tensor *k_new, int32_t rotary_dim, size_t *bytes) {
    g_last_error[0] = 0;
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes is NULL");
    KvArgs a;
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, &a.q))) return rc;
    if ((rc = check_tensor(k_cache, "k_cache", 4, q->dtype, &a.kc))) return rc;
    if ((rc = check_tensor(v_cache, "v_cache", 4, q->dtype, &a.vc))) return rc;
    if (a.kc.n[2] <= 0 || a.q.n[2] % a.kc.n[2]) return fail(FA_ERR_INVALID_ARG, "h_q must be a multiple of h_kv");
    int64_t s_new = k_new ? k_new->shape[1] : 0;
    KvPlan pl = plan_kvcache(a.q.n[0], a.q.n[1], a.q.n[2], a.kc.n[2], a.q.n[3], a.vc.n[3], a.kc.n[1], s_new,
                             rotary_dim > 0);
    *bytes = pl.ws_bytes;
    return FA_OK;
}

int fa_kvcache_plan(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                    const fa_tensor *k_new, int32_t rotary_dim, fa_plan *plan) {
    g_last_error[0] = 0;
    if (!plan) return fail(FA_ERR_INVALID_ARG, "plan is NULL");
    Dims4 qd, kd, vd;
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, &qd))) return rc;
    if ((rc = check_tensor(k_cache, "k_cache", 4, q->dtype, &kd))) return rc;
    if ((rc = check_tensor(v_cache, "v_cache", 4, q->dtype, &vd))) return rc;
    if (kd.n[2] <= 0 || qd.n[2] % kd.n[2]) return fail(FA_ERR_INVALID_ARG, "h_q must be a multiple of h_kv");
    const int64_t s_new = k_new ? k_new->shape[1] : 0;
    const KvPlan pl = plan_kvcache(qd.n[0], qd.n[1], qd.n[2], kd.n[2], qd.n[3], vd.n[3], kd.n[1], s_new,
                                   rotary_dim > 0);
    plan->path = pl.decode ? FA_PATH_DECODE : FA_PATH_PREFILL;
    plan->n_splits = pl.decode ? pl.n_splits : 1;
    plan->chunk = pl.decode ? pl.chunk : 0;
    plan->launches = pl.decode ? (pl.n_splits > 1 ? 3 : 2) : ((s_new > 0 || rotary_dim > 0) ? 2 : 1);
    plan->workspace_bytes = pl.ws_bytes;
    return FA_OK;
}

int fa_fwd_plan(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, fa_plan *plan) {
    g_last_error[0] = 0;
    if (!plan) return fail(FA_ERR_INVALID_ARG, "plan is NULL");
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, nullptr))) return rc;
    if ((rc = check_tensor(k, "k", 4, q->dtype, nullptr))) return rc;
    if ((rc = check_tensor(v, "v", 4, q->dtype, nullptr))) return rc;
    plan->path = FA_PATH_DENSE;
    plan->launches = 1;
    plan->n_splits = 1;
    plan->chunk = 0;
    plan->workspace_bytes = 0;
    return FA_OK;
}

int fa_kvcache_fwd(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                   const fa_tensor *k_new, const fa_tensor *v_new, const fa_tensor *cos,
                   const fa_tensor *sin, const int32_t *cache_seqlens, int32_t rotary_dim,
                   int32_t interleaved, int32_t causal, float scale, const fa_tensor *out, float *lse,
                   int32_t cache_seqlens_scalar, void *workspace, size_t workspace_bytes, void *stream) {
    return fa_kvcache_fwd_window(q, k_cache, v_cache, k_new, v_new, cos, sin, cache_seqlens, rotary_dim,
                                 interleaved, causal, -1, -1, scale, out, lse, cache_seqlens_scalar, workspace,
                                 workspace_bytes, stream);
}

int fa_kvcache_fwd_window(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                          const fa_tensor *k_new, const fa_tensor *v_new, const fa_tensor *cos,
                          const fa_tensor *sin, const int32_t *cache_seqlens, int32_t rotary_dim,
                          int32_t interleaved, int32_t causal, int32_t window_left, int32_t window_right,
                          float scale, const fa_tensor *out, float *lse, int32_t cache_seqlens_scalar,
                          void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error[0] = 0;
    if (window_left < -1 || window_right < -1)
        return fail(FA_ERR_INVALID_ARG, "window bounds must be >= -1 (-1 = unbounded)");
    KvArgs a;
    int rc = validate_kvcache(q, k_cache, v_cache, k_new, v_new, cos, sin, rotary_dim, &a);
    if (rc) return rc;
    Dims4 od;
    if ((rc = check_tensor(out, "out", 4, a.dtype, &od))) return rc;
    if (od.n[0] != a.b || od.n[1] != a.s_q || od.n[2] != a.h_q || od.n[3] != a.d_v)
        return fail(FA_ERR_INVALID_ARG, "out shape must be [b, s_q, h_q, d_v]");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) return fail(FA_ERR_LAYOUT, "lse not 4-byte aligned");
    if (!cache_seqlens) {
        const int64_t L = cache_seqlens_scalar;
        if (L < 0 || L + a.s_new > a.cap)
            return fail(FA_ERR_INVALID_ARG, "cache_seqlens %lld + s_new %lld outside capacity %lld", (long long)L,
                        (long long)a.s_new, (long long)a.cap);
        if (a.r > 0 && L + std::max(a.s_q, a.s_new) > a.s_ro)
            return fail(FA_ERR_INVALID_ARG, "rotary table has %lld rows, positions reach %lld", (long long)a.s_ro,
                        (long long)(L + std::max(a.s_q, a.s_new)));
    }
    const KvPlan pl = plan_kvcache(a.b, a.s_q, a.h_q, a.h_kv, a.d_qk, a.d_v, a.cap, a.s_new, a.r > 0);
    if (pl.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < pl.ws_bytes))
        return fail(FA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", pl.ws_bytes, workspace_bytes);
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(FA_ERR_LAYOUT, "workspace must be 256-byte aligned");
    if (a.b == 0 || a.s_q == 0 || a.h_q == 0) return FA_OK;
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)a.d_qk);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t *status = status_word();
    if (!status) return fail(FA_ERR_CUDA, "no CUDA device");
    const int cs_row = cos ? (int)cos->stride[0] : 0;

    // The rope+append kernel: rotated k_new and raw v_new into the cache at
    // L_b, and (when asked) q rotated at L_b + i into `q_rot`.
    auto rope_append = [&](void *q_rot, int32_t *zero_word) -> int {
        RopeAppendParams p{};
        p.status = status;
        p.k_new = a.has_new ? k_new->data : nullptr;
        p.kn = a.has_new ? s3(a.kn) : Strides3{0, 0, 0};
        p.v_new = a.has_new ? v_new->data : nullptr;
        p.vn = a.has_new ? s3(a.vn) : Strides3{0, 0, 0};
        p.k_cache = k_cache->data;
        p.kc = s3(a.kc);
        p.v_cache = v_cache->data;
        p.vc = s3(a.vc);
        p.q = q->data;
        p.qs = s3(a.q);
        p.q_rot = q_rot;
        p.cos = a.r ? cos->data : nullptr;
        p.sin = a.r ? sin->data : nullptr;
        p.cs_row = cs_row;
        p.cs_rows = a.s_ro;
        p.seqlens = cache_seqlens;
        p.seqlen_scalar = cache_seqlens_scalar;
        p.b = (int)a.b;
        p.s_q = (int)a.s_q;
        p.s_new = (int)a.s_new;
        p.h_q = (int)a.h_q;
        p.h_kv = (int)a.h_kv;
        p.d_qk = (int)a.d_qk;
        p.d_v = (int)a.d_v;
        p.r = a.r;
        p.interleaved = interleaved ? 1 : 0;
        p.cap = a.cap;
        p.zero_word = zero_word;
        cudaError_t e = launch_rope_append(p, a.dtype, st);
        if (e != cudaSuccess) return cuda_fail(e, "rope/append launch");
        return FA_OK;
    };

    if (pl.decode) {
        char *ws = static_cast<char *>(workspace);
        int32_t *pool = reinterpret_cast<int32_t *>(ws + pl.off_pool);
        if ((rc = rope_append(workspace, pool))) return rc;
        // q rows in the workspace: contiguous [b, s_q, h_q, d_qk]
        fa_tensor qr = *q;
        qr.data = workspace;
        qr.stride[3] = 1;
        qr.stride[2] = a.d_qk;
        qr.stride[1] = a.h_q * a.d_qk;
        qr.stride[0] = a.s_q * a.h_q * a.d_qk;
        CUtensorMap tmQ, tmK, tmV;
        if ((rc = make_rows_map(&tmQ, &qr, (int)a.s_q, "q_rot", (int)(a.h_q / a.h_kv)))) return rc;
        if ((rc = make_rows_map(&tmK, k_cache, 64, "k_cache", 1, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))) return rc;
        if ((rc = make_rows_map(&tmV, v_cache, 64, "v_cache", 1, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))) return rc;
        DecodeParams p{};
        p.status = status;
        p.cs_rows = a.s_ro;
        p.seqlens = cache_seqlens;
        p.seqlen_scalar = cache_seqlens_scalar;
        p.out = out->data;
        p.os = s3(od);
        p.lse = lse;
        p.pool = pool;
        p.o_part = pl.n_splits > 1 ? reinterpret_cast<float *>(ws + pl.off_o_part) : nullptr;
        p.lse_part = pl.n_splits > 1 ? reinterpret_cast<float *>(ws + pl.off_lse_part) : nullptr;
        p.b = (int)a.b;
        p.s_q = (int)a.s_q;
        p.s_new = (int)a.s_new;
        p.h_q = (int)a.h_q;
        p.h_kv = (int)a.h_kv;
        p.g = (int)(a.h_q / a.h_kv);
        p.r = a.r;
        p.causal = causal ? 1 : 0;
        p.win_left = window_left;
        p.win_right = window_right;
        p.cap = a.cap;
        p.scale_log2 = sc * 1.4426950408889634f;
        p.chunk = pl.chunk;
        p.n_splits = pl.n_splits;
        cudaError_t e = launch_decode(p, tmQ, tmK, tmV, a.dtype, (int)a.d_qk, (int)a.d_v, pl.mt, st);
        if (e != cudaSuccess) return cuda_fail(e, "decode launch");
        return FA_OK;
    }

    // prefill / chunked path: rotate + append, then attention over the cache
    void *q_att = q->data;
    Strides3 q_att_s = s3(a.q);
    if (a.has_new || pl.rotate_q_to_ws) {
        if ((rc = rope_append(pl.rotate_q_to_ws ? workspace : nullptr, nullptr))) return rc;
        if (pl.rotate_q_to_ws) {
            q_att = workspace;
            q_att_s = Strides3{a.s_q * a.h_q * a.d_qk, a.h_q * a.d_qk, a.d_qk};
        }
    }
    if (prefill_supported((int)a.d_qk, (int)a.d_v)) {
        fa_tensor qd = *q;
        qd.data = q_att;
        qd.stride[0] = q_att_s.b;
        qd.stride[1] = q_att_s.s;
        qd.stride[2] = q_att_s.h;
        qd.stride[3] = 1;
        return run_tc_attention(&qd, k_cache, v_cache, out, lse, true, cache_seqlens, cache_seqlens_scalar,
                                a.s_new, a.cap, causal, window_left, window_right, sc * 1.4426950408889634f,
                                status, st);
    }
    SimtAttnParams p{};
    p.status = status;
    p.q = q_att;
    p.qs = q_att_s;
    p.k = k_cache->data;
    p.ks = s3(a.kc);
    p.v = v_cache->data;
    p.vs = s3(a.vc);
    p.out = out->data;
    p.os = s3(od);
    p.lse = lse;
    p.seqlens = cache_seqlens;
    p.seqlen_scalar = cache_seqlens_scalar;
    p.s_new = (int)a.s_new;
    p.s_k = 0;
    p.cap = a.cap;
    p.b = (int)a.b;
    p.s_q = (int)a.s_q;
    p.h_q = (int)a.h_q;
    p.h_kv = (int)a.h_kv;
    p.g = (int)(a.h_q / a.h_kv);
    p.d_qk = (int)a.d_qk;
    p.d_v = (int)a.d_v;
    p.causal = causal ? 1 : 0;
    p.win_left = window_left;
    p.win_right = window_right;
    p.scale_log2 = sc * 1.4426950408889634f;
    cudaError_t e = launch_simt_attn(p, a.dtype, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return FA_OK;
}

int fa_fwd_workspace_size(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, size_t *bytes) {
    g_last_error[0] = 0;
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes is NULL");
    (void)q;
    (void)k;
    (void)v;
    *bytes = 0;
    return FA_OK;
}

int fa_fwd(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, int32_t causal, float scale,
           const fa_tensor *out, float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    return fa_fwd_window(q, k, v, causal, -1, -1, scale, out, lse, workspace, workspace_bytes, stream);
}

int fa_fwd_window(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, int32_t causal, int32_t window_left,
                  int32_t window_right, float scale, const fa_tensor *out, float *lse, void *workspace,
                  size_t workspace_bytes, void *stream) {
    g_last_error[0] = 0;
    if (window_left < -1 || window_right < -1)
        return fail(FA_ERR_INVALID_ARG, "window bounds must be >= -1 (-1 = unbounded)");
    (void)workspace;
    (void)workspace_bytes;
    Dims4 qd, kd, vd, od;
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, &qd))) return rc;
    if ((rc = check_tensor(k, "k", 4, q->dtype, &kd))) return rc;
    if ((rc = check_tensor(v, "v", 4, q->dtype, &vd))) return rc;
    if ((rc = check_tensor(out, "out", 4, q->dtype, &od))) return rc;
    const int64_t b = qd.n[0], s_q = qd.n[1], h_q = qd.n[2], d_qk = qd.n[3];
    const int64_t s_k = kd.n[1], h_kv = kd.n[2], d_v = vd.n[3];
    if (kd.n[0] != b || vd.n[0] != b) return fail(FA_ERR_INVALID_ARG, "k/v batch differs from q");
    if (kd.n[3] != d_qk) return fail(FA_ERR_INVALID_ARG, "k head dim differs from q");
    if (vd.n[1] != s_k || vd.n[2] != h_kv) return fail(FA_ERR_INVALID_ARG, "v shape differs from k");
    if (h_kv <= 0 || h_q % h_kv) return fail(FA_ERR_INVALID_ARG, "h_q must be a multiple of h_kv");
    if (!head_dim_ok(d_qk) || !head_dim_ok(d_v))
        return fail(FA_ERR_UNSUPPORTED, "head dims must be multiples of 8 in 8..256");
    if (od.n[0] != b || od.n[1] != s_q || od.n[2] != h_q || od.n[3] != d_v)
        return fail(FA_ERR_INVALID_ARG, "out shape must be [b, s_q, h_q, d_v]");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) return fail(FA_ERR_LAYOUT, "lse not 4-byte aligned");
    if (b == 0 || s_q == 0 || h_q == 0) return FA_OK;
    int32_t *status = status_word();
    if (!status) return fail(FA_ERR_CUDA, "no CUDA device");
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d_qk);
    if (prefill_supported((int)d_qk, (int)d_v))
        return run_tc_attention(q, k, v, out, lse, false, nullptr, 0, 0, 0, causal, window_left, window_right,
                                sc * 1.4426950408889634f, status, static_cast<cudaStream_t>(stream));
    SimtAttnParams p{};
    p.status = status;
    p.q = q->data;
    p.qs = s3(qd);
    p.k = k->data;
    p.ks = s3(kd);
    p.v = v->data;
    p.vs = s3(vd);
    p.out = out->data;
    p.os = s3(od);
    p.lse = lse;
    p.seqlens = nullptr;
    p.s_k = s_k;
    p.cap = 0;
    p.b = (int)b;
    p.s_q = (int)s_q;
    p.h_q = (int)h_q;
    p.h_kv = (int)h_kv;
    p.g = (int)(h_q / h_kv);
    p.d_qk = (int)d_qk;
    p.d_v = (int)d_v;
    p.causal = causal ? 1 : 0;
    p.win_left = window_left;
    p.win_right = window_right;
    p.scale_log2 = sc * 1.4426950408889634f;
    cudaError_t e = launch_simt_attn(p, q->dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return FA_OK;
}

int fa_fwd_varlen(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, const int32_t *cu_seqlens_q,
                  const int32_t *cu_seqlens_k, int32_t n_seqs, int32_t max_seqlen_q, int32_t causal,
                  int32_t window_left, int32_t window_right, float scale, const fa_tensor *out, float *lse,
                  void *stream) {
    g_last_error[0] = 0;
    if (window_left < -1 || window_right < -1)
        return fail(FA_ERR_INVALID_ARG, "window bounds must be >= -1 (-1 = unbounded)");
    Dims4 qd, kd, vd, od;
    int rc;
    if ((rc = check_tensor(q, "q", 3, 0, &qd))) return rc;
    if ((rc = check_tensor(k, "k", 3, q->dtype, &kd))) return rc;
    if ((rc = check_tensor(v, "v", 3, q->dtype, &vd))) return rc;
    if ((rc = check_tensor(out, "out", 3, q->dtype, &od))) return rc;
    const int64_t total_q = qd.n[0], h_q = qd.n[1], d_qk = qd.n[2];
    const int64_t total_k = kd.n[0], h_kv = kd.n[1], d_v = vd.n[2];
    if (kd.n[2] != d_qk) return fail(FA_ERR_INVALID_ARG, "k head dim differs from q");
    if (vd.n[0] != total_k || vd.n[1] != h_kv) return fail(FA_ERR_INVALID_ARG, "v shape differs from k");
    if (h_kv <= 0 || h_q % h_kv) return fail(FA_ERR_INVALID_ARG, "h_q must be a multiple of h_kv");
    if (od.n[0] != total_q || od.n[1] != h_q || od.n[2] != d_v)
        return fail(FA_ERR_INVALID_ARG, "out shape must be [total_q, h_q, d_v]");
    if (!cu_seqlens_q || !cu_seqlens_k || n_seqs < 0 || max_seqlen_q < 0)
        return fail(FA_ERR_INVALID_ARG, "cu_seqlens_q/k, n_seqs >= 0 and max_seqlen_q >= 0 are required");
    if (!prefill_supported((int)d_qk, (int)d_v))
        return fail(FA_ERR_UNSUPPORTED, "packed sequences need head dims the tcgen05 kernel takes "
                    "(d_qk/d_v in 64/64, 128/128, 192/128, 128/64, 64/128, 192/64)");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) return fail(FA_ERR_LAYOUT, "lse not 4-byte aligned");
    if (n_seqs == 0 || max_seqlen_q == 0 || total_q == 0 || h_q == 0) return FA_OK;
    int32_t *status = status_word();
    if (!status) return fail(FA_ERR_CUDA, "no CUDA device");
    // [total, h, d] as a batch of one [1, total, h, d]
    auto as4 = [](const fa_tensor *t) {
        fa_tensor r = *t;
        r.ndim = 4;
        r.shape[3] = t->shape[2];
        r.shape[2] = t->shape[1];
        r.shape[1] = t->shape[0];
        r.shape[0] = 1;
        r.stride[3] = 1;
        r.stride[2] = t->stride[1];
        r.stride[1] = t->stride[0];
        r.stride[0] = t->stride[0] * t->shape[0];
        return r;
    };
    const fa_tensor q4 = as4(q), k4 = as4(k), v4 = as4(v), o4 = as4(out);
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d_qk);
    return run_tc_attention(&q4, &k4, &v4, &o4, lse, false, nullptr, 0, 0, 0, causal, window_left, window_right,
                            sc * 1.4426950408889634f, status, static_cast<cudaStream_t>(stream), cu_seqlens_q,
                            cu_seqlens_k, n_seqs, max_seqlen_q);
}

int fa_bwd_workspace_size(const fa_tensor *q, size_t *bytes) {
    g_last_error[0] = 0;
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes is NULL");
    Dims4 qd;
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, &qd))) return rc;
    // lse * log2(e) and D_i, each [b, h_q, s_q rounded up to 64]
    const size_t rows = (size_t)qd.n[0] * qd.n[2] * (size_t)((qd.n[1] + 63) / 64 * 64);
    *bytes = 2 * align_up(rows * sizeof(float), 256);
    return FA_OK;
}

int fa_bwd(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, const fa_tensor *out,
           const fa_tensor *dout, const float *lse, int32_t causal, int32_t window_left, int32_t window_right,
           float scale, const fa_tensor *dq, const fa_tensor *dk, const fa_tensor *dv, void *workspace,
           size_t workspace_bytes, void *stream) {
    g_last_error[0] = 0;
    if (window_left < -1 || window_right < -1)
        return fail(FA_ERR_INVALID_ARG, "window bounds must be >= -1 (-1 = unbounded)");
    Dims4 qd, kd, vd, od, dod, dqd, dkd, dvd;
    int rc;
    if ((rc = check_tensor(q, "q", 4, 0, &qd))) return rc;
    if ((rc = check_tensor(k, "k", 4, q->dtype, &kd))) return rc;
    if ((rc = check_tensor(v, "v", 4, q->dtype, &vd))) return rc;
    if ((rc = check_tensor(out, "out", 4, q->dtype, &od))) return rc;
    if ((rc = check_tensor(dout, "dout", 4, q->dtype, &dod))) return rc;
    if ((rc = check_tensor(dq, "dq", 4, q->dtype, &dqd))) return rc;
    if ((rc = check_tensor(dk, "dk", 4, q->dtype, &dkd))) return rc;
    if ((rc = check_tensor(dv, "dv", 4, q->dtype, &dvd))) return rc;
    const int64_t b = qd.n[0], s_q = qd.n[1], h_q = qd.n[2], d_qk = qd.n[3];
    const int64_t s_k = kd.n[1], h_kv = kd.n[2], d_v = vd.n[3];
    if (kd.n[0] != b || vd.n[0] != b) return fail(FA_ERR_INVALID_ARG, "k/v batch differs from q");
    if (kd.n[3] != d_qk) return fail(FA_ERR_INVALID_ARG, "k head dim differs from q");
    if (vd.n[1] != s_k || vd.n[2] != h_kv) return fail(FA_ERR_INVALID_ARG, "v shape differs from k");
    if (h_kv <= 0 || h_q % h_kv) return fail(FA_ERR_INVALID_ARG, "h_q must be a multiple of h_kv");
    auto same = [](const Dims4 &a, int64_t n0, int64_t n1, int64_t n2, int64_t n3) {
        return a.n[0] == n0 && a.n[1] == n1 && a.n[2] == n2 && a.n[3] == n3;
    };
    if (!same(od, b, s_q, h_q, d_v)) return fail(FA_ERR_INVALID_ARG, "out shape must be [b, s_q, h_q, d_v]");
    if (!same(dod, b, s_q, h_q, d_v)) return fail(FA_ERR_INVALID_ARG, "dout shape must be [b, s_q, h_q, d_v]");
    if (!same(dqd, b, s_q, h_q, d_qk)) return fail(FA_ERR_INVALID_ARG, "dq shape must be that of q");
    if (!same(dkd, b, s_k, h_kv, d_qk)) return fail(FA_ERR_INVALID_ARG, "dk shape must be that of k");
    if (!same(dvd, b, s_k, h_kv, d_v)) return fail(FA_ERR_INVALID_ARG, "dv shape must be that of v");
    if (!bwd_supported((int)d_qk, (int)d_v))
        return fail(FA_ERR_UNSUPPORTED, "backward head dims (d_qk, d_v) must be 64/64, 128/128 or 192/128");
    if (s_q > INT32_MAX || s_k > INT32_MAX || b > 65535 || h_q > 65535)
        return fail(FA_ERR_UNSUPPORTED, "sizes past the launch limits");
    if (!lse && b * s_q * h_q > 0) return fail(FA_ERR_INVALID_ARG, "lse is NULL");
    if (reinterpret_cast<uintptr_t>(lse) & 3) return fail(FA_ERR_LAYOUT, "lse not 4-byte aligned");
    if (b == 0 || h_q == 0) return FA_OK;
    size_t need = 0;
    if ((rc = fa_bwd_workspace_size(q, &need))) return rc;
    if (workspace_bytes < need || (need && !workspace))
        return fail(FA_ERR_WORKSPACE, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) & 15) return fail(FA_ERR_LAYOUT, "workspace not 16-byte aligned");
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)d_qk);
    int32_t *status = status_word();
    if (!status) return fail(FA_ERR_CUDA, "no CUDA device");
    BwdParams p{};
    p.status = status;
    p.q = q->data;
    p.qs = s3(qd);
    p.k = k->data;
    p.ks = s3(kd);
    p.v = v->data;
    p.vs = s3(vd);
    p.out = out->data;
    p.os = s3(od);
    p.dout = dout->data;
    p.dos = s3(dod);
    p.lse = lse;
    p.s_q_pad = (int)((s_q + 63) / 64 * 64);
    p.lsum = static_cast<float *>(workspace);
    p.dsum = reinterpret_cast<float *>(static_cast<char *>(workspace) + need / 2);
    p.dq = dq->data;
    p.dqs = s3(dqd);
    p.dk = dk->data;
    p.dks = s3(dkd);
    p.dv = dv->data;
    p.dvs = s3(dvd);
    p.b = (int)b;
    p.s_q = (int)s_q;
    p.s_k = (int)s_k;
    p.h_q = (int)h_q;
    p.h_kv = (int)h_kv;
    p.g = (int)(h_q / h_kv);
    p.d_qk = (int)d_qk;
    p.d_v = (int)d_v;
    p.causal = causal ? 1 : 0;
    p.win_left = window_left;
    p.win_right = window_right;
    p.scale = sc;
    p.scale_log2 = sc * 1.4426950408889634f;
    // TMA maps of the tiles the kernels load; a side with no rows (s_q or s_k
    // = 0) is never loaded (the kernels then only write zeros), and a map
    // cannot be encoded over it
    BwdMaps m;
    std::memset(&m, 0, sizeof(m));
    auto map = [&](CUtensorMap *tm, const fa_tensor *t, int rows, const char *name) {
        return t->shape[1] == 0 ? (int)FA_OK : make_rows_map(tm, t, rows, name);
    };
    if ((rc = map(&m.k128, k, 128, "k"))) return rc;
    if ((rc = map(&m.v128, v, 128, "v"))) return rc;
    if ((rc = map(&m.q64, q, 64, "q"))) return rc;
    if ((rc = map(&m.do64, dout, 64, "dout"))) return rc;
    if ((rc = map(&m.q128, q, 128, "q"))) return rc;
    if ((rc = map(&m.do128, dout, 128, "dout"))) return rc;
    if ((rc = map(&m.k64, k, 64, "k"))) return rc;
    if ((rc = map(&m.v64, v, 64, "v"))) return rc;
    cudaError_t e = launch_bwd(p, m, q->dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return FA_OK;
}

int fa_device_status(void *stream, int32_t *status) {
    g_last_error[0] = 0;
    if (!status) return fail(FA_ERR_INVALID_ARG, "status is NULL");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int32_t v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status");
    *status = v;
    return FA_OK;
}

}  // extern "C"
