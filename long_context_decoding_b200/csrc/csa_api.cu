// csa_api.cu -- the C ABI of libcsa.so (declared in include/csa.h).
//
// Host-side only: argument validation, the workspace layout, the per-stream
// record of the last call and kernel dispatch.  No device memory is
// allocated here; every buffer belongs to the caller.
#include <math.h>
#include <mutex>
#include <stdio.h>
#include <string.h>
#include <unordered_map>

#include "common.cuh"
#include "internal.h"

namespace csa {

int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 148;
    }
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Last kernel-launching call per stream handle.  Forgetting an entry is
// always safe (the decode then waits before it reads anything), so the table
// is simply cleared when it grows large.
static std::mutex g_calls_mu;
static std::unordered_map<const void*, CallKind> g_calls;

void note_stream_call(const void* stream, CallKind kind) {
    std::lock_guard<std::mutex> lock(g_calls_mu);
    if (g_calls.size() > 4096) g_calls.clear();
    g_calls[stream] = kind;
}

CallKind last_stream_call(const void* stream) {
    std::lock_guard<std::mutex> lock(g_calls_mu);
    auto it = g_calls.find(stream);
    return it == g_calls.end() ? kCallOther : it->second;
}

WsLayout workspace_layout(const Shape& s) {
    WsLayout w;
    const size_t units = (size_t)s.B * s.Hkv;
    size_t off = 0;
    w.flags = off;
    off = align_up(off + 4, 256);
    w.rec_range = off;
    off = align_up(off + 16 * units, 256);
    w.keyrange = off;
    off = align_up(off + 8 * units, 256);
    w.scores = off;
    off = align_up(off + 4 * units * (size_t)s.MP, 256);
    w.partials = off;
    // record slots per phase: a decode CTA or a prefix/window CTA of the fused
    // kernel per slot plus one per unit, or the 8 CTAs of each unit's cluster
    size_t slots = (size_t)decode_grid(s) + units;
    const size_t fused = (size_t)fused_phase0_ctas(s) + units;
    if (fused > slots) slots = fused;
    if (8 * units > slots) slots = 8 * units;
    w.dec_slots = slots;
    off = align_up(off + 2 * 4 * w.dec_slots * decode_record_floats(s), 256);
    w.total = off;
    return w;
}

// ---------------------------------------------------------------- validation
static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_dims(const csa_dims* d, Shape* s) {
    if (!d) return CSA_ERR_INVALID_ARG;
    if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->D < 1 || d->max_pages_per_seq < 1 ||
        d->num_pages < 1 || d->max_sel < 1)
        return CSA_ERR_INVALID_ARG;
    if (d->Hq % d->Hkv != 0) return CSA_ERR_INVALID_ARG;
    if (d->page_size != kPage) return CSA_ERR_UNSUPPORTED;
    if (d->D != 64 && d->D != 128 && d->D != 256) return CSA_ERR_UNSUPPORTED;
    const int G = d->Hq / d->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return CSA_ERR_UNSUPPORTED;
    if ((long long)d->B * d->Hkv > kMaxUnits) return CSA_ERR_UNSUPPORTED;
    if ((long long)d->num_pages * d->Hkv * kPage >= (1ll << 31)) return CSA_ERR_UNSUPPORTED;
    if ((long long)d->max_pages_per_seq * kPage >= (1ll << 31)) return CSA_ERR_UNSUPPORTED;
    if ((long long)d->B * d->Hkv * (d->max_pages_per_seq + 2) >= (1ll << 31))
        return CSA_ERR_UNSUPPORTED;   // flattened page lists are indexed with int
    s->B = d->B;
    s->Hq = d->Hq;
    s->Hkv = d->Hkv;
    s->G = G;
    s->D = d->D;
    s->MP = d->max_pages_per_seq;
    s->NPG = d->num_pages;
    s->max_sel = d->max_sel;
    return CSA_OK;
}

#define CSA_REQUIRE(ptr)                                  \
    do {                                                  \
        if (!(ptr) || !aligned16(ptr)) return CSA_ERR_INVALID_ARG; \
    } while (0)
#define CSA_OPTIONAL(ptr)                                 \
    do {                                                  \
        if ((ptr) && !aligned16(ptr)) return CSA_ERR_INVALID_ARG; \
    } while (0)

static int check_ws(const Shape& s, void* ws, size_t bytes, WsLayout* w) {
    if (!ws || !aligned16(ws)) return CSA_ERR_WORKSPACE;
    *w = workspace_layout(s);
    if (bytes < w->total) return CSA_ERR_WORKSPACE;
    return CSA_OK;
}

static int launch_status(cudaError_t e) {
    if (e == cudaSuccess) return CSA_OK;
    cudaGetLastError();
    return CSA_ERR_CUDA;
}

template <typename T>
static T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace csa

using namespace csa;

extern "C" {

int csa_version(void) { return 102; }

const char* csa_status_string(int st) {
    switch (st) {
        case CSA_OK: return "ok";
        case CSA_ERR_INVALID_ARG: return "invalid argument";
        case CSA_ERR_UNSUPPORTED: return "unsupported shape";
        case CSA_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA_ERR_CUDA: return "CUDA error";
        case CSA_ERR_DEVICE_FLAG: return "device-side error flag set";
        default: return "unknown status";
    }
}

size_t csa_workspace_size(const csa_dims* d) {
    Shape s;
    if (check_dims(d, &s) != CSA_OK) return 0;
    return workspace_layout(s).total;
}

int csa_workspace_init(void* workspace, size_t bytes, void* stream) {
    if (!workspace || !aligned16(workspace)) return CSA_ERR_WORKSPACE;
    return launch_status(cudaMemsetAsync(workspace, 0, bytes, (cudaStream_t)stream));
}

static int meta_update_common(const csa_dims* d, void* k_cache, void* v_cache, void* meta,
                              void* meta8, const int32_t* page_table, const int32_t* seq_lens,
                              const void* new_k, const void* new_v, int n_new, void* workspace,
                              size_t workspace_bytes, void* stream) {
    Shape s;
    int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    CSA_REQUIRE(meta);
    CSA_REQUIRE(page_table);
    CSA_REQUIRE(seq_lens);
    CSA_REQUIRE(k_cache);
    if (n_new < 1) return CSA_ERR_INVALID_ARG;
    if ((new_k == nullptr) != (new_v == nullptr)) return CSA_ERR_INVALID_ARG;
    if (new_k) {
        CSA_REQUIRE(v_cache);
        CSA_REQUIRE(new_k);
        CSA_REQUIRE(new_v);
        if ((long long)n_new > (long long)s.MP * kPage) return CSA_ERR_INVALID_ARG;
    }
    WsLayout w;
    rc = check_ws(s, workspace, workspace_bytes, &w);
    if (rc != CSA_OK) return rc;
    MetaParams p;
    p.k_cache = static_cast<uint16_t*>(k_cache);
    p.v_cache = static_cast<uint16_t*>(v_cache);
    p.meta = static_cast<uint16_t*>(meta);
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.new_k = static_cast<const uint16_t*>(new_k);
    p.new_v = static_cast<const uint16_t*>(new_v);
    p.meta8 = static_cast<uint8_t*>(meta8);
    p.n_new = n_new;
    p.flags = at<uint32_t>(workspace, w.flags);
    p.s = s;
    note_stream_call(stream, kCallOther);
    return launch_status(launch_meta_update(p, (cudaStream_t)stream));
}

static int score_select_common(const csa_dims* d, const void* q, const void* meta,
                               const void* meta8, const int32_t* page_table,
                               const int32_t* seq_lens, int prefix, int window, int budget_tokens,
                               int32_t* sel_pages, int32_t* n_sel, float* scores_out,
                               void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    CSA_REQUIRE(q);
    if (meta8) {
        CSA_REQUIRE(meta8);
    } else {
        CSA_REQUIRE(meta);
    }
    CSA_REQUIRE(page_table);
    CSA_REQUIRE(seq_lens);
    CSA_REQUIRE(sel_pages);
    CSA_REQUIRE(n_sel);
    CSA_OPTIONAL(scores_out);
    if (prefix < 0 || window < 0 || budget_tokens < 0) return CSA_ERR_INVALID_ARG;
    const int k_pages = budget_tokens / kPage;
    if (k_pages > s.max_sel) return CSA_ERR_INVALID_ARG;
    WsLayout w;
    rc = check_ws(s, workspace, workspace_bytes, &w);
    if (rc != CSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    ScoreParams sp;
    sp.q = static_cast<const uint16_t*>(q);
    sp.meta = static_cast<const uint16_t*>(meta);
    sp.page_table = page_table;
    sp.seq_lens = seq_lens;
    sp.prefix = prefix;
    sp.window = window;
    sp.scores_ws = at<float>(workspace, w.scores);
    sp.scores_out = scores_out;
    sp.meta8 = static_cast<const uint8_t*>(meta8);
    sp.keyrange = at<uint2>(workspace, w.keyrange);
    sp.flags = at<uint32_t>(workspace, w.flags);
    sp.s = s;
    // scores are needed only where a unit has more candidates than it keeps
    const long long n_max = (long long)s.MP - prefix / kPage - window / kPage;
    if ((k_pages > 0 && k_pages < n_max) || scores_out) {
        rc = launch_status(launch_score(sp, st));
        if (rc != CSA_OK) {
            note_stream_call(stream, kCallOther);
            return rc;
        }
    }
    SelectParams lp;
    lp.scores_ws = sp.scores_ws;
    lp.seq_lens = seq_lens;
    lp.prefix = prefix;
    lp.window = window;
    lp.k_pages = k_pages;
    lp.sel = sel_pages;
    lp.n_sel = n_sel;
    lp.keyrange = sp.keyrange;
    lp.flags = sp.flags;
    lp.smem_keys = 0;
    lp.s = s;
    rc = launch_status(launch_select(lp, st));
    note_stream_call(stream, rc == CSA_OK ? kCallScoreSelect : kCallOther);
    return rc;
}

static int decode_common(const csa_dims* d, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* page_table, const int32_t* seq_lens,
                         const int32_t* sel_pages, const int32_t* n_sel, int prefix, int window,
                         int dense, float scale, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
    Shape s;
    int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    CSA_REQUIRE(q);
    CSA_REQUIRE(k_cache);
    CSA_REQUIRE(v_cache);
    CSA_REQUIRE(page_table);
    CSA_REQUIRE(seq_lens);
    CSA_REQUIRE(out);
    CSA_OPTIONAL(lse);
    if (!dense) {
        CSA_REQUIRE(sel_pages);
        CSA_REQUIRE(n_sel);
        if (prefix < 0 || window < 0) return CSA_ERR_INVALID_ARG;
    }
    if (!(scale == scale) || isinf(scale)) return CSA_ERR_INVALID_ARG;
    WsLayout w;
    rc = check_ws(s, workspace, workspace_bytes, &w);
    if (rc != CSA_OK) return rc;
    DecodeParams p;
    p.q = static_cast<const uint16_t*>(q);
    p.k_cache = static_cast<const uint16_t*>(k_cache);
    p.v_cache = static_cast<const uint16_t*>(v_cache);
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.sel = sel_pages;
    p.n_sel = n_sel;
    p.prefix = prefix;
    p.window = window;
    p.dense = dense;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)s.D);
    p.scale_log2 = sc * 1.4426950408889634f;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.flags = at<uint32_t>(workspace, w.flags);
    p.rec_range = at<int4>(workspace, w.rec_range);
    p.partials = at<float>(workspace, w.partials);
    p.phase_floats = w.dec_slots * decode_record_floats(s);
    p.early = last_stream_call(stream) == kCallScoreSelect ? 1 : 0;
    p.s = s;
    note_stream_call(stream, kCallOther);
    return launch_status(launch_decode(p, (cudaStream_t)stream));
}

int csa_decode(const csa_dims* d, const void* q, const void* k_cache, const void* v_cache,
               const int32_t* page_table, const int32_t* seq_lens, const int32_t* sel_pages,
               const int32_t* n_sel, int prefix, int window, float scale, void* out, float* lse,
               void* workspace, size_t workspace_bytes, void* stream) {
    return decode_common(d, q, k_cache, v_cache, page_table, seq_lens, sel_pages, n_sel, prefix,
                         window, 0, scale, out, lse, workspace, workspace_bytes, stream);
}

int csa_decode_full(const csa_dims* d, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* page_table, const int32_t* seq_lens, float scale, void* out,
                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    return decode_common(d, q, k_cache, v_cache, page_table, seq_lens, nullptr, nullptr, 0, 0, 1,
                         scale, out, lse, workspace, workspace_bytes, stream);
}

static int sparse_attention_common(const csa_dims* d, const void* q, const void* k_cache,
                                   const void* v_cache, const void* meta, const void* meta8,
                                   const int32_t* page_table, const int32_t* seq_lens, int prefix,
                                   int window, int budget_tokens, float scale,
                                   int32_t* sel_pages, int32_t* n_sel, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    CSA_REQUIRE(q);
    CSA_REQUIRE(k_cache);
    CSA_REQUIRE(v_cache);
    if (meta8) {
        CSA_REQUIRE(meta8);
    } else {
        CSA_REQUIRE(meta);
    }
    CSA_REQUIRE(page_table);
    CSA_REQUIRE(seq_lens);
    CSA_REQUIRE(sel_pages);
    CSA_REQUIRE(n_sel);
    CSA_REQUIRE(out);
    CSA_OPTIONAL(lse);
    if (prefix < 0 || window < 0 || budget_tokens < 0) return CSA_ERR_INVALID_ARG;
    const int k_pages = budget_tokens / kPage;
    if (k_pages > s.max_sel) return CSA_ERR_INVALID_ARG;
    if (!(scale == scale) || isinf(scale)) return CSA_ERR_INVALID_ARG;
    WsLayout w;
    rc = check_ws(s, workspace, workspace_bytes, &w);
    if (rc != CSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    note_stream_call(stream, kCallOther);
    const long long n_max = (long long)s.MP - prefix / kPage - window / kPage;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)s.D);

    ScoreParams sp;
    sp.q = static_cast<const uint16_t*>(q);
    sp.meta = static_cast<const uint16_t*>(meta);
    sp.page_table = page_table;
    sp.seq_lens = seq_lens;
    sp.prefix = prefix;
    sp.window = window;
    sp.scores_ws = at<float>(workspace, w.scores);
    sp.scores_out = nullptr;
    sp.meta8 = static_cast<const uint8_t*>(meta8);
    sp.keyrange = at<uint2>(workspace, w.keyrange);
    sp.flags = at<uint32_t>(workspace, w.flags);
    sp.s = s;
    if (k_pages > 0 && k_pages < n_max) {      // else every unit keeps all its candidates
        rc = launch_status(launch_score(sp, st));
        if (rc != CSA_OK) return rc;
    }

    DecodeParams dp;
    dp.q = sp.q;
    dp.k_cache = static_cast<const uint16_t*>(k_cache);
    dp.v_cache = static_cast<const uint16_t*>(v_cache);
    dp.page_table = page_table;
    dp.seq_lens = seq_lens;
    dp.sel = sel_pages;
    dp.n_sel = n_sel;
    dp.prefix = prefix;
    dp.window = window;
    dp.dense = 0;
    dp.scale_log2 = sc * 1.4426950408889634f;
    dp.out = static_cast<uint16_t*>(out);
    dp.lse = lse;
    dp.flags = sp.flags;
    dp.rec_range = at<int4>(workspace, w.rec_range);
    dp.partials = at<float>(workspace, w.partials);
    dp.phase_floats = w.dec_slots * decode_record_floats(s);
    dp.s = s;

    // A budget that keeps every candidate of every unit attends to every
    // token: the selection still reports all candidates, and the decode is
    // the dense one (its work split suits a full sequence).
    if (k_pages >= n_max) dp.dense = 1;
    if (!dp.dense && fused_eligible(s, prefix, window, k_pages)) {
        FusedParams fp;
        fp.d = dp;
        fp.d.early = 1;
        fp.scores_ws = sp.scores_ws;
        fp.k_pages = k_pages;
        fp.sel = sel_pages;
        fp.n_sel = n_sel;
        fp.keyrange = sp.keyrange;
        fp.n0 = fused_phase0_ctas(s, prefix, window);
        return launch_status(launch_fused(fp, st));
    }
    SelectParams lp;
    lp.scores_ws = sp.scores_ws;
    lp.seq_lens = seq_lens;
    lp.prefix = prefix;
    lp.window = window;
    lp.k_pages = k_pages;
    lp.sel = sel_pages;
    lp.n_sel = n_sel;
    lp.keyrange = sp.keyrange;
    lp.flags = sp.flags;
    lp.smem_keys = 0;
    lp.s = s;
    rc = launch_status(launch_select(lp, st));
    if (rc != CSA_OK) return rc;
    dp.early = 1;   // our own scoring and selection kernels are the ones ahead
    return launch_status(launch_decode(dp, st));
}

int csa_meta_update(const csa_dims* d, void* k_cache, void* v_cache, void* meta,
                    const int32_t* page_table, const int32_t* seq_lens, const void* new_k,
                    const void* new_v, int n_new, void* workspace, size_t workspace_bytes,
                    void* stream) {
    return meta_update_common(d, k_cache, v_cache, meta, nullptr, page_table, seq_lens, new_k,
                              new_v, n_new, workspace, workspace_bytes, stream);
}

int csa_meta_update_fp8(const csa_dims* d, void* k_cache, void* v_cache, void* meta,
                        void* meta8, const int32_t* page_table, const int32_t* seq_lens,
                        const void* new_k, const void* new_v, int n_new, void* workspace,
                        size_t workspace_bytes, void* stream) {
    CSA_REQUIRE(meta8);
    return meta_update_common(d, k_cache, v_cache, meta, meta8, page_table, seq_lens, new_k,
                              new_v, n_new, workspace, workspace_bytes, stream);
}

int csa_score_select(const csa_dims* d, const void* q, const void* meta,
                     const int32_t* page_table, const int32_t* seq_lens, int prefix, int window,
                     int budget_tokens, int32_t* sel_pages, int32_t* n_sel, float* scores_out,
                     void* workspace, size_t workspace_bytes, void* stream) {
    return score_select_common(d, q, meta, nullptr, page_table, seq_lens, prefix, window,
                               budget_tokens, sel_pages, n_sel, scores_out, workspace,
                               workspace_bytes, stream);
}

int csa_score_select_fp8(const csa_dims* d, const void* q, const void* meta8,
                         const int32_t* page_table, const int32_t* seq_lens, int prefix,
                         int window, int budget_tokens, int32_t* sel_pages, int32_t* n_sel,
                         float* scores_out, void* workspace, size_t workspace_bytes,
                         void* stream) {
    CSA_REQUIRE(meta8);
    return score_select_common(d, q, nullptr, meta8, page_table, seq_lens, prefix, window,
                               budget_tokens, sel_pages, n_sel, scores_out, workspace,
                               workspace_bytes, stream);
}

int csa_sparse_attention(const csa_dims* d, const void* q, const void* k_cache,
                         const void* v_cache, const void* meta, const int32_t* page_table,
                         const int32_t* seq_lens, int prefix, int window, int budget_tokens,
                         float scale, int32_t* sel_pages, int32_t* n_sel, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, void* stream) {
    return sparse_attention_common(d, q, k_cache, v_cache, meta, nullptr, page_table, seq_lens,
                                   prefix, window, budget_tokens, scale, sel_pages, n_sel, out,
                                   lse, workspace, workspace_bytes, stream);
}

int csa_sparse_attention_fp8(const csa_dims* d, const void* q, const void* k_cache,
                             const void* v_cache, const void* meta8, const int32_t* page_table,
                             const int32_t* seq_lens, int prefix, int window, int budget_tokens,
                             float scale, int32_t* sel_pages, int32_t* n_sel, void* out,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    CSA_REQUIRE(meta8);
    return sparse_attention_common(d, q, k_cache, v_cache, nullptr, meta8, page_table, seq_lens,
                                   prefix, window, budget_tokens, scale, sel_pages, n_sel, out,
                                   lse, workspace, workspace_bytes, stream);
}

int csa_select_scores(const csa_dims* d, const float* scores, const int32_t* seq_lens,
                      int prefix, int window, int budget_tokens, int32_t* sel_pages,
                      int32_t* n_sel, void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    CSA_REQUIRE(scores);
    CSA_REQUIRE(seq_lens);
    CSA_REQUIRE(sel_pages);
    CSA_REQUIRE(n_sel);
    if (prefix < 0 || window < 0 || budget_tokens < 0) return CSA_ERR_INVALID_ARG;
    const int k_pages = budget_tokens / kPage;
    if (k_pages > s.max_sel) return CSA_ERR_INVALID_ARG;
    WsLayout w;
    rc = check_ws(s, workspace, workspace_bytes, &w);
    if (rc != CSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    note_stream_call(stream, kCallOther);
    // the selection rewrites its scores in place: it works on a copy
    float* ws_scores = at<float>(workspace, w.scores);
    const size_t bytes = sizeof(float) * (size_t)s.B * s.Hkv * s.MP;
    if (cudaMemcpyAsync(ws_scores, scores, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return launch_status(cudaGetLastError());
    SelectParams lp;
    lp.scores_ws = ws_scores;
    lp.seq_lens = seq_lens;
    lp.prefix = prefix;
    lp.window = window;
    lp.k_pages = k_pages;
    lp.sel = sel_pages;
    lp.n_sel = n_sel;
    lp.keyrange = at<uint2>(workspace, w.keyrange);   // zero: the full key range
    lp.flags = at<uint32_t>(workspace, w.flags);
    lp.smem_keys = 0;
    lp.s = s;
    rc = launch_status(launch_select(lp, st));
    // the selection kernel lets the next grid start before it writes sel: a
    // decode that follows reads the selection only after its wait
    note_stream_call(stream, rc == CSA_OK ? kCallScoreSelect : kCallOther);
    return rc;
}

int csa_shard_selection(const csa_dims* d, const int32_t* sel_pages, const int32_t* n_sel,
                        int page_lo, int page_hi, int max_sel_local, int32_t* sel_local,
                        int32_t* n_sel_local, void* stream) {
    Shape s;
    int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    CSA_REQUIRE(sel_pages);
    CSA_REQUIRE(n_sel);
    CSA_REQUIRE(sel_local);
    CSA_REQUIRE(n_sel_local);
    if (page_lo < 0 || page_hi < page_lo || max_sel_local < s.max_sel) return CSA_ERR_INVALID_ARG;
    note_stream_call(stream, kCallOther);
    return launch_status(launch_shard_selection(s, sel_pages, n_sel, page_lo, page_hi,
                                                max_sel_local, sel_local, n_sel_local,
                                                (cudaStream_t)stream));
}

int csa_merge_attention(int parts, int batch, int q_heads, int head_dim, const void* out_parts,
                        const float* lse_parts, void* out, float* lse, void* stream) {
    if (parts < 1 || parts > 64 || batch < 1 || q_heads < 1) return CSA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return CSA_ERR_INVALID_ARG;
    if ((long long)batch * q_heads > (1ll << 30)) return CSA_ERR_INVALID_ARG;
    CSA_REQUIRE(out_parts);
    CSA_REQUIRE(lse_parts);
    CSA_REQUIRE(out);
    CSA_OPTIONAL(lse);
    note_stream_call(stream, kCallOther);
    return launch_status(launch_merge(parts, batch * q_heads, head_dim, out_parts, lse_parts,
                                      out, lse, (cudaStream_t)stream));
}

int csa_get_device_status(void* workspace, void* stream, int* flags_out) {
    if (!workspace || !aligned16(workspace)) return CSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t flags = 0;
    if (cudaMemcpyAsync(&flags, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    if (flags_out) *flags_out = (int)flags;
    return flags ? CSA_ERR_DEVICE_FLAG : CSA_OK;
}

}  // extern "C"
