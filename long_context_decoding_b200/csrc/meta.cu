// meta.cu -- token append and page-metadata maintenance.
//
// The KV cache stays full size ("Why It Matters", roboaidigest post), and
// the Quest-style selection ("Methodology", arxivlens analysis) scores a page
// from its per-channel key minimum and maximum.  This kernel writes the new
// tokens into their page slots and brings the min/max of every touched page
// up to date: from the new keys alone when the page starts inside the new
// tokens, else by folding the new keys into the stored min/max (exact, since
// min and max of bf16 values are bf16 values).  In rebuild mode (no new
// tokens) it recomputes the touched pages' min/max from the cache.
//
// One CTA per (sequence, kv-head, touched page), D/2 threads, each owning a
// bf16x2 channel pair: every global access is a coalesced 4-byte word per
// thread.  The work is tiny (a few KB per layer per step); it is a latency
// kernel, not a bandwidth one.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

struct Pair {
    uint32_t lo, hi;   // bf16x2 minimum / maximum, channel 2c in bits 0..15
};

__device__ __forceinline__ uint32_t sel_half(uint32_t cur, uint32_t v, int half, bool take) {
    const uint32_t m = half ? 0xffff0000u : 0x0000ffffu;
    return take ? ((cur & ~m) | (v & m)) : cur;
}

// Fold key word v into the running min/max (strict comparisons: on equal
// values the earlier token's bits stay).
__device__ __forceinline__ void fold(Pair& p, uint32_t v) {
    const float v0 = bf16_lo(v), v1 = bf16_hi(v);
    p.lo = sel_half(p.lo, v, 0, v0 < bf16_lo(p.lo));
    p.lo = sel_half(p.lo, v, 1, v1 < bf16_hi(p.lo));
    p.hi = sel_half(p.hi, v, 0, v0 > bf16_lo(p.hi));
    p.hi = sel_half(p.hi, v, 1, v1 > bf16_hi(p.hi));
}

// Append the new tokens of logical page `page` and refresh its min/max.
// phys is the page's physical id (page_table[b][page]).
__device__ void update_page(const MetaParams& p, int b, int g, int c, int L, int start, int page,
                            int phys) {
    const int Hkv = p.s.Hkv, D = p.s.D;
    const bool append = p.new_k != nullptr;
    const int t0 = page * kPage;
    const int t_end = t0 + kPage < L ? t0 + kPage : L;
    if (phys < 0 || phys >= p.s.NPG) {
        if (c == 0) latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
        return;
    }
    const int W = D / 2;                                    // words per key row
    const size_t tile = ((size_t)phys * Hkv + g) * kPage * W;
    uint32_t* kc = reinterpret_cast<uint32_t*>(p.k_cache) + tile;
    uint32_t* vc = reinterpret_cast<uint32_t*>(p.v_cache) + tile;
    uint32_t* mt = reinterpret_cast<uint32_t*>(p.meta) + ((size_t)phys * Hkv + g) * 2 * W;
    const int first_new = t0 > start ? t0 : start;

    Pair acc;
    bool have = false;
    if (append) {
        const uint32_t* nk = reinterpret_cast<const uint32_t*>(p.new_k);
        const uint32_t* nv = reinterpret_cast<const uint32_t*>(p.new_v);
        if (first_new > t0) {                 // older tokens: stored min/max
            acc.lo = mt[c];
            acc.hi = mt[W + c];
            have = true;
        }
        for (int t = first_new; t < t_end; ++t) {
            const size_t src = (((size_t)b * p.n_new + (t - start)) * Hkv + g) * W + c;
            const uint32_t kw = nk[src];
            kc[(size_t)(t - t0) * W + c] = kw;
            vc[(size_t)(t - t0) * W + c] = nv[src];
            if (have) {
                fold(acc, kw);
            } else {
                acc.lo = acc.hi = kw;
                have = true;
            }
        }
    } else {
        for (int t = t0; t < t_end; ++t) {
            const uint32_t kw = kc[(size_t)(t - t0) * W + c];
            if (have) {
                fold(acc, kw);
            } else {
                acc.lo = acc.hi = kw;
                have = true;
            }
        }
    }
    mt[c] = acc.lo;
    mt[W + c] = acc.hi;
}

__global__ void meta_update_kernel(MetaParams p) {
    const int u = blockIdx.x;
    const int Hkv = p.s.Hkv, D = p.s.D, MP = p.s.MP;
    const int b = u / Hkv, g = u % Hkv;
    const int c = threadIdx.x;                  // channel pair
    // seq_lens and page_table are caller inputs, read before the dependency
    // wait; the cache, the metadata and the new tokens only after it
    const int L = p.seq_lens[b];
    const bool append = p.new_k != nullptr;
    const bool bad_len = L < 0 || L > MP * kPage || (append && L < p.n_new);
    const int start = bad_len ? 0 : (L - p.n_new > 0 ? L - p.n_new : 0);   // first new token
    const int n_touched = bad_len || L == 0 ? 0 : (L - 1) / kPage - start / kPage + 1;
    const int j0 = (int)blockIdx.y;
    const int phys0 = j0 < n_touched ? p.page_table[(size_t)b * MP + start / kPage + j0] : -1;
    pdl_wait();
    pdl_launch_dependents();
    if (bad_len) {
        if (c == 0 && blockIdx.y == 0) latch_flag(p.flags, CSA_DEVFLAG_BAD_SEQ_LEN);
        return;
    }
    if (c >= D / 2) return;
    for (int j = j0; j < n_touched; j += (int)gridDim.y) {
        const int page = start / kPage + j;
        const int phys = j == j0 ? phys0 : p.page_table[(size_t)b * MP + page];
        update_page(p, b, g, c, L, start, page, phys);
    }
}

}  // namespace

cudaError_t launch_meta_update(const MetaParams& p, cudaStream_t st) {
    const int units = p.s.B * p.s.Hkv;
    int pages = (p.n_new + kPage - 1) / kPage + 1;          // pages one chunk can touch
    if (pages > p.s.MP) pages = p.s.MP;
    if (pages > 65535) pages = 65535;                       // grid.y limit; the kernel strides
    if (units == 0 || pages <= 0) return cudaSuccess;
    dim3 grid(units, pages);
    return launch_pdl(meta_update_kernel, grid, dim3(p.s.D / 2), 0, st, p);
}

}  // namespace csa
