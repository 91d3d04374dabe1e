// select.cu -- exact top-k page selection per (sequence, kv-head).
//
// The fixed budget of the most relevant tokens ("Accelerating Long-Context
// Decoding ...", abstract) is taken as the k = floor(budget / 16) candidate
// pages with the highest Quest score ("Methodology"; "The Move": paged
// top-k).  Ties go to the lower logical page and the result is returned in
// ascending page order.
//
// One CTA per unit.  The fp32 scores are mapped to order-preserving uint32
// keys and held in shared memory.  The k-th largest key is found by an
// MSB-first radix select (8-bit digits): a block min/max first strips the
// bits that every key shares, so the first histogram already splits the
// occupied range; a pass ends the search early when the digit bin that
// holds the k-th key is taken whole.  A final pass over the keys in index
// order writes the selected pages with ballot-based compaction: every key
// above the threshold, plus the lowest-index keys equal to it.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSmemKeys = 40960;     // keys held in shared memory (160 KB)

__device__ __forceinline__ uint32_t block_reduce_min_max(uint32_t v_min, uint32_t v_max,
                                                         uint32_t* red, bool want_max) {
    // two-stage: warp redux, then warp 0 over the per-warp results
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t v = want_max ? __reduce_max_sync(0xffffffffu, v_max)
                          : __reduce_min_sync(0xffffffffu, v_min);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t r = red[0];
    for (int w = 1; w < kSelWarps; ++w) r = want_max ? max(r, red[w]) : min(r, red[w]);
    __syncthreads();
    return r;
}

template <bool kSmemKeys>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectParams p) {
    extern __shared__ __align__(16) uint32_t skeys[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t red[kSelWarps];
    __shared__ uint32_t warp_gt[kSelWarps], warp_eq[kSelWarps];
    __shared__ uint32_t s_digit, s_gt, s_cnt;

    const int u = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hkv = p.s.Hkv, MP = p.s.MP;
    const int b = u / Hkv;
    int L = p.seq_lens[b];
    if (L < 0 || L > MP * kPage) L = 0;       // flagged by the scoring kernel
    const SeqGeom sg = seq_geom(L, p.prefix, p.window);
    const int n = sg.c_hi - sg.c_lo;
    const int kk = p.k_pages < n ? p.k_pages : n;
    int32_t* out = p.sel + (size_t)u * p.s.max_sel;
    // scores (and the previous readers of sel) belong to earlier kernels
    pdl_wait();
    pdl_launch_dependents();

    if (kk == n) {                              // every candidate fits the budget
        for (int i = tid; i < n; i += kSelThreads) out[i] = sg.c_lo + i;
        if (tid == 0) p.n_sel[u] = n;
        return;
    }
    if (kk == 0) {
        if (tid == 0) p.n_sel[u] = 0;
        return;
    }

    // keys: shared memory when they fit, else in place over the fp32 scores;
    // eight independent loads per thread are in flight before any key is stored
    const float* sc = p.scores_ws + (size_t)u * MP + sg.c_lo;
    uint32_t* keys = kSmemKeys ? skeys : reinterpret_cast<uint32_t*>(
                                             p.scores_ws + (size_t)u * MP + sg.c_lo);
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int base = 0; base < n; base += 8 * kSelThreads) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + j * kSelThreads + tid;
            v[j] = i < n ? __ldcg(sc + i) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + j * kSelThreads + tid;
            if (i < n) {
                const uint32_t k = order_key(v[j]);
                keys[i] = k;
                kmin = min(kmin, k);
                kmax = max(kmax, k);
            }
        }
    }
    kmin = block_reduce_min_max(kmin, kmax, red, false);   // syncs also publish keys[]
    kmax = block_reduce_min_max(kmin, kmax, red, true);

    uint32_t pmask = 0, pval = 0;       // resolved high bits of the k-th key
    uint32_t remaining = (uint32_t)kk;  // still to take among keys matching pval
    bool take_all = false;
    if (kmin == kmax) {
        pmask = 0xffffffffu;
        pval = kmax;
    } else {
        int hb = 31 - __clz(kmin ^ kmax);          // highest bit where keys differ
        pmask = hb >= 31 ? 0u : (0xffffffffu << (hb + 1));
        pval = kmax & pmask;
        for (;;) {
            const int lo_bit = hb - 7 > 0 ? hb - 7 : 0;
            const int width = hb - lo_bit + 1;
            const uint32_t dmask = (1u << width) - 1u;
            if (tid < 256) hist[tid] = 0;
            __syncthreads();
            for (int i = tid; i < n; i += kSelThreads) {
                const uint32_t k = keys[i];
                if ((k & pmask) == pval) atomicAdd(&hist[(k >> lo_bit) & dmask], 1u);
            }
            __syncthreads();
            // bins in descending digit order (position i <-> digit 255 - i),
            // inclusive scan by warps 0..7
            uint32_t v = 0, incl = 0;
            if (tid < 256) {
                v = hist[255 - tid];
                incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (lane == 31) red[warp] = incl;
            }
            __syncthreads();
            if (tid < 256) {
                uint32_t base = 0;
                for (int w = 0; w < warp; ++w) base += red[w];
                const uint32_t ge = incl + base;   // keys with digit >= 255 - tid
                const uint32_t gt = ge - v;        // keys with digit >  255 - tid
                if (gt < remaining && remaining <= ge) {   // exactly one bin qualifies
                    s_digit = 255 - tid;
                    s_gt = gt;
                    s_cnt = v;
                }
            }
            __syncthreads();
            const uint32_t d = s_digit, gt = s_gt, cnt = s_cnt;
            remaining -= gt;
            pval |= d << lo_bit;
            pmask |= dmask << lo_bit;
            if (cnt == remaining) {
                take_all = true;
                break;
            }
            if (lo_bit == 0) break;
            hb = lo_bit - 1;
            __syncthreads();
        }
    }

    // ---- index-ordered compaction: warp w owns keys [w * span, (w + 1) * span)
    const int span = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;
    const int lo = warp * span;
    const int hi = lo + span < n ? lo + span : n;
    uint32_t cgt = 0, ceq = 0;
    for (int i0 = lo; i0 < hi; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < hi ? (keys[i] & pmask) : 0u;
        const bool in = i < hi;
        cgt += __popc(__ballot_sync(0xffffffffu, in && k > pval));
        ceq += __popc(__ballot_sync(0xffffffffu, in && k == pval));
    }
    if (lane == 0) {
        warp_gt[warp] = cgt;
        warp_eq[warp] = ceq;
    }
    __syncthreads();
    uint32_t gt_base = 0, eq_base = 0;
    for (int w = 0; w < warp; ++w) {
        gt_base += warp_gt[w];
        eq_base += warp_eq[w];
    }
    const uint32_t eq_take = take_all ? 0xffffffffu : remaining;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int i0 = lo; i0 < hi; i0 += 32) {
        const int i = i0 + lane;
        const bool in = i < hi;
        const uint32_t k = in ? (keys[i] & pmask) : 0u;
        const bool is_gt = in && k > pval, is_eq = in && k == pval;
        const uint32_t bgt = __ballot_sync(0xffffffffu, is_gt);
        const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t eq_before = eq_base + __popc(beq & lt_mask);
        const uint32_t gt_before = gt_base + __popc(bgt & lt_mask);
        if (is_gt || (is_eq && eq_before < eq_take)) {
            const uint32_t pos = gt_before + (eq_before < eq_take ? eq_before : eq_take);
            if (pos < (uint32_t)kk) out[pos] = sg.c_lo + i;
        }
        gt_base += __popc(bgt);
        eq_base += __popc(beq);
    }
    if (tid == 0) p.n_sel[u] = kk;
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t st) {
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    const int smem = kSmemKeys * 4;
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    const int units = p.s.B * p.s.Hkv;
    if (units == 0) return cudaSuccess;
    // only as much shared memory as the longest candidate list needs; longer
    // lists keep their keys in place of the scores in global memory
    if (p.s.MP <= kSmemKeys) {
        return launch_pdl(select_kernel<true>, dim3(units), dim3(kSelThreads),
                          (size_t)p.s.MP * 4, st, p);
    }
    return launch_pdl(select_kernel<false>, dim3(units), dim3(kSelThreads), 0, st, p);
}

}  // namespace csa
