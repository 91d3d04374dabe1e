// select.cu -- exact top-k page selection per (sequence, kv-head).
//
// The fixed budget of the most relevant tokens ("Accelerating Long-Context
// Decoding ...", abstract) is taken as the k = floor(budget / 16) candidate
// pages with the highest Quest score ("Methodology"; "The Move": paged
// top-k).  Ties go to the lower logical page and the result is returned in
// ascending page order.
//
// Main path: a cluster of 8 CTAs per unit (256 threads each, 8 keys per
// thread in registers, up to 16384 candidates).  Every CTA keeps a local
// histogram; the histograms, the min/max and the compaction counts are
// merged in rank 0's shared memory through distributed shared memory, so a
// unit's selection is spread over eight SMs instead of one.
//
// Fallback (longer candidate lists): one CTA of 1024 threads per unit; the unit's fp32 scores become
// order-preserving uint32 keys.  When the candidate list fits (up to
// 1024 x 16 keys), warp w keeps the contiguous span [w * S, (w + 1) * S) of
// keys in registers, lane l holding keys w * S + 32 j + l (coalesced loads,
// no shared memory in the passes); longer lists keep their keys in shared
// memory (or, beyond that, in place over the scores).
//   1. block min/max strips the high bits that every key shares;
//   2. MSB-first radix select with 8-bit digits finds the k-th largest key
//      (a pass ends the search early when the digit bin holding the k-th key
//      is taken whole);
//   3. ballots in index order inside every warp span, plus one scan of the
//      per-warp (above, equal) counts, place every selected page: all keys
//      above the threshold plus the lowest-index keys equal to it, written
//      in index order.
#include "common.cuh"
#include "internal.h"
#include "select_core.cuh"

namespace csa {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kRegKeys = 16;                          // keys per thread in registers
constexpr int kRegCap = kSelThreads * kRegKeys;       // 16384 candidates
constexpr int kSmemKeys = 40960;                      // keys held in shared memory (160 KB)

struct SelShared {
    uint32_t hist[256];
    uint32_t red[kSelWarps];
    uint32_t wgt[kSelWarps], weq[kSelWarps];
    uint32_t digit, gt, cnt;
};

// Block-wide min and max of one value per thread (every warp reduces the
// per-warp results with one redux each; no serial loop).
__device__ __forceinline__ void block_min_max(uint32_t& kmin, uint32_t& kmax, SelShared& sh) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t wmin = __reduce_min_sync(0xffffffffu, kmin);
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        sh.red[warp] = wmin;
        sh.wgt[warp] = wmax;
    }
    __syncthreads();
    kmin = __reduce_min_sync(0xffffffffu, lane < kSelWarps ? sh.red[lane] : 0xffffffffu);
    kmax = __reduce_max_sync(0xffffffffu, lane < kSelWarps ? sh.wgt[lane] : 0u);
    __syncthreads();
}

// Digit d of the bin holding the `remaining`-th largest key; sets
// (d, keys in bins above d, keys in bin d).
__device__ __forceinline__ void find_digit(SelShared& sh, uint32_t remaining) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t v = 0, incl = 0;
    if (tid < 256) {                  // bins in descending digit order
        v = sh.hist[255 - tid];
        incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) sh.red[warp] = incl;
    }
    __syncthreads();
    if (tid < 256) {
        const uint32_t base = warp_prefix(sh.red, 8);
        const uint32_t ge = incl + base;   // keys with digit >= 255 - tid
        const uint32_t gtc = ge - v;       // keys with digit >  255 - tid
        if (gtc < remaining && remaining <= ge) {   // exactly one bin qualifies
            sh.digit = 255 - tid;
            sh.gt = gtc;
            sh.cnt = v;
        }
    }
    __syncthreads();
}

// Up to kRegCap candidates in registers (warp spans); longer lists keep their
// keys in shared memory (or in place over the scores).
__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(SelectParams p) {
    extern __shared__ __align__(16) uint32_t skeys[];
    __shared__ SelShared sh;

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
    if (tid == 0) p.keyrange[u] = make_uint2(0u, 0u);   // left by the scoring kernel, unused

    if (kk == n) {                              // every candidate fits the budget
        for (int i = tid; i < n; i += kSelThreads) out[i] = sg.c_lo + i;
        if (tid == 0) p.n_sel[u] = n;
        return;
    }
    if (kk == 0) {
        if (tid == 0) p.n_sel[u] = 0;
        return;
    }

    const float* sc = p.scores_ws + (size_t)u * MP + sg.c_lo;
    const bool kRegs = n <= kRegCap;
    uint32_t kr[kRegKeys];
    uint32_t* keys = n <= p.smem_keys ? skeys
                                      : reinterpret_cast<uint32_t*>(p.scores_ws + (size_t)u * MP +
                                                                    sg.c_lo);
    // register mode: warp w owns [w * span, (w + 1) * span), lane l the keys
    // w * span + 32 j + l
    const int span = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;
    const int wlo = warp * span;
    const int whi = wlo + span < n ? wlo + span : n;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    if (kRegs) {
        float v[kRegKeys];
#pragma unroll
        for (int j = 0; j < kRegKeys; ++j) {
            const int i = wlo + 32 * j + lane;
            v[j] = __ldcg(sc + (i < whi ? i : 0));
        }
#pragma unroll
        for (int j = 0; j < kRegKeys; ++j) {
            kr[j] = order_key(v[j]);
            if (wlo + 32 * j + lane < whi) {
                kmin = min(kmin, kr[j]);
                kmax = max(kmax, kr[j]);
            }
        }
    } else {
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
    }
    block_min_max(kmin, kmax, sh);     // its barriers also publish keys[]

    uint32_t pmask, pval;               // resolved high bits of the k-th key
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
            const uint32_t dmask = (1u << (hb - lo_bit + 1)) - 1u;
            if (tid < 256) sh.hist[tid] = 0;
            __syncthreads();
            if (kRegs) {
#pragma unroll
                for (int j = 0; j < kRegKeys; ++j)
                    if (wlo + 32 * j + lane < whi && (kr[j] & pmask) == pval)
                        atomicAdd(&sh.hist[(kr[j] >> lo_bit) & dmask], 1u);
            } else {
                for (int i = tid; i < n; i += kSelThreads) {
                    const uint32_t k = keys[i];
                    if ((k & pmask) == pval) atomicAdd(&sh.hist[(k >> lo_bit) & dmask], 1u);
                }
            }
            __syncthreads();
            find_digit(sh, remaining);
            const uint32_t d = sh.digit, gt = sh.gt, cnt = sh.cnt;
            remaining -= gt;
            pval |= d << lo_bit;
            pmask |= dmask << lo_bit;
            if (cnt == remaining) {
                take_all = true;
                break;
            }
            if (lo_bit == 0) break;
            hb = lo_bit - 1;
        }
    }
    const uint32_t eq_take = take_all ? 0xffffffffu : remaining;

    if (kRegs) {
        // ballot compaction in index order inside the warp span
        uint32_t cgt = 0, ceq = 0;
#pragma unroll
        for (int j = 0; j < kRegKeys; ++j) {
            const bool in = wlo + 32 * j + lane < whi;
            const uint32_t k = kr[j] & pmask;
            cgt += __popc(__ballot_sync(0xffffffffu, in && k > pval));
            ceq += __popc(__ballot_sync(0xffffffffu, in && k == pval));
        }
        if (lane == 0) {
            sh.wgt[warp] = cgt;
            sh.weq[warp] = ceq;
        }
        __syncthreads();
        uint32_t gt_base = warp_prefix(sh.wgt, kSelWarps);
        uint32_t eq_base = warp_prefix(sh.weq, kSelWarps);
        const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
        for (int j = 0; j < kRegKeys; ++j) {
            const int i = wlo + 32 * j + lane;
            const bool in = i < whi;
            const uint32_t k = kr[j] & pmask;
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
    } else {
        // warp w owns keys [w * span, (w + 1) * span): ballot compaction
        const int lo = wlo;
        const int hi = whi;
        uint32_t cgt = 0, ceq = 0;
        for (int i0 = lo; i0 < hi; i0 += 32) {
            const int i = i0 + lane;
            const bool in = i < hi;
            const uint32_t k = in ? (keys[i] & pmask) : 0u;
            cgt += __popc(__ballot_sync(0xffffffffu, in && k > pval));
            ceq += __popc(__ballot_sync(0xffffffffu, in && k == pval));
        }
        if (lane == 0) {
            sh.wgt[warp] = cgt;
            sh.weq[warp] = ceq;
        }
        __syncthreads();
        uint32_t gt_base = warp_prefix(sh.wgt, kSelWarps);
        uint32_t eq_base = warp_prefix(sh.weq, kSelWarps);
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
    }
    if (tid == 0) p.n_sel[u] = kk;
}


// ------------------------------------------------------------ cluster path
__global__ void __cluster_dims__(kCl, 1, 1) __launch_bounds__(kClThreads)
select_cluster_kernel(SelectParams p) {
    __shared__ ClShared sh;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int u = blockIdx.x / kCl;
    const int tid = threadIdx.x;
    const int Hkv = p.s.Hkv, MP = p.s.MP;
    int L = p.seq_lens[u / Hkv];
    if (L < 0 || L > MP * kPage) L = 0;       // flagged by the scoring kernel
    const SeqGeom sg = seq_geom(L, p.prefix, p.window);
    const int n = sg.c_hi - sg.c_lo;
    const int kk = p.k_pages < n ? p.k_pages : n;
    int32_t* out = p.sel + (size_t)u * p.s.max_sel;
    pdl_wait();                 // scores and the previous readers of sel
    pdl_launch_dependents();

    if (kk == n) {              // every candidate fits the budget
        for (int i = rank * kClThreads + tid; i < n; i += kCl * kClThreads) out[i] = sg.c_lo + i;
        if (rank == 0 && tid == 0) {
            p.n_sel[u] = n;
            p.keyrange[u] = make_uint2(0u, 0u);
        }
        return;
    }
    if (kk == 0 || n > kClCap) {
        if (rank == 0 && tid == 0) {
            p.n_sel[u] = 0;
            p.keyrange[u] = make_uint2(0u, 0u);
            if (n > kClCap) latch_flag(p.flags, CSA_DEVFLAG_BAD_SELECTION);
        }
        return;
    }
    const int c_lo = sg.c_lo;
    uint32_t kmin, kmax;
    key_range(p.keyrange[u], kmin, kmax);
    cluster_select(cl, sh, p.scores_ws + (size_t)u * MP + c_lo, n, kk, kmin, kmax,
                   [&](int pos, int i) { out[pos] = c_lo + i; });
    cluster_sync_all();         // no CTA's shared memory is read after this
    if (rank == 0 && tid == 0) {   // every CTA read the range before the last barrier
        p.n_sel[u] = kk;
        p.keyrange[u] = make_uint2(0u, 0u);
    }
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t st) {
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemKeys * 4);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    const int units = p.s.B * p.s.Hkv;
    if (units == 0) return cudaSuccess;
    // candidates per unit are at most max_pages - prefix/16 - window/16
    const long long n_max = (long long)p.s.MP - p.prefix / kPage - p.window / kPage;
    if (n_max <= kClCap)
        return launch_pdl(select_cluster_kernel, dim3(units * kCl), dim3(kClThreads), 0, st, p);
    // lists longer than the register capacity keep their keys in shared
    // memory when they fit, else in place over the scores
    SelectParams q = p;
    q.smem_keys = p.s.MP <= kRegCap ? 0 : (p.s.MP <= kSmemKeys ? p.s.MP : 0);
    return launch_pdl(select_kernel, dim3(units), dim3(kSelThreads), (size_t)q.smem_keys * 4, st,
                      q);
}

}  // namespace csa
