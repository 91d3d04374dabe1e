// select_core.cuh -- exact top-k of one unit's page scores with a cluster of
// 8 CTAs, shared by the selection kernel and the fused selection + decode
// kernel.
//
// The fixed budget of the most relevant tokens ("Accelerating Long-Context
// Decoding ...", abstract) is taken as the k = floor(budget / 16) candidate
// pages with the highest Quest score ("Methodology"; "The Move": paged
// top-k); ties go to the lower logical page.  The 8 CTAs of a cluster (256
// threads, 8 keys per thread in registers, up to 16384 candidates) turn the
// fp32 scores into order-preserving uint32 keys, strip the high bits every
// key shares (cluster min/max), and run an MSB-first radix select with 8-bit
// digits: local histograms are merged in rank 0's shared memory through
// distributed shared memory, every CTA reads the merged histogram and finds
// the same digit, and a pass ends the search early when the bin holding the
// k-th key is taken whole.  Per-warp, per-CTA and per-cluster prefixes of the
// (above, equal) counts then give every selected candidate its position in
// ascending index order: all keys above the threshold plus the lowest-index
// keys equal to it.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace csa {

namespace cg = cooperative_groups;

// Exclusive prefix over the warps of v_warp (one value per warp, published in
// buf by lane 0): returns sum of buf[w] for w < this warp.
__device__ __forceinline__ uint32_t warp_prefix(const uint32_t* buf, int nwarps) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t x = lane < nwarps ? buf[lane] : 0u, incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    return __shfl_sync(0xffffffffu, incl - x, warp);
}

constexpr int kCl = 8;                              // CTAs per unit
constexpr int kClThreads = 256;
constexpr int kClWarps = kClThreads / 32;
constexpr int kClKeys = 8;                          // keys per thread
constexpr int kClCap = kCl * kClThreads * kClKeys;  // 16384 candidates
constexpr int kClPasses = 4;                        // at most four 8-bit digits

struct ClShared {
    uint32_t hist[kClPasses][256];   // rank 0: merged histogram of each pass
    uint32_t local[256];             // this CTA's histogram / copy of the merged one
    uint32_t kmin, kmax;             // rank 0: cluster min / max
    uint32_t cgt[kCl], ceq[kCl];     // rank 0: per-CTA (above, equal) counts
    uint32_t red[kClWarps], wgt[kClWarps], weq[kClWarps];
    uint32_t digit, gt, cnt;
};

// Rank 0's merge buffers start empty; call before the first cluster barrier
// (the first barrier of cluster_select publishes them).
__device__ __forceinline__ void cluster_select_init(ClShared& sh) {
    for (int i = threadIdx.x; i < kClPasses * 256; i += kClThreads) (&sh.hist[0][0])[i] = 0;
    if (threadIdx.x == 0) {
        sh.kmin = 0xffffffffu;
        sh.kmax = 0u;
    }
}

// Selects the kk largest of the n scores sc[0, n) (0 < kk < n <= kClCap)
// with the CTAs of the cluster; calls emit(pos, i) for every selected
// candidate i in this CTA's share, pos being its rank in ascending index
// order.  Called by every thread of all kCl CTAs.
template <typename Emit>
__device__ void cluster_select(cg::cluster_group& cl, ClShared& sh, const float* sc, int n, int kk,
                               Emit emit) {
    const int rank = (int)cl.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    ClShared* sh0 = cl.map_shared_rank(&sh, 0);

    // this CTA's chunk of the candidates; warp w holds a span, lane l the
    // keys span_lo + 32 j + l (coalesced loads)
    const int chunk = (n + kCl - 1) / kCl;
    const int clo = rank * chunk, chi = clo + chunk < n ? clo + chunk : n;
    const int wspan = ((chunk + kClWarps - 1) / kClWarps + 31) & ~31;
    const int wlo = clo + warp * wspan;
    const int whi = wlo + wspan < chi ? wlo + wspan : chi;
    uint32_t kr[kClKeys];
    float v[kClKeys];
#pragma unroll
    for (int j = 0; j < kClKeys; ++j) {
        const int i = wlo + 32 * j + lane;
        v[j] = __ldcg(sc + (i < whi ? i : 0));
    }
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int j = 0; j < kClKeys; ++j) {
        kr[j] = order_key(v[j]);
        if (wlo + 32 * j + lane < whi) {
            kmin = min(kmin, kr[j]);
            kmax = max(kmax, kr[j]);
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        sh.red[warp] = kmin;
        sh.wgt[warp] = kmax;
    }
    cl.sync();                  // rank 0 buffers initialised everywhere; warp results in
    if (warp == 0) {
        kmin = __reduce_min_sync(0xffffffffu, lane < kClWarps ? sh.red[lane] : 0xffffffffu);
        kmax = __reduce_max_sync(0xffffffffu, lane < kClWarps ? sh.wgt[lane] : 0u);
        if (lane == 0) {
            atomicMin(&sh0->kmin, kmin);
            atomicMax(&sh0->kmax, kmax);
        }
    }
    cl.sync();
    kmin = sh0->kmin;
    kmax = sh0->kmax;

    uint32_t pmask, pval;
    uint32_t remaining = (uint32_t)kk;
    bool take_all = false;
    if (kmin == kmax) {
        pmask = 0xffffffffu;
        pval = kmax;
    } else {
        int hb = 31 - __clz(kmin ^ kmax);
        pmask = hb >= 31 ? 0u : (0xffffffffu << (hb + 1));
        pval = kmax & pmask;
        for (int pass = 0;; ++pass) {
            const int lo_bit = hb - 7 > 0 ? hb - 7 : 0;
            const uint32_t dmask = (1u << (hb - lo_bit + 1)) - 1u;
            sh.local[tid] = 0;
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kClKeys; ++j)
                if (wlo + 32 * j + lane < whi && (kr[j] & pmask) == pval)
                    atomicAdd(&sh.local[(kr[j] >> lo_bit) & dmask], 1u);
            __syncthreads();
            if (sh.local[tid]) atomicAdd(&sh0->hist[pass][tid], sh.local[tid]);
            cl.sync();
            // every CTA reads the merged histogram and finds the same digit
            const uint32_t vbin = sh0->hist[pass][255 - tid];   // descending digit order
            uint32_t incl = vbin;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane == 31) sh.red[warp] = incl;
            __syncthreads();
            const uint32_t ge = incl + warp_prefix(sh.red, kClWarps);
            const uint32_t gtc = ge - vbin;
            if (gtc < remaining && remaining <= ge) {
                sh.digit = 255 - tid;
                sh.gt = gtc;
                sh.cnt = vbin;
            }
            __syncthreads();
            const uint32_t d = sh.digit, gt = sh.gt, cnt = sh.cnt;
            remaining -= gt;
            pval |= d << lo_bit;
            pmask |= dmask << lo_bit;
            if (cnt == remaining) {
                take_all = true;
                break;
            }
            if (lo_bit == 0 || pass + 1 == kClPasses) break;
            hb = lo_bit - 1;
        }
    }
    const uint32_t eq_take = take_all ? 0xffffffffu : remaining;

    // compaction: per-warp, per-CTA and per-cluster prefixes of (above, equal)
    uint32_t cgt = 0, ceq = 0;
#pragma unroll
    for (int j = 0; j < kClKeys; ++j) {
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
    uint32_t gt_base = warp_prefix(sh.wgt, kClWarps);
    uint32_t eq_base = warp_prefix(sh.weq, kClWarps);
    if (tid == kClThreads - 1) {     // this CTA's totals to rank 0
        sh0->cgt[rank] = gt_base + cgt;
        sh0->ceq[rank] = eq_base + ceq;
    }
    cl.sync();
    {
        const uint32_t x = lane < kCl && lane < rank ? sh0->cgt[lane] : 0u;
        const uint32_t y = lane < kCl && lane < rank ? sh0->ceq[lane] : 0u;
        gt_base += __reduce_add_sync(0xffffffffu, x);
        eq_base += __reduce_add_sync(0xffffffffu, y);
    }
    cl.sync();                  // rank 0 stays alive until every CTA has read it
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kClKeys; ++j) {
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
            if (pos < (uint32_t)kk) emit((int)pos, i);
        }
        gt_base += __popc(bgt);
        eq_base += __popc(beq);
    }
}

}  // namespace csa
