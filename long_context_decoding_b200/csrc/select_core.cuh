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
    uint32_t local[256];             // this CTA's histogram
    uint32_t cgt[kCl], ceq[kCl];     // every CTA: the (above, equal) counts of each rank
    uint32_t red[kClWarps], wgt[kClWarps], weq[kClWarps];
    uint32_t digit, gt, cnt;
};

// Split cluster barrier (arrive now, wait later) with release / acquire
// semantics on the cluster's shared memory.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Empties rank 0's merge buffers and arrives at the cluster barrier that
// publishes them; call before the dependency wait (it touches only this
// CTA's shared memory).  cluster_select waits on that barrier before its
// first remote access.
__device__ __forceinline__ void cluster_select_begin(ClShared& sh) {
    for (int i = threadIdx.x; i < kClPasses * 256; i += kClThreads) (&sh.hist[0][0])[i] = 0;
    __syncthreads();
    cluster_arrive();
}

// Key range of a unit as published by the scoring kernel: x = ~min key,
// y = max key (both merged with atomicMax, so zero means "nothing yet").
// A range nobody wrote becomes the full key space, which is still exact.
__device__ __forceinline__ void key_range(uint2 r, uint32_t& kmin, uint32_t& kmax) {
    kmin = ~r.x;
    kmax = r.y;
    if (kmin > kmax) {
        kmin = 0u;
        kmax = 0xffffffffu;
    }
}

// Selects the kk largest of the n scores sc[0, n) (0 < kk < n <= kClCap),
// whose order keys all lie in [kmin, kmax], with the CTAs of the cluster;
// calls emit(pos, i) for every selected candidate i in this CTA's share, pos
// being its rank in ascending index order.  Called by every thread of all
// kCl CTAs after cluster_select_begin; ends with a cluster barrier, after
// which no CTA reads another's shared memory.
template <typename Emit>
__device__ void cluster_select(cg::cluster_group& cl, ClShared& sh, const float* sc, int n, int kk,
                               uint32_t kmin, uint32_t kmax, Emit emit) {
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
#pragma unroll
    for (int j = 0; j < kClKeys; ++j) {
        const int i = wlo + 32 * j + lane;
        kr[j] = order_key(__ldcg(sc + (i < whi ? i : 0)));
    }
    cluster_wait();             // rank 0's buffers are empty everywhere

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

    // compaction: per-warp, per-CTA and per-cluster prefixes of (above, equal);
    // every CTA sends its totals to every CTA, so one barrier suffices
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
    if (tid >= kClThreads - kCl) {   // last warp (its gt_base + cgt is the CTA's total)
        ClShared* dst = cl.map_shared_rank(&sh, tid - (kClThreads - kCl));
        dst->cgt[rank] = gt_base + cgt;
        dst->ceq[rank] = eq_base + ceq;
    }
    cl.sync();                  // counts everywhere; no remote reads after this
    {
        const uint32_t x = lane < kCl && lane < rank ? sh.cgt[lane] : 0u;
        const uint32_t y = lane < kCl && lane < rank ? sh.ceq[lane] : 0u;
        gt_base += __reduce_add_sync(0xffffffffu, x);
        eq_base += __reduce_add_sync(0xffffffffu, y);
    }
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
