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
// key shares (the unit's key range from the scoring kernel), and run an
// MSB-first radix select with 8-bit digits.  In each pass every CTA builds
// its histogram in its own shared memory, one cluster barrier publishes
// them, and every CTA reads all 8 through distributed shared memory (one
// round trip), sums them and finds the same digit; a pass ends the search
// early when the bin holding the k-th key is taken whole.  The same reads
// give every CTA each rank's count of keys above the digit and in it, so
// after the last pass every CTA knows each rank's (above, equal) totals
// without another exchange, and per-warp prefixes give every selected
// candidate its position in ascending index order: all keys above the
// threshold plus the lowest-index keys equal to it.
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
    uint32_t hist[2][256];           // this CTA's histogram, by pass parity
    uint32_t rgt[kClWarps][kCl];     // per warp: each rank's keys above the digit
    uint32_t req[kCl];               // each rank's keys in the digit's bin
    uint32_t cgt[kCl], ceq[kCl];     // each rank's (above, equal) totals
    uint32_t red[kClWarps], wgt[kClWarps], weq[kClWarps];
    uint32_t digit, gt, cnt;
};

// Cluster barrier with release / acquire semantics on the cluster's shared
// memory (every thread of every CTA).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
// whose order keys all lie in [kmin, kmax] (a key outside is clamped into
// it, so a stale range still gives kk distinct positions), with the CTAs of
// the cluster; calls emit(pos, i) for every selected candidate i in this
// CTA's share, pos being its rank in ascending index order.  Called by every
// thread of all kCl CTAs.  The last remote access is a read before emit; the
// caller ends with a cluster barrier (cluster_sync_all) after emit and
// before any CTA exits.
template <typename Emit>
__device__ void cluster_select(cg::cluster_group& cl, ClShared& sh, const float* sc, int n, int kk,
                               uint32_t kmin, uint32_t kmax, Emit emit) {
    const int rank = (int)cl.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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
        const uint32_t k = order_key(__ldcg(sc + (i < whi ? i : 0)));
        kr[j] = k < kmin ? kmin : (k > kmax ? kmax : k);
    }

    uint32_t pmask, pval;
    uint32_t remaining = (uint32_t)kk;
    bool take_all = false;
    uint32_t gt_acc = 0;        // thread r < kCl: rank r's keys above the digits so far
    if (kmin == kmax) {
        pmask = 0xffffffffu;
        pval = kmax;
        if (tid < kCl) {        // every key equal: a rank's count is its chunk's size
            const int lo = tid * chunk, hi = lo + chunk < n ? lo + chunk : n;
            sh.req[tid] = hi > lo ? (uint32_t)(hi - lo) : 0u;
        }
    } else {
        int hb = 31 - __clz(kmin ^ kmax);
        pmask = hb >= 31 ? 0u : (0xffffffffu << (hb + 1));
        pval = kmax & pmask;
        for (int pass = 0;; ++pass) {
            const int lo_bit = hb - 7 > 0 ? hb - 7 : 0;
            const uint32_t dmask = (1u << (hb - lo_bit + 1)) - 1u;
            // the buffer of this parity was last read by the other CTAs in
            // pass - 2, before they arrived at the barrier of pass - 1
            uint32_t* hl = sh.hist[pass & 1];
            hl[tid] = 0;
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kClKeys; ++j)
                if (wlo + 32 * j + lane < whi && (kr[j] & pmask) == pval)
                    atomicAdd(&hl[(kr[j] >> lo_bit) & dmask], 1u);
            cluster_sync_all();             // every CTA's histogram is complete
            // bin 255 - tid of every rank (descending digit order)
            uint32_t h[kCl];
#pragma unroll
            for (int r = 0; r < kCl; ++r) h[r] = cl.map_shared_rank(hl, r)[255 - tid];
            uint32_t vbin = 0;
#pragma unroll
            for (int r = 0; r < kCl; ++r) vbin += h[r];
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
#pragma unroll
                for (int r = 0; r < kCl; ++r) sh.req[r] = h[r];
            }
            __syncthreads();
            const uint32_t d = sh.digit, gt = sh.gt, cnt = sh.cnt;
            // each rank's keys in the bins above the digit (this thread's bin
            // is 255 - tid)
            const bool above = (uint32_t)(255 - tid) > d;
#pragma unroll
            for (int r = 0; r < kCl; ++r) {
                const uint32_t v = __reduce_add_sync(0xffffffffu, above ? h[r] : 0u);
                if (lane == 0) sh.rgt[warp][r] = v;
            }
            __syncthreads();
            if (tid < kCl) {
#pragma unroll
                for (int w = 0; w < kClWarps; ++w) gt_acc += sh.rgt[w][tid];
            }
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
    if (tid < kCl) {
        sh.cgt[tid] = gt_acc;
        sh.ceq[tid] = sh.req[tid];
    }

    // compaction: per-warp prefixes of (above, equal) in this CTA, on top of
    // the lower ranks' totals
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
