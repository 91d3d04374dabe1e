// decode.cu -- split-K flash decoding over the attended pages, in two phases,
// and the kernel that merges the split results.
//
// Combined sparse attention ("Accelerating Long-Context Decoding in
// Large-Scale Hybrid LLMs Without Retraining", abstract): every query head
// attends to a pinned prefix, a sliding window and the selected top-k pages.
// For (sequence b, kv-head g) the attended tokens are
//     A = { t < L : t < Pe  or  t >= L - We  or  page(t) selected }
// and for each of the G query heads of the group
//     out_h = sum_{t in A} softmax_t(scale * q_h . k_t) v_t .
// The dense layer (csa_decode_full) is the same kernel with every page fixed.
//
// Two phases.  Phase 0 takes the fixed list of every unit: the pages holding
// prefix or window tokens, masked to those tokens.  Phase 1 takes the
// selected pages, masked to their other tokens (a selected boundary page is
// split between the phases, so the union is token-exact and nothing counts
// twice).  Phase 0 does not depend on the selection: when the call follows
// csa_score_select on the same stream it runs before the dependency wait,
// while the selection kernel is still working, and only phase 1 waits.  In
// each phase the lists of all units are flattened and split evenly over the
// grid, so ragged lengths and budgets stay balanced.
//
// Per CTA and phase: the page ids of its slice are resolved once into shared
// memory; every warp then streams its own pages (round-robin over the slice)
// with 16-byte cp.async copies into a private double buffer, laid out with
// the 128-byte XOR swizzle (16-byte chunk c of token row r at c ^ (r & 7)),
// so ldmatrix reads it without bank conflicts; slots past the end of the
// sequence are zero-filled by the copy itself.  (Per-page TMA copies were
// measured slower here: their issue cost, paid serially by one thread, caps
// a CTA's request rate.)  Per page a warp computes S^T = K Q^T (16 tokens x
// 8 heads) with mma.sync m16n8k16 (K fragments by ldmatrix, Q^T fragments
// resident in registers), masks it, runs the fp32 online softmax in the exp2
// domain, turns P into the B operand with movmatrix, and accumulates
// O^T += V^T P^T with ldmatrix.trans fragments of V.  At the end of a unit
// the warps merge through shared memory and the CTA writes one partial
// record (m, l, o) of the unit for the phase; the combine kernel merges the
// records of both phases and writes bf16 out and lse.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

template <int D, int NB>
struct DecCfg {
    static constexpr int kWarps = D == 256 ? 8 : 4;
    static constexpr int kThreads = 32 * kWarps;
    // D <= 128 with up to 8 heads per group: registers for four CTAs per SM,
    // so that three fit beside a CTA of the selection kernel when both are
    // resident (16 heads would spill at that bound)
    static constexpr int kMinBlocks = D == 256 ? 1 : (NB == 1 ? 4 : 3);
    static constexpr int kBufs = D == 256 ? 1 : 2;      // page buffers per warp
    static constexpr int kHalf = 32 * D;                // bytes of one page's K (or V) tile
    static constexpr int kPageBytes = 2 * kHalf;
    static constexpr int kHeads = 8 * NB;               // query heads per CTA (padded)
    static constexpr int kMB = D / 16;                  // 16-channel blocks
    static constexpr size_t kStageArea = (size_t)kWarps * kBufs * kPageBytes;
    static constexpr size_t kOw = (size_t)kWarps * kHeads * D * 4;   // aliases the stage area
    static_assert(kOw <= kStageArea, "the merge buffer lives in the stage area");
    static constexpr size_t kMl = (size_t)2 * kWarps * kHeads * 4;
    static constexpr size_t kItems = (size_t)kDecodeItemCap * 8;
    static __host__ __device__ size_t smem_bytes(int units) {
        return 1024 /* alignment slack */ + kStageArea + kMl + kItems + unit_bytes(units);
    }
    // uoff [units + 1] | uinfo [units] (int2: validated seq_len, unused)
    static __host__ __device__ size_t unit_bytes(int units) {
        return (((size_t)(units + 1) * 4 + 15) & ~(size_t)15) + (size_t)units * 8;
    }
};

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Token masks of a work item: which tokens of its page are attended.
constexpr int kMaskAll = 0;     // every valid token (t < L)
constexpr int kMaskFixed = 1;   // prefix or window tokens (t < Pe or t >= L - We)
constexpr int kMaskRest = 2;    // the others (Pe <= t < L - We)

// Fixed list of a unit: the pages holding prefix or window tokens, ascending:
// [0, c_lo) | c_lo when it holds prefix tokens | c_hi - 1 when it holds
// window tokens | [c_hi, np).  With no page left to select from (or in dense
// mode) it is every page, unmasked.
struct FixedList {
    int n_pre, n_blo, n_bhi, n_win;
    __device__ int total() const { return n_pre + n_blo + n_bhi + n_win; }
};

__device__ __forceinline__ FixedList fixed_list(const SeqGeom& sg, bool dense) {
    FixedList f;
    f.n_blo = f.n_bhi = f.n_win = 0;
    if (dense || sg.c_lo == sg.c_hi) {
        f.n_pre = sg.np;
        return f;
    }
    f.n_pre = sg.c_lo;
    f.n_blo = (sg.Pe % kPage) != 0 ? 1 : 0;
    const bool hi_partial = sg.We > 0 && ((sg.L - sg.We) % kPage) != 0;
    f.n_bhi = (hi_partial && !(sg.c_hi - 1 == sg.c_lo && f.n_blo)) ? 1 : 0;
    f.n_win = sg.np - sg.c_hi;
    return f;
}

__device__ __forceinline__ void fixed_item(const SeqGeom& sg, const FixedList& f, int j,
                                           int& page, int& mask) {
    mask = kMaskAll;
    if (j < f.n_pre) { page = j; return; }
    j -= f.n_pre;
    mask = kMaskFixed;
    if (j < f.n_blo) { page = sg.c_lo; return; }
    j -= f.n_blo;
    if (j < f.n_bhi) { page = sg.c_hi - 1; return; }
    j -= f.n_bhi;
    mask = kMaskAll;
    page = sg.c_hi + j;
}

// Unit whose list holds flattened item x (largest u with uoff[u] <= x).
__device__ __forceinline__ int find_unit(const int* uoff, int units, long long x) {
    int lo = 0, hi = units;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (uoff[mid] <= x) lo = mid; else hi = mid;
    }
    while (lo + 1 < units && uoff[lo + 1] <= x) ++lo;   // skip empty units
    return lo;
}

// CTA whose slice [T*i/n, T*(i+1)/n) holds item x.
__device__ __forceinline__ int cta_of(long long x, long long T, int n) {
    long long i = ((x + 1) * n + T - 1) / T - 1;
    return (int)(i < n - 1 ? i : n - 1);
}

// Partial record of one (CTA, unit): o[G][D] relative to the CTA's own max,
// then m[G] (max, exp2 domain) and l[G] (sum); the stride keeps o 16-byte
// aligned.
__host__ __device__ __forceinline__ size_t record_stride(int G, int D) {
    return ((size_t)G * D + 2 * G + 3) & ~(size_t)3;
}

// Combine kernel: merges the partial records of every unit, written in phase
// 0 (fixed pages) by CTAs rec_range.x .. .y and in phase 1 (selected pages)
// by CTAs .z .. .w:
//   M = max_r m_r,  out = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r.
// A unit without records (nothing attended) gets out = 0 and lse = -inf.
// A CTA covers 64 float4 columns of one unit's [G][D] output; its 256 threads
// split the records four ways (online max-rescaled sums, merged with
// shuffles), so no thread walks all the records.
constexpr int kCombineCols = 64;

template <int D>
__global__ void __launch_bounds__(256) combine_kernel(DecodeParams p) {
    pdl_wait();                 // the records belong to the decode kernel
    pdl_launch_dependents();
    const int u = blockIdx.y;
    const int4 rr = p.rec_range[u];
    const int G = p.s.G, Hq = p.s.Hq;
    const int cols = G * D / 4;
    const int c = blockIdx.x * kCombineCols + (threadIdx.x & (kCombineCols - 1));
    const int grp = threadIdx.x / kCombineCols;      // 0..3: record subset
    if (blockIdx.x * kCombineCols >= cols) return;
    const int cc = c < cols ? c : cols - 1;
    const int h = (4 * cc) / D;
    const size_t rs = record_stride(G, D);
    const int n0 = rr.y >= rr.x ? rr.y - rr.x + 1 : 0;
    const int n1 = rr.w >= rr.z ? rr.w - rr.z + 1 : 0;
    const float* base0 = p.partials + ((size_t)rr.x + u) * rs;
    const float* base1 = p.partials + p.phase_floats + ((size_t)rr.z + u) * rs;
    const int nrec = n0 + n1;
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = grp; r0 < nrec; r0 += 4 * 4) {
        float mr[4], lr[4];
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = r0 + 4 * k;
            const float* rc = r < n0 ? base0 + (size_t)r * rs
                                     : (r < nrec ? base1 + (size_t)(r - n0) * rs
                                                 : (n0 > 0 ? base0 : base1));
            mr[k] = r < nrec ? __ldcg(rc + (size_t)G * D + h) : -INFINITY;
            lr[k] = __ldcg(rc + (size_t)G * D + G + h);
            v[k] = __ldcg(reinterpret_cast<const float4*>(rc) + cc);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (mr[k] == -INFINITY) continue;
            const float mn = fmaxf(m, mr[k]);
            const float a = m == -INFINITY ? 0.f : ex2(m - mn), w = ex2(mr[k] - mn);
            acc.x = acc.x * a + v[k].x * w;
            acc.y = acc.y * a + v[k].y * w;
            acc.z = acc.z * a + v[k].z * w;
            acc.w = acc.w * a + v[k].w * w;
            l = l * a + lr[k] * w;
            m = mn;
        }
    }
    // merge the four record groups (threads t, t+64, t+128, t+192)
    __shared__ float sm[4][kCombineCols][6];
    const int col = threadIdx.x & (kCombineCols - 1);
    sm[grp][col][0] = m;
    sm[grp][col][1] = l;
    sm[grp][col][2] = acc.x;
    sm[grp][col][3] = acc.y;
    sm[grp][col][4] = acc.z;
    sm[grp][col][5] = acc.w;
    __syncthreads();
    if (grp != 0 || c >= cols) return;
    float M = -INFINITY;
#pragma unroll
    for (int g2 = 0; g2 < 4; ++g2) M = fmaxf(M, sm[g2][col][0]);
    float L = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < 4; ++g2) {
        const float mg = sm[g2][col][0];
        const float f = mg == -INFINITY ? 0.f : ex2(mg - M);
        L += sm[g2][col][1] * f;
        o0 += sm[g2][col][2] * f;
        o1 += sm[g2][col][3] * f;
        o2 += sm[g2][col][4] * f;
        o3 += sm[g2][col][5] * f;
    }
    const int b = u / p.s.Hkv, g = u % p.s.Hkv;
    const int ch = (4 * c) % D;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const size_t oi = (size_t)b * Hq + (size_t)g * G + h;
    uint2 pk;
    pk.x = pack_bf16x2(o0 * inv, o1 * inv);
    pk.y = pack_bf16x2(o2 * inv, o3 * inv);
    *reinterpret_cast<uint2*>(p.out + oi * D + ch) = pk;
    if (ch == 0 && p.lse) p.lse[oi] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// Issues the cp.async copies of one page's K and V tiles (16 tokens x D) into
// a swizzled buffer; token rows >= rows_valid are zero-filled.
template <int D>
__device__ __forceinline__ void load_page(uint32_t buf, const uint16_t* kt, const uint16_t* vt,
                                          int rows_valid, int lane) {
    constexpr int kChunksPerRow = D / 8;
    constexpr int kChunks = 16 * kChunksPerRow;
#pragma unroll
    for (int i = 0; i < kChunks / 32; ++i) {
        const int idx = i * 32 + lane;
        const int r = idx / kChunksPerRow, c16 = idx % kChunksPerRow;
        const uint32_t off = (c16 >> 3) * 2048 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
        const uint32_t n = r < rows_valid ? 16u : 0u;
        cp_async_16(buf + off, kt + (size_t)r * D + c16 * 8, n);
        cp_async_16(buf + 32 * D + off, vt + (size_t)r * D + c16 * 8, n);
    }
}

template <int D, int NB>
__global__ void __launch_bounds__(DecCfg<D, NB>::kThreads, DecCfg<D, NB>::kMinBlocks)
decode_kernel(DecodeParams p) {
    using C = DecCfg<D, NB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzled page buffers need 1024-byte alignment in the shared window
    uint8_t* stages = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* Ow = reinterpret_cast<float*>(stages);      // reused after the page loop
    float* ms = reinterpret_cast<float*>(stages + C::kStageArea);
    float* ls = ms + C::kWarps * C::kHeads;
    int2* items = reinterpret_cast<int2*>(ls + C::kWarps * C::kHeads);
    int* uoff = reinterpret_cast<int*>(items + kDecodeItemCap);
    const int units = p.s.B * p.s.Hkv;
    int2* uinfo = reinterpret_cast<int2*>(reinterpret_cast<uint8_t*>(uoff) +
                                          (((size_t)(units + 1) * 4 + 15) & ~(size_t)15));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hkv = p.s.Hkv, G = p.s.G, Hq = p.s.Hq;
    int2* rr2 = reinterpret_cast<int2*>(p.rec_range);   // [unit][phase]: first, last CTA
    if (!p.early) {   // wait for everything ahead before reading anything
        pdl_wait();
        pdl_launch_dependents();
    }
    for (int u = tid; u < units; u += C::kThreads) {
        int L = p.seq_lens[u / Hkv];
        if (L < 0 || L > p.s.MP * kPage) {
            latch_flag(p.flags, CSA_DEVFLAG_BAD_SEQ_LEN);
            L = 0;
        }
        uinfo[u] = make_int2(L, 0);
    }

    const int gq = lane >> 2, tq = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    // per-lane ldmatrix geometry (chunk c of row r sits at c ^ (r & 7))
    const int k_tok = ri + ((mi & 1) << 3), k_half = mi >> 1;
    const int v_tok = ri + ((mi >> 1) << 3), v_half = mi & 1;
    const float sl2 = p.scale_log2;
    const uint32_t wbuf = smem_u32(stages) + (uint32_t)(warp * C::kBufs * C::kPageBytes);
    const size_t rs = record_stride(G, D);

    // Phase 0 streams the fixed pages (prefix and window), which do not depend
    // on the selection; phase 1 the selected pages.  With p.early set, phase 0
    // runs while the selection kernel ahead is still working.
    for (int ph = 0; ph < 2; ++ph) {
        if (ph == 1 && p.early) {
            pdl_wait();         // the selection is complete and visible
            pdl_launch_dependents();
        }
        __syncthreads();        // uinfo written; smem of the previous phase free
        // ---- per-unit list lengths and their exclusive scan
        for (int u = tid; u < units; u += C::kThreads) {
            const SeqGeom sg = seq_geom(uinfo[u].x, p.prefix, p.window);
            int n = 0;
            if (ph == 0) {
                n = fixed_list(sg, p.dense).total();
            } else if (!p.dense && sg.c_lo < sg.c_hi) {
                n = p.n_sel[u];
                const int cap = p.s.max_sel < sg.c_hi - sg.c_lo ? p.s.max_sel : sg.c_hi - sg.c_lo;
                if (n < 0 || n > cap) {
                    latch_flag(p.flags, CSA_DEVFLAG_BAD_SELECTION);
                    n = n < 0 ? 0 : cap;
                }
            }
            uoff[u] = n;
        }
        __syncthreads();
        if (warp == 0) {
            int carry = 0;
            for (int base = 0; base < units; base += 32) {
                const int u = base + lane;
                const int v = u < units ? uoff[u] : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (u < units) uoff[u] = carry + incl - v;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) uoff[units] = carry;
        }
        __syncthreads();
        const long long T = uoff[units];
        // at least kMinItems pages per CTA (fewer partial records to merge;
        // measured faster than one or two pages per warp in either phase),
        // and every participating CTA owns at least one item
        constexpr long long kMinItems = 4 * C::kWarps;
        long long want = (T + kMinItems - 1) / kMinItems;
        if (want < 1) want = 1;
        const int n_cta = (int)(want < (long long)gridDim.x ? want : gridDim.x);
        const long long s = blockIdx.x < (unsigned)n_cta ? T * blockIdx.x / n_cta : T;
        const long long e = blockIdx.x < (unsigned)n_cta ? T * (blockIdx.x + 1) / n_cta : T;
        if (blockIdx.x == 0) {   // units without pages in this phase: no records
            for (int u = tid; u < units; u += C::kThreads)
                if (uoff[u + 1] == uoff[u]) rr2[2 * u + ph] = make_int2(0, -1);
        }
        if (s >= e) continue;

        // ---- resolve the physical page of every item of this CTA's slice
        for (long long x = s + tid; x < e; x += C::kThreads) {
            const int u = find_unit(uoff, units, x);
            const int b = u / Hkv;
            const int j = (int)(x - uoff[u]);
            const SeqGeom sg = seq_geom(uinfo[u].x, p.prefix, p.window);
            int page = 0, mask = kMaskAll;
            bool ok = true;
            if (ph == 0) {
                fixed_item(sg, fixed_list(sg, p.dense), j, page, mask);
            } else {
                const int32_t* su = p.sel + (size_t)u * p.s.max_sel;
                page = su[j];
                mask = kMaskRest;
                ok = page >= sg.c_lo && page < sg.c_hi && (j == 0 || su[j - 1] < page);
                if (!ok) latch_flag(p.flags, CSA_DEVFLAG_BAD_SELECTION);
            }
            int phys = -1;
            if (ok) {
                phys = p.page_table[(size_t)b * p.s.MP + page];
                if (phys < 0 || phys >= p.s.NPG) {
                    latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
                    phys = -1;
                }
            }
            items[x - s] = make_int2(phys, page * 4 + mask);
        }
        __syncthreads();

        const int u_first = find_unit(uoff, units, s);
        const int u_last = find_unit(uoff, units, e - 1);
        float* region = p.partials + (size_t)ph * p.phase_floats;

        for (int u = u_first; u <= u_last; ++u) {
            const long long a = s > uoff[u] ? s : uoff[u];
            const long long bnd = e < uoff[u + 1] ? e : uoff[u + 1];
            if (a >= bnd) continue;
            const int b = u / Hkv, g = u % Hkv;
            const int L = uinfo[u].x;
            const SeqGeom sg = seq_geom(L, p.prefix, p.window);
            const int Pe = sg.Pe, Lw = L - sg.We;

            // Q^T as the B operand: b0 = q[head][16kb + 2tq, +1], b1 = +8
            uint32_t qf[C::kMB][NB][2];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int head = nb * 8 + gq;
                const uint32_t* qw = reinterpret_cast<const uint32_t*>(
                    p.q + ((size_t)b * Hq + (size_t)g * G + (head < G ? head : 0)) * D);
#pragma unroll
                for (int kb = 0; kb < C::kMB; ++kb) {
                    qf[kb][nb][0] = head < G ? __ldg(qw + 8 * kb + tq) : 0u;
                    qf[kb][nb][1] = head < G ? __ldg(qw + 8 * kb + 4 + tq) : 0u;
                }
            }
            float m[NB][2], l[NB][2], o[C::kMB][NB][4];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                m[nb][0] = m[nb][1] = -INFINITY;
                l[nb][0] = l[nb][1] = 0.f;
#pragma unroll
                for (int mb = 0; mb < C::kMB; ++mb)
                    o[mb][nb][0] = o[mb][nb][1] = o[mb][nb][2] = o[mb][nb][3] = 0.f;
            }

            // this warp's items of the segment: a + warp, a + warp + kWarps, ...
            auto issue = [&](long long x, int slot) {
                const int2 it = items[x - s];
                if (it.x >= 0) {
                    const int page = it.y >> 2;
                    const size_t tile = ((size_t)it.x * Hkv + g) * kPage * D;
                    const int rows = L - page * kPage < kPage ? L - page * kPage : kPage;
                    load_page<D>(wbuf + (uint32_t)(slot * C::kPageBytes), p.k_cache + tile,
                                 p.v_cache + tile, rows, lane);
                }
                cp_async_commit();
            };
            long long x = a + warp;
            int slot = 0;
            if (x < bnd) issue(x, 0);
            for (; x < bnd; x += C::kWarps) {
                const long long xn = x + C::kWarps;
                if (C::kBufs == 2) {
                    if (xn < bnd) {
                        issue(xn, slot ^ 1);
                        cp_async_wait<1>();
                    } else {
                        cp_async_wait<0>();
                    }
                } else {
                    cp_async_wait<0>();
                }
                __syncwarp();
                const int2 it = items[x - s];
                if (it.x >= 0) {
                    const int page = it.y >> 2;
                    const int mask = it.y & 3;
                    const uint32_t kbase = wbuf + (uint32_t)(slot * C::kPageBytes);
                    const uint32_t vbase = kbase + C::kHalf;
                    // ---- S^T = K Q^T
                    float sacc[NB][4];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
                        sacc[nb][0] = sacc[nb][1] = sacc[nb][2] = sacc[nb][3] = 0.f;
#pragma unroll
                    for (int kb = 0; kb < C::kMB; ++kb) {
                        const int chunk = 2 * kb + k_half;
                        const uint32_t addr = kbase + (chunk >> 3) * 2048 + k_tok * 128 +
                                              (((chunk & 7) ^ ri) << 4);
                        uint32_t af[4];
                        ldsm_x4(af, addr);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
                            mma_bf16_16816(sacc[nb], af, qf[kb][nb][0], qf[kb][nb][1]);
                    }
                    // ---- mask and online softmax (exp2 domain)
                    const int t0 = page * kPage + gq, t1 = t0 + 8;
                    const bool f0 = t0 < Pe || t0 >= Lw, f1 = t1 < Pe || t1 >= Lw;
                    const bool in0 = t0 < L && (mask == kMaskAll || (mask == kMaskFixed) == f0);
                    const bool in1 = t1 < L && (mask == kMaskAll || (mask == kMaskFixed) == f1);
                    uint32_t pb[NB][2];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const float s00 = in0 ? sacc[nb][0] * sl2 : -INFINITY;
                        const float s01 = in0 ? sacc[nb][1] * sl2 : -INFINITY;
                        const float s10 = in1 ? sacc[nb][2] * sl2 : -INFINITY;
                        const float s11 = in1 ? sacc[nb][3] * sl2 : -INFINITY;
                        float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
                        for (int o2 = 4; o2 < 32; o2 <<= 1) {
                            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
                            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
                        }
                        const float mn0 = fmaxf(m[nb][0], mx0), mn1 = fmaxf(m[nb][1], mx1);
                        const float base0 = mn0 == -INFINITY ? 0.f : mn0;
                        const float base1 = mn1 == -INFINITY ? 0.f : mn1;
                        const float al0 = ex2(m[nb][0] - base0), al1 = ex2(m[nb][1] - base1);
                        const uint32_t P0 = pack_bf16x2(ex2(s00 - base0), ex2(s01 - base1));
                        const uint32_t P1 = pack_bf16x2(ex2(s10 - base0), ex2(s11 - base1));
                        l[nb][0] = l[nb][0] * al0 + bf16_lo(P0) + bf16_lo(P1);
                        l[nb][1] = l[nb][1] * al1 + bf16_hi(P0) + bf16_hi(P1);
                        m[nb][0] = mn0;
                        m[nb][1] = mn1;
#pragma unroll
                        for (int mb = 0; mb < C::kMB; ++mb) {
                            o[mb][nb][0] *= al0;
                            o[mb][nb][1] *= al1;
                            o[mb][nb][2] *= al0;
                            o[mb][nb][3] *= al1;
                        }
                        pb[nb][0] = movmatrix_trans(P0);
                        pb[nb][1] = movmatrix_trans(P1);
                    }
                    // ---- O^T += V^T P^T
#pragma unroll
                    for (int mb = 0; mb < C::kMB; ++mb) {
                        const int chunk = 2 * mb + v_half;
                        const uint32_t addr = vbase + (chunk >> 3) * 2048 + v_tok * 128 +
                                              (((chunk & 7) ^ ri) << 4);
                        uint32_t af[4];
                        ldsm_x4_trans(af, addr);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
                            mma_bf16_16816(o[mb][nb], af, pb[nb][0], pb[nb][1]);
                    }
                }
                __syncwarp();                 // the buffer is refilled next
                if (C::kBufs == 1) {
                    if (xn < bnd) issue(xn, 0);
                } else {
                    slot ^= 1;
                }
            }

            // ---- merge the warps of this CTA (Ow aliases the page buffers)
            __syncthreads();
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v = l[nb][hh];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    l[nb][hh] = v;
                }
                if (gq == 0) {
                    ms[warp * C::kHeads + nb * 8 + 2 * tq] = m[nb][0];
                    ms[warp * C::kHeads + nb * 8 + 2 * tq + 1] = m[nb][1];
                    ls[warp * C::kHeads + nb * 8 + 2 * tq] = l[nb][0];
                    ls[warp * C::kHeads + nb * 8 + 2 * tq + 1] = l[nb][1];
                }
#pragma unroll
                for (int mb = 0; mb < C::kMB; ++mb) {
                    float* ow = Ow + (size_t)warp * C::kHeads * D;
                    const int h0 = nb * 8 + 2 * tq, c0 = mb * 16 + gq;
                    ow[(size_t)h0 * D + c0] = o[mb][nb][0];
                    ow[(size_t)(h0 + 1) * D + c0] = o[mb][nb][1];
                    ow[(size_t)h0 * D + c0 + 8] = o[mb][nb][2];
                    ow[(size_t)(h0 + 1) * D + c0 + 8] = o[mb][nb][3];
                }
            }
            __syncthreads();

            // ---- this CTA's partial record of the unit (merged by the combine kernel)
            float* rec = region + ((size_t)blockIdx.x + u) * rs;
            for (int idx = tid; idx < G * D; idx += C::kThreads) {
                const int h = idx / D, c = idx % D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, ms[w * C::kHeads + h]);
                float acc = 0.f, lsum = 0.f;
#pragma unroll
                for (int w = 0; w < C::kWarps; ++w) {
                    const float mw = ms[w * C::kHeads + h];
                    const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
                    acc += Ow[((size_t)w * C::kHeads + h) * D + c] * f;
                    lsum += ls[w * C::kHeads + h] * f;
                }
                rec[(size_t)h * D + c] = acc;
                if (c == 0) {
                    rec[(size_t)G * D + h] = M;
                    rec[(size_t)G * D + G + h] = lsum;
                }
            }
            const int first_cta = cta_of(uoff[u], T, n_cta);
            if (blockIdx.x == first_cta && tid == 0)
                rr2[2 * u + ph] = make_int2(first_cta, cta_of(uoff[u + 1] - 1, T, n_cta));
            __syncthreads();   // Ow / ms / ls and the page buffers are reused next
        }
    }
}

template <int D, int NB>
cudaError_t launch_decode_t(const DecodeParams& p, cudaStream_t st) {
    using C = DecCfg<D, NB>;
    auto kern = decode_kernel<D, NB>;
    const int units = p.s.B * p.s.Hkv;
    const size_t smem = C::smem_bytes(units);
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)C::smem_bytes(kMaxUnits));
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    const int grid = decode_grid(p.s);
    cudaError_t e = launch_pdl(kern, dim3(grid), dim3(C::kThreads), smem, st, p);
    if (e != cudaSuccess) return e;
    const int col_blocks = (p.s.G * D / 4 + kCombineCols - 1) / kCombineCols;
    return launch_pdl(combine_kernel<D>, dim3(col_blocks, units), dim3(256), 0, st, p);
}

}  // namespace

// Resident CTAs of the decode kernel for this shape (shared memory decides),
// times the SM count, and at least enough CTAs that no slice exceeds the
// per-CTA item capacity.
template <int D, int NB>
static int resident_per_sm(int units) {
    const size_t per_cta = DecCfg<D, NB>::smem_bytes(units) + 1024;   // + per-CTA reserve
    int n = (int)((size_t)(228 * 1024) / per_cta);
    if (n > 3) n = 3;
    return n < 1 ? 1 : n;
}

int decode_grid(const Shape& s) {
    const int units = s.B * s.Hkv;
    const bool nb2 = s.G > 8;
    int per_sm = 1;
    switch (s.D) {
        case 64: per_sm = nb2 ? resident_per_sm<64, 2>(units) : resident_per_sm<64, 1>(units); break;
        case 128: per_sm = nb2 ? resident_per_sm<128, 2>(units) : resident_per_sm<128, 1>(units); break;
        default: per_sm = nb2 ? resident_per_sm<256, 2>(units) : resident_per_sm<256, 1>(units); break;
    }
    long long grid = (long long)per_sm * device_sm_count();
    // a list may exceed its sequence's pages by the two boundary pages when a
    // caller-provided selection is malformed; size for that too
    const long long ub = (long long)units * (s.MP + 2);
    const long long need = (ub + kDecodeItemCap - 1) / kDecodeItemCap;
    if (need > grid) grid = need;
    return (int)(grid < 1 ? 1 : grid);
}

size_t decode_record_floats(const Shape& s) { return record_stride(s.G, s.D); }

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st) {
    const int nb = p.s.G > 8 ? 2 : 1;
    switch (p.s.D * 10 + nb) {
        case 641: return launch_decode_t<64, 1>(p, st);
        case 642: return launch_decode_t<64, 2>(p, st);
        case 1281: return launch_decode_t<128, 1>(p, st);
        case 1282: return launch_decode_t<128, 2>(p, st);
        case 2561: return launch_decode_t<256, 1>(p, st);
        case 2562: return launch_decode_t<256, 2>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
