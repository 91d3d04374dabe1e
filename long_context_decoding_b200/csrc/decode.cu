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
// with 16-byte cp.async copies into a private ring of K/V tile slots (four at
// D <= 128, two at D = 256), laid out with the 128-byte XOR swizzle (16-byte
// chunk c of token row r at c ^ (r & 7)),
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
#include "attend_core.cuh"
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
    static constexpr int kHalves = D == 256 ? 3 : 4;    // K/V tile slots per warp
    using Tile = TileCfg<D, NB, kWarps, kHalves>;
    static constexpr size_t kStageArea = Tile::kStageArea;
    static constexpr size_t kMl = Tile::kMl;
    static constexpr int kHeads = Tile::kHeads;
    static constexpr size_t kItems = (size_t)kDecodeItemCap * 8;
    static __host__ __device__ size_t smem_bytes(int units) {
        return 1024 /* alignment slack */ + kStageArea + kMl + kItems + unit_bytes(units);
    }
    // uoff [units + 1] | uinfo [units] (int2: validated seq_len, fixed items of the pass)
    static __host__ __device__ size_t unit_bytes(int units) {
        return (((size_t)(units + 1) * 4 + 15) & ~(size_t)15) + (size_t)units * 8;
    }
};

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

template <int D, int NB>
__global__ void __launch_bounds__(DecCfg<D, NB>::kThreads, DecCfg<D, NB>::kMinBlocks)
decode_kernel(DecodeParams p) {
    using C = DecCfg<D, NB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzled page buffers need 1024-byte alignment in the shared window
    uint8_t* stages = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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
    // Until the dependency wait the kernel reads only caller inputs (lengths,
    // selection, page table); the cache, the record ranges and the partial
    // records, which the kernels ahead may still use, only after it.
    for (int u = tid; u < units; u += C::kThreads) {
        int L = p.seq_lens[u / Hkv];
        if (L < 0 || L > p.s.MP * kPage) {
            latch_flag(p.flags, CSA_DEVFLAG_BAD_SEQ_LEN);
            L = 0;
        }
        uinfo[u] = make_int2(L, 0);
    }

    AttendArgs A;
    A.q = p.q;
    A.k_cache = p.k_cache;
    A.v_cache = p.v_cache;
    A.Hq = Hq;
    A.Hkv = Hkv;
    A.G = G;
    A.prefix = p.prefix;
    A.window = p.window;
    A.scale_log2 = p.scale_log2;
    const size_t rs = record_stride(G, D);

    // Phase 0 streams the fixed pages (prefix and window), which do not depend
    // on the selection; phase 1 the selected pages.  With p.early set, phase 0
    // runs while the selection kernel ahead is still working.  Without it
    // both lists form one pass: each unit's fixed pages, then its selected
    // pages, flattened and split together (one chain of round trips, not two).
    const int passes = p.early ? 2 : 1;
    for (int ph = 0; ph < passes; ++ph) {
        if (ph == 1) {
            pdl_wait();         // the selection is complete and visible
            pdl_launch_dependents();
        }
        const bool with_fixed = ph == 0, with_sel = ph == 1 || !p.early;
        __syncthreads();        // uinfo written; smem of the previous phase free
        // ---- per-unit list lengths (fixed in uinfo.y) and their exclusive scan
        for (int u = tid; u < units; u += C::kThreads) {
            const SeqGeom sg = seq_geom(uinfo[u].x, p.prefix, p.window);
            const int nf = with_fixed ? fixed_list(sg, p.dense).total() : 0;
            int n = 0;
            if (with_sel && !p.dense && sg.c_lo < sg.c_hi) {
                n = p.n_sel[u];
                const int cap = p.s.max_sel < sg.c_hi - sg.c_lo ? p.s.max_sel : sg.c_hi - sg.c_lo;
                if (n < 0 || n > cap) {
                    latch_flag(p.flags, CSA_DEVFLAG_BAD_SELECTION);
                    n = n < 0 ? 0 : cap;
                }
            }
            uinfo[u].y = nf;
            uoff[u] = nf + n;
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

        // ---- resolve the physical page of every item of this CTA's slice
        for (long long x = s + tid; x < e; x += C::kThreads) {
            const int u = find_unit(uoff, units, x);
            const int b = u / Hkv;
            const int j = (int)(x - uoff[u]);
            const SeqGeom sg = seq_geom(uinfo[u].x, p.prefix, p.window);
            int page = 0, mask = kMaskAll;
            bool ok = true;
            if (j < uinfo[u].y) {
                fixed_item(sg, fixed_list(sg, p.dense), j, page, mask);
            } else {
                const int js = j - uinfo[u].y;
                const int32_t* su = p.sel + (size_t)u * p.s.max_sel;
                page = su[js];
                mask = kMaskRest;
                ok = page >= sg.c_lo && page < sg.c_hi && (js == 0 || su[js - 1] < page);
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
        if (!p.early) {          // the one pass: wait for everything ahead now
            pdl_wait();
            pdl_launch_dependents();
        }
        if (blockIdx.x == 0) {   // units without pages in this phase: no records
            for (int u = tid; u < units; u += C::kThreads) {
                if (uoff[u + 1] == uoff[u]) rr2[2 * u + ph] = make_int2(0, -1);
                if (passes == 1) rr2[2 * u + 1] = make_int2(0, -1);   // one pass: region 0 only
            }
        }
        if (s >= e) continue;

        const int u_first = find_unit(uoff, units, s);
        const int u_last = find_unit(uoff, units, e - 1);
        float* region = p.partials + (size_t)ph * p.phase_floats;

        for (int u = u_first; u <= u_last; ++u) {
            const long long a = s > uoff[u] ? s : uoff[u];
            const long long bnd = e < uoff[u + 1] ? e : uoff[u + 1];
            if (a >= bnd) continue;
            attend_unit<D, NB, C::kWarps, C::kHalves>(A, u, uinfo[u].x, items, s, a, bnd, stages, ms,
                                                     ls, region + ((size_t)blockIdx.x + u) * rs);
            const int first_cta = cta_of(uoff[u], T, n_cta);
            if (blockIdx.x == first_cta && tid == 0)
                rr2[2 * u + ph] = make_int2(first_cta, cta_of(uoff[u + 1] - 1, T, n_cta));
            __syncthreads();   // Ow / ms / ls and the page buffers are reused next
        }
    }
}

template <int D>
cudaError_t launch_combine_t(const DecodeParams& p, cudaStream_t st) {
    const int units = p.s.B * p.s.Hkv;
    const int col_blocks = (p.s.G * D / 4 + kCombineCols - 1) / kCombineCols;
    return launch_pdl(combine_kernel<D>, dim3(col_blocks, units), dim3(256), 0, st, p);
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
    return launch_combine_t<D>(p, st);
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

cudaError_t launch_combine(const DecodeParams& p, cudaStream_t st) {
    switch (p.s.D) {
        case 64: return launch_combine_t<64>(p, st);
        case 128: return launch_combine_t<128>(p, st);
        case 256: return launch_combine_t<256>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

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
