// attend.cu -- the top-k selection and the sparse decode in one launch
// (csa_sparse_attention), after the scoring kernel.
//
// Combined sparse attention ("Accelerating Long-Context Decoding in
// Large-Scale Hybrid LLMs Without Retraining", abstract; "Methodology": the
// Quest-style top-k pages) attends, per (sequence, kv-head) unit, to the
// prefix and window tokens and to the tokens of the k best-scoring candidate
// pages.  Split into separate launches, the part after the selection is a
// chain of dependent round trips (counts, page lists, page table, K/V) plus a
// launch; here it shrinks to the page table and the K/V loads.
//
// The grid holds two roles, both in clusters of 8 CTAs of 8 warps:
//   - selection clusters, one per unit (the first 8 * units CTAs): after the
//     dependency wait (the scores) the cluster selects the unit's top-k pages
//     (the cluster radix select of select_core.cuh), each CTA receives an
//     even share of the selected pages, in ascending order, through
//     distributed shared memory, and its 8 warps attend over that share: the
//     pages' tokens outside prefix and window (a selected boundary page keeps
//     its prefix/window tokens in the other role).  Every CTA writes one
//     partial record of its unit (slot 8u + rank of the second record region).
//   - prefix/window CTAs (the rest: as many clusters as stay resident beside
//     the selection clusters): they attend over every unit's fixed list (the
//     pages holding prefix or window tokens, masked to those tokens),
//     flattened and split evenly, and never wait: nothing they read
//     is written by the scoring kernel, and by the time this grid starts the
//     kernels before the scoring kernel (the token append among them) have
//     finished.  They run while the scoring kernel ends and while the
//     clusters select, when DRAM would otherwise idle.
// Both roles end in one loop over the CTA's jobs (its units' item segments
// and record slots), so that the page loop appears once in the kernel.
// The combine kernel then merges each unit's records of both roles.
#include "attend_core.cuh"
#include "common.cuh"
#include "internal.h"
#include "select_core.cuh"

namespace csa {
namespace {

constexpr int kFusedUnits = 32;            // units the fused path serves
constexpr int kFusedItems = kClCap / kCl;  // work items of one CTA: its share of a unit's
                                           // selected pages (2048), or its prefix/window slice
constexpr int kFusedMinItems = 4 * 8;      // prefix/window pages per CTA, at least (16 measured slower)

template <int D, int NB>
struct FusedCfg {
    static constexpr int kWarps = 8;                    // == kClThreads / 32
    // K/V tile slots per warp: two keep two CTAs per SM at D <= 128 (three
    // slots, with smaller item lists, measured no faster); at D = 256 one CTA
    // fills the SM either way and a third slot fits
    static constexpr int kHalves = D == 256 ? 3 : 2;
    using Tile = TileCfg<D, NB, kWarps, kHalves>;
    static constexpr size_t kItems = (size_t)kFusedItems * 8;
    static constexpr size_t kUnits = (size_t)(kFusedUnits + 1) * 4 + (size_t)kFusedUnits * 4;
    static constexpr size_t kSmem = 1024 /* alignment slack */ + Tile::kStageArea + Tile::kMl +
                                    kItems + kFusedItems * 4 /* share */ + kUnits;
};
static_assert(kClThreads == 256, "the fused kernel runs 8 warps per CTA");
static_assert(FusedCfg<256, 2>::kSmem + sizeof(ClShared) + 1024 <= 232448,
              "one fused CTA fits an SM at D = 256");
static_assert(2 * (FusedCfg<128, 1>::kSmem + sizeof(ClShared) + 1024) <= 233472,
              "two fused CTAs fit an SM at D <= 128");

template <int D, int NB>
__global__ void __cluster_dims__(kCl, 1, 1)
    __launch_bounds__(kClThreads, (D <= 128 && NB == 1) ? 2 : 1) fused_kernel(FusedParams P) {
    using C = FusedCfg<D, NB>;
    using T = typename C::Tile;
    __shared__ ClShared sh;
    // this CTA's work: per job a unit, its segment [a, b) of the items, the
    // sequence length and the record slot (one attention call site for both
    // roles keeps one copy of the page loop in the instruction stream)
    __shared__ int job_u[kFusedUnits], job_a[kFusedUnits], job_b[kFusedUnits],
        job_len[kFusedUnits];
    __shared__ float* job_rec[kFusedUnits];
    __shared__ int n_jobs;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzled page buffers need 1024-byte alignment in the shared window
    uint8_t* stages = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* ms = reinterpret_cast<float*>(stages + T::kStageArea);
    float* ls = ms + C::kWarps * T::kHeads;
    int2* items = reinterpret_cast<int2*>(ls + C::kWarps * T::kHeads);
    int* share = reinterpret_cast<int*>(items + kFusedItems);
    int* uoff = share + kFusedItems;
    int* ulen = uoff + kFusedUnits + 1;

    const DecodeParams& p = P.d;
    const int units = p.s.B * p.s.Hkv;
    const int Hkv = p.s.Hkv, MP = p.s.MP, G = p.s.G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    AttendArgs A;
    A.q = p.q;
    A.k_cache = p.k_cache;
    A.v_cache = p.v_cache;
    A.Hq = p.s.Hq;
    A.Hkv = Hkv;
    A.G = G;
    A.prefix = p.prefix;
    A.window = p.window;
    A.scale_log2 = p.scale_log2;
    const size_t rs = record_stride(G, D);
    int2* rr2 = reinterpret_cast<int2*>(p.rec_range);   // [unit][role]: first, last slot
    const int n_sel_ctas = kCl * units;

    if ((int)blockIdx.x >= n_sel_ctas) {
        // ------------------------------------------- prefix/window role
        // work slot of this CTA: rank-major over the role's clusters (n0 is
        // a multiple of 8), so that the slots in use, the first n_cta, fall
        // in as many clusters, and so SMs, as there are slots
        const int n0 = (int)gridDim.x - n_sel_ctas, rel = (int)blockIdx.x - n_sel_ctas;
        const int c0 = (rel % kCl) * (n0 / kCl) + rel / kCl;
        for (int u = tid; u < units; u += kClThreads) {
            int L = p.seq_lens[u / Hkv];
            if (L < 0 || L > MP * kPage) L = 0;          // flagged by the scoring kernel
            ulen[u] = L;
            uoff[u] = fixed_list(seq_geom(L, p.prefix, p.window), false).total();
        }
        __syncthreads();
        if (warp == 0) {   // exclusive scan (units <= 32: one warp step)
            const int v = lane < units ? uoff[lane] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane < units) uoff[lane] = incl - v;
            if (lane == 31) uoff[units] = incl;
        }
        __syncthreads();
        const long long T0 = uoff[units];
        long long want = (T0 + kFusedMinItems - 1) / kFusedMinItems;
        if (want < 1) want = 1;
        const int n_cta = (int)(want < (long long)n0 ? want : n0);
        const long long s = c0 < n_cta ? T0 * c0 / n_cta : T0;
        const long long e = c0 < n_cta ? T0 * (c0 + 1) / n_cta : T0;
        if (c0 == 0) {   // units without prefix/window pages: no records
            for (int u = tid; u < units; u += kClThreads)
                if (uoff[u + 1] == uoff[u]) rr2[2 * u] = make_int2(0, -1);
        }
        if (s >= e) return;
        // jobs: the units of the slice, items indexed from s
        if (tid == 0) {
            const int u_first = find_unit(uoff, units, s);
            const int u_last = find_unit(uoff, units, e - 1);
            int nj = 0;
            for (int u = u_first; u <= u_last; ++u) {
                const long long a = s > uoff[u] ? s : uoff[u];
                const long long bnd = e < uoff[u + 1] ? e : uoff[u + 1];
                if (a >= bnd) continue;
                job_u[nj] = u;
                job_a[nj] = (int)(a - s);
                job_b[nj] = (int)(bnd - s);
                job_len[nj] = ulen[u];
                job_rec[nj] = p.partials + ((size_t)c0 + u) * rs;
                ++nj;
                const int first = cta_of(uoff[u], T0, n_cta);
                if (c0 == first) rr2[2 * u] = make_int2(first, cta_of(uoff[u + 1] - 1, T0, n_cta));
            }
            n_jobs = nj;
        }
        for (long long x = s + tid; x < e; x += kClThreads) {
            const int u = find_unit(uoff, units, x);
            const SeqGeom sg = seq_geom(ulen[u], p.prefix, p.window);
            int page = 0, mask = kMaskAll;
            fixed_item(sg, fixed_list(sg, false), (int)(x - uoff[u]), page, mask);
            int phys = p.page_table[(size_t)(u / Hkv) * MP + page];
            if (phys < 0 || phys >= p.s.NPG) {
                latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
                phys = -1;
            }
            items[x - s] = make_int2(phys, page * 4 + mask);
        }
    } else {
        // ----------------------------------------------- selection role
        cg::cluster_group cl = cg::this_cluster();
        const int rank = (int)cl.block_rank();
        const int u = (int)blockIdx.x / kCl;
        const int b = u / Hkv;
        int L = p.seq_lens[b];
        if (L < 0 || L > MP * kPage) L = 0;                  // flagged by the scoring kernel
        const SeqGeom sg = seq_geom(L, p.prefix, p.window);
        const int n = sg.c_hi - sg.c_lo;
        const int kk = P.k_pages < n ? P.k_pages : n;
        const int c_lo = sg.c_lo;
        const int lo = kk * rank / kCl, hi = kk * (rank + 1) / kCl;   // this CTA's share
        int32_t* out = P.sel + (size_t)u * p.s.max_sel;
        if (tid < G * D / 64) {     // this unit's queries (a caller input) into L1
            const uint16_t* qrow =
                p.q + ((size_t)b * p.s.Hq + (size_t)(u % Hkv) * G) * D + tid * 64;
            asm volatile("prefetch.global.L1 [%0];" ::"l"(qrow));
        }
        pdl_wait();                 // the scores, and the previous readers of sel
        pdl_launch_dependents();

        if (kk == n) {              // every candidate fits the budget
            for (int j = lo + tid; j < hi; j += kClThreads) share[j - lo] = c_lo + j;
        } else if (kk > 0) {
            uint32_t kmin, kmax;
            key_range(P.keyrange[u], kmin, kmax);
            // only shared-memory stores before the barrier (its release then
            // waits for no global store); each CTA writes its share of the
            // output list afterwards
            cluster_select(cl, sh, P.scores_ws + (size_t)u * MP + c_lo, n, kk, kmin, kmax,
                           [&](int pos, int i) {
                               const int dst = ((pos + 1) * kCl + kk - 1) / kk - 1;
                               int* d = cl.map_shared_rank(share, dst);
                               d[pos - kk * dst / kCl] = c_lo + i;
                           });
            cluster_sync_all();     // every share is complete; no remote access after this
        }
        if (rank == 0 && tid == 0) {   // every CTA read the key range before the last barrier
            P.n_sel[u] = kk;
            P.keyrange[u] = make_uint2(0u, 0u);
            rr2[2 * u + 1] = make_int2((kCl - 1) * u, (kCl - 1) * u + kCl - 1);   // slots 8u + r
        }
        __syncthreads();
        const int cnt = hi - lo;
        for (int j = tid; j < cnt; j += kClThreads) {
            const int page = share[j];
            out[lo + j] = page;
            int phys = p.page_table[(size_t)b * MP + page];
            if (phys < 0 || phys >= p.s.NPG) {
                latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
                phys = -1;
            }
            items[j] = make_int2(phys, page * 4 + kMaskRest);
        }
        if (tid == 0) {             // one job: the share (an empty one leaves an empty record)
            job_u[0] = u;
            job_a[0] = 0;
            job_b[0] = cnt;
            job_len[0] = L;
            job_rec[0] = p.partials + p.phase_floats + ((size_t)kCl * u + rank) * rs;
            n_jobs = 1;
        }
    }
    __syncthreads();
    for (int jb = 0; jb < n_jobs; ++jb)
        attend_unit<D, NB, C::kWarps, C::kHalves>(A, job_u[jb], job_len[jb], items, 0, job_a[jb],
                                                 job_b[jb], stages, ms, ls, job_rec[jb]);
}

template <int D, int NB>
cudaError_t launch_fused_t(const FusedParams& p, cudaStream_t st) {
    using C = FusedCfg<D, NB>;
    auto kern = fused_kernel<D, NB>;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)C::kSmem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    const int units = p.d.s.B * p.d.s.Hkv;
    const int grid = kCl * units + p.n0;
    cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kClThreads), C::kSmem, st, p);
    if (e != cudaSuccess) return e;
    return launch_combine(p.d, st);
}

// Clusters of the fused kernel that are resident at once on the current
// device (clusters of 8 must sit in one GPC, so this is below SMs x CTAs per
// SM / 8); 0 when the query fails.
template <int D, int NB>
int resident_clusters_t() {
    static int cache[64] = {0};   // per device: the count, or -1 after a failed query
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && cache[dev] != 0) return cache[dev] > 0 ? cache[dev] : 0;
    using C = FusedCfg<D, NB>;
    auto kern = fused_kernel<D, NB>;
    int n = 0;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmem);
    if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kCl * 64);
        cfg.blockDim = dim3(kClThreads);
        cfg.dynamicSmemBytes = C::kSmem;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (dev < 64) cache[dev] = n > 0 ? n : -1;
    return n > 0 ? n : 0;
}

int resident_clusters(const Shape& s) {
    const int nb = s.G > 8 ? 2 : 1;
    switch (s.D * 10 + nb) {
        case 641: return resident_clusters_t<64, 1>();
        case 642: return resident_clusters_t<64, 2>();
        case 1281: return resident_clusters_t<128, 1>();
        case 1282: return resident_clusters_t<128, 2>();
        case 2561: return resident_clusters_t<256, 1>();
        case 2562: return resident_clusters_t<256, 2>();
        default: return 0;
    }
}

// Least CTAs of the prefix/window role for a call: no slice may exceed the
// item capacity (every unit's fixed list holds at most ceil(prefix / 16) +
// ceil(window / 16) + 2 pages).
long long phase0_min_ctas(const Shape& s, long long prefix, long long window) {
    const long long units = (long long)s.B * s.Hkv;
    long long fixed = (prefix + kPage - 1) / kPage + (window + kPage - 1) / kPage + 2;
    if (fixed > (long long)s.MP + 2) fixed = (long long)s.MP + 2;
    return (units * fixed + kFusedItems - 1) / kFusedItems;
}

long long round_to_clusters(long long n0) {
    if (n0 < kCl) n0 = kCl;
    n0 = (n0 + kCl - 1) / kCl * kCl;
    return n0 < (1ll << 30) ? n0 : (1ll << 30);
}

}  // namespace

// The fused path serves up to 32 units, with at most kClCap candidates per
// unit (the cluster select's capacity) and at least one page to select.
bool fused_eligible(const Shape& s, int prefix, int window, int k_pages) {
    const long long n_max = (long long)s.MP - prefix / kPage - window / kPage;
    return k_pages > 0 && (long long)s.B * s.Hkv <= kFusedUnits && n_max <= kClCap;
}

// The most CTAs of the prefix/window role any call of the shape launches
// (for the workspace): what stays of two (or one) CTAs per SM beside the
// selection clusters, at least the item capacity's minimum, whole clusters.
int fused_phase0_ctas(const Shape& s) {
    const long long units = (long long)s.B * s.Hkv;
    const int per_sm = (s.D <= 128 && s.G <= 8) ? 2 : 1;
    const long long all = (long long)s.MP * kPage;
    long long n0 = (long long)per_sm * device_sm_count() - kCl * units;
    const long long need = phase0_min_ctas(s, all, all);
    return (int)round_to_clusters(n0 > need ? n0 : need);
}

// CTAs of the prefix/window role for a call: the clusters that stay resident
// beside the selection clusters (so that none of the role waits for a second
// wave), at least the call's item-capacity minimum, at most the workspace's
// count.
int fused_phase0_ctas(const Shape& s, long long prefix, long long window) {
    const long long units = (long long)s.B * s.Hkv;
    const long long most = fused_phase0_ctas(s);
    long long n0 = most;
    const int resident = resident_clusters(s);
    if (resident > units) {
        const long long fit = ((long long)resident - units) * kCl;
        if (fit < n0) n0 = fit;
    }
    const long long need = phase0_min_ctas(s, prefix, window);
    if (n0 < need) n0 = need;
    n0 = round_to_clusters(n0);
    return (int)(n0 < most ? n0 : most);
}

cudaError_t launch_fused(const FusedParams& p, cudaStream_t st) {
    const int nb = p.d.s.G > 8 ? 2 : 1;
    switch (p.d.s.D * 10 + nb) {
        case 641: return launch_fused_t<64, 1>(p, st);
        case 642: return launch_fused_t<64, 2>(p, st);
        case 1281: return launch_fused_t<128, 1>(p, st);
        case 1282: return launch_fused_t<128, 2>(p, st);
        case 2561: return launch_fused_t<256, 1>(p, st);
        case 2562: return launch_fused_t<256, 2>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
