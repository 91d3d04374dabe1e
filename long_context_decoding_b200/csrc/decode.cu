// decode.cu -- split-K flash decoding over the attended pages, with the
// cross-CTA merge fused in ("last CTA per unit combines").
//
// Combined sparse attention ("Accelerating Long-Context Decoding in
// Large-Scale Hybrid LLMs Without Retraining", abstract): every query head
// attends to a pinned prefix, a sliding window and the selected top-k pages.
// For (sequence b, kv-head g) the attended tokens are
//     A = { t < L : t < Pe  or  t >= L - We  or  page(t) selected }
// and for each of the G query heads of the group
//     out_h = sum_{t in A} softmax_t(scale * q_h . k_t) v_t .
// The dense layer (csa_decode_full) is the same kernel with every page
// selected.
//
// Work list.  Per unit the pages to read are, in order: the prefix-only
// pages [0, c_lo), the prefix boundary page c_lo when it is not selected but
// holds prefix tokens, the selected pages, the window boundary page c_hi - 1
// when it is not selected but holds window tokens, and the window-only pages
// [c_hi, np).  A token mask (t < L and (selected-page or t < Pe or
// t >= L - We)) makes the union token-exact with nothing counted twice.  The
// lists of all units are flattened and split evenly over a grid that fills
// every SM, so ragged lengths and budgets stay balanced.
//
// Per CTA: the page ids of its slice are resolved once into shared memory;
// a producer warp streams each page's K and V tile (16 tokens x D, bf16) with
// 2-D TMA tensor copies, 64 channels (128 bytes) per box, 128-byte swizzle,
// into a ring of stages tracked by mbarriers; four consumer warps take pages
// round-robin.  Per page a warp computes S^T = K Q^T (16 tokens x 8 heads)
// with mma.sync m16n8k16 (K fragments by ldmatrix, Q^T fragments resident
// in registers), masks it, runs the fp32 online softmax in the exp2 domain,
// turns P into the B operand with movmatrix, and accumulates
// O^T += V^T P^T with ldmatrix.trans fragments of V.  At the end of a unit
// the warps merge through shared memory; a unit split over several CTAs
// leaves one partial record (m, l, o) per CTA in the workspace, and the CTA
// that takes the unit's last ticket merges them and writes bf16 out and lse.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

template <int D, int NB>
struct DecCfg {
    static constexpr int kConsumers = 4;
    static constexpr int kThreads = 32 * (kConsumers + 1);
    static constexpr int kBoxes = D / 64;               // 64-channel TMA boxes per K (or V) page
    static constexpr int kHalf = kBoxes * 2048;         // bytes of one page's K (or V) tile
    static constexpr int kStageBytes = 2 * kHalf;
    static constexpr int kStages = D == 256 ? 4 : (D == 128 ? 8 : 16);
    // a stage's previous use must belong to the same consumer warp, so that a
    // parity wait can never be two phases ahead of the barrier
    static_assert(kStages % kConsumers == 0, "stages must be a multiple of consumers");
    static constexpr int kHeads = 8 * NB;               // query heads per CTA (padded)
    static constexpr int kMB = D / 16;                  // 16-channel blocks
    static constexpr size_t kOw = (size_t)kConsumers * kHeads * D * 4;
    static constexpr size_t kMl = (size_t)2 * kConsumers * kHeads * 4;
    static constexpr size_t kItems = (size_t)kDecodeItemCap * 8;
    static __host__ __device__ size_t smem_bytes(int units) {
        return 1024 /* alignment slack */ + (size_t)kStages * kStageBytes + kOw + kMl + kItems +
               unit_bytes(units) + 16 * (size_t)kStages;
    }
    // uoff [units + 1] | uinfo [units] (int2: seq_len, n_sel | n_blo << 30 | n_bhi << 31)
    static __host__ __device__ size_t unit_bytes(int units) {
        return (((size_t)(units + 1) * 4 + 15) & ~(size_t)15) + (size_t)units * 8;
    }
};

// What one unit reads, as counts of the five page groups of its work list.
struct UnitPlan {
    int b, g, L, Pe, We, np, c_lo, c_hi;
    int n_pre, n_blo, n_sel, n_bhi, n_win;
    const int32_t* sel;
    __device__ int total() const { return n_pre + n_blo + n_sel + n_bhi + n_win; }
};

__device__ UnitPlan make_plan(const DecodeParams& p, int u) {
    UnitPlan q;
    q.b = u / p.s.Hkv;
    q.g = u % p.s.Hkv;
    int L = p.seq_lens[q.b];
    if (L < 0 || L > p.s.MP * kPage) {
        latch_flag(p.flags, CSA_DEVFLAG_BAD_SEQ_LEN);
        L = 0;
    }
    const SeqGeom sg = seq_geom(L, p.prefix, p.window);
    q.L = L;
    q.Pe = sg.Pe;
    q.We = sg.We;
    q.np = sg.np;
    q.c_lo = sg.c_lo;
    q.c_hi = sg.c_hi;
    q.sel = nullptr;
    q.n_blo = q.n_sel = q.n_bhi = 0;
    if (p.dense || sg.c_lo == sg.c_hi) {     // every valid token is attended
        q.n_pre = sg.np;
        q.n_win = 0;
        return q;
    }
    q.n_pre = sg.c_lo;
    q.n_win = sg.np - sg.c_hi;
    int ns = p.n_sel[u];
    const int cap = p.s.max_sel < sg.c_hi - sg.c_lo ? p.s.max_sel : sg.c_hi - sg.c_lo;
    if (ns < 0 || ns > cap) {
        latch_flag(p.flags, CSA_DEVFLAG_BAD_SELECTION);
        ns = ns < 0 ? 0 : cap;
    }
    q.n_sel = ns;
    q.sel = p.sel + (size_t)u * p.s.max_sel;
    const int first = ns > 0 ? q.sel[0] : -1;
    const int last = ns > 0 ? q.sel[ns - 1] : -1;
    const bool lo_partial = (sg.Pe % kPage) != 0;
    const bool hi_partial = sg.We > 0 && ((L - sg.We) % kPage) != 0;
    q.n_blo = (lo_partial && first != sg.c_lo) ? 1 : 0;
    q.n_bhi = (hi_partial && last != sg.c_hi - 1 && !(sg.c_hi - 1 == sg.c_lo && q.n_blo)) ? 1 : 0;
    return q;
}

// The plan of unit u again, from the (seq_len, packed counts) kept in
// shared memory by the first pass: no global loads.
__device__ __forceinline__ UnitPlan cached_plan(const DecodeParams& p, int u, int2 info) {
    UnitPlan q;
    q.b = u / p.s.Hkv;
    q.g = u % p.s.Hkv;
    const SeqGeom sg = seq_geom(info.x, p.prefix, p.window);
    q.L = info.x;
    q.Pe = sg.Pe;
    q.We = sg.We;
    q.np = sg.np;
    q.c_lo = sg.c_lo;
    q.c_hi = sg.c_hi;
    q.n_sel = info.y & 0x3fffffff;
    q.n_blo = (info.y >> 30) & 1;
    q.n_bhi = (int)(((unsigned)info.y >> 31) & 1u);
    q.sel = p.sel ? p.sel + (size_t)u * p.s.max_sel : nullptr;
    if (p.dense || sg.c_lo == sg.c_hi) {
        q.n_pre = sg.np;
        q.n_win = 0;
    } else {
        q.n_pre = sg.c_lo;
        q.n_win = sg.np - sg.c_hi;
    }
    return q;
}

// Item j of a unit's list -> logical page and whether all its valid tokens
// are attended (else the prefix/window token mask applies).  Returns false
// for a selection entry that is out of range or out of order.
__device__ bool plan_item(const UnitPlan& q, int j, int& page, bool& whole) {
    if (j < q.n_pre) { page = j; whole = true; return true; }
    j -= q.n_pre;
    if (j < q.n_blo) { page = q.c_lo; whole = false; return true; }
    j -= q.n_blo;
    if (j < q.n_sel) {
        page = q.sel[j];
        whole = true;
        const bool in_range = page >= q.c_lo && page < q.c_hi;
        const bool ordered = j == 0 || q.sel[j - 1] < page;
        return in_range && ordered;
    }
    j -= q.n_sel;
    if (j < q.n_bhi) { page = q.c_hi - 1; whole = false; return true; }
    j -= q.n_bhi;
    page = q.c_hi + j;
    whole = true;
    return true;
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

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(4 * 32) : "memory");
}

// The CTA holding a unit's last ticket merges the unit's partial records
// (o relative to its own max m, with m and l) written by CTAs
// first .. last:  M = max_r m_r,  w_r = 2^(m_r - M),  out = sum_r w_r o_r /
// sum_r w_r l_r.  Records are read through L2 in chunks: the weights of a
// chunk go to shared memory first, then every thread sums its (head, channel)
// elements with independent loads.
template <int D>
__device__ void merge_records(const DecodeParams& p, int b, int g, int u, int first, int last,
                              size_t rec_stride, float* wsm, float* Msm, float* Lsm, int ctid) {
    const int G = p.s.G, Hq = p.s.Hq;
    const int nrec = last - first + 1;
    const float* base = p.partials + ((size_t)first + u) * rec_stride;
    // M and L per head: one warp per head, lanes over records
    const int warp = ctid >> 5, lane = ctid & 31;
    for (int h = warp; h < G; h += 4) {
        float m = -INFINITY;
        for (int r = lane; r < nrec; r += 32)
            m = fmaxf(m, __ldcg(base + (size_t)r * rec_stride + (size_t)h * (D + 2) + D));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int r = lane; r < nrec; r += 32) {
            const float* rc = base + (size_t)r * rec_stride + (size_t)h * (D + 2);
            const float mr = __ldcg(rc + D);
            l += mr == -INFINITY ? 0.f : __ldcg(rc + D + 1) * ex2(mr - m);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            Msm[h] = m;
            Lsm[h] = l;
        }
    }
    consumer_sync();
    constexpr int kPer = 8;                       // elements per thread and pass
    const int total = G * D;
    const int chunk = (4 * 8 * D) / G;            // records whose weights fit in wsm
    for (int e0 = 0; e0 < total; e0 += 128 * kPer) {
        float acc[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
        for (int r0 = 0; r0 < nrec; r0 += chunk) {
            const int rn = nrec - r0 < chunk ? nrec - r0 : chunk;
            for (int i = ctid; i < rn * G; i += 128) {
                const int r = r0 + i / G, h = i % G;
                const float mr = __ldcg(base + (size_t)r * rec_stride + (size_t)h * (D + 2) + D);
                wsm[i] = mr == -INFINITY ? 0.f : ex2(mr - Msm[h]);
            }
            consumer_sync();
            for (int r = 0; r < rn; ++r) {
                const float* rc = base + (size_t)(r0 + r) * rec_stride;
#pragma unroll
                for (int j = 0; j < kPer; ++j) {
                    const int idx = e0 + j * 128 + ctid;
                    if (idx < total) {
                        const int h = idx / D, c = idx % D;
                        acc[j] += __ldcg(rc + (size_t)h * (D + 2) + c) * wsm[r * G + h];
                    }
                }
            }
            consumer_sync();
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int idx = e0 + j * 128 + ctid;
            if (idx < total) {
                const int h = idx / D, c = idx % D;
                const float l = Lsm[h];
                const size_t oi = (size_t)b * Hq + (size_t)g * G + h;
                p.out[oi * D + c] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(l > 0.f ? acc[j] / l : 0.f));
                if (c == 0 && p.lse)
                    p.lse[oi] = l > 0.f ? (Msm[h] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            }
        }
    }
}

template <int D, int NB>
__global__ void __launch_bounds__(DecCfg<D, NB>::kThreads)
decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              DecodeParams p) {
    using C = DecCfg<D, NB>;
    static_assert(C::kConsumers == 4, "consumer_sync counts 4 warps");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzled TMA destinations need 1024-byte alignment in the shared window
    uint8_t* stages = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* Ow = reinterpret_cast<float*>(stages + (size_t)C::kStages * C::kStageBytes);
    float* ms = Ow + C::kConsumers * C::kHeads * D;
    float* ls = ms + C::kConsumers * C::kHeads;
    int2* items = reinterpret_cast<int2*>(ls + C::kConsumers * C::kHeads);
    int* uoff = reinterpret_cast<int*>(items + kDecodeItemCap);
    const int units = p.s.B * p.s.Hkv;
    int2* uinfo = reinterpret_cast<int2*>(reinterpret_cast<uint8_t*>(uoff) +
                                          (((size_t)(units + 1) * 4 + 15) & ~(size_t)15));
    uint64_t* full = reinterpret_cast<uint64_t*>(uinfo + units);
    uint64_t* empty = full + C::kStages;
    __shared__ int s_abort, s_last, s_issued;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hkv = p.s.Hkv, G = p.s.G, Hq = p.s.Hq;
    if (tid == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    // the selection, the appended tokens and the previous users of the
    // workspace belong to earlier kernels
    pdl_wait();
    pdl_launch_dependents();

    // ---- per-unit list lengths and their exclusive scan
    for (int u = tid; u < units; u += C::kThreads) {
        const UnitPlan q = make_plan(p, u);
        uoff[u] = q.total();
        uinfo[u] = make_int2(q.L, q.n_sel | (q.n_blo << 30) | (q.n_bhi << 31));
    }
    if (tid == 0) {
        s_abort = 0;
        s_issued = 0;
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
    // partition over at most T CTAs so that every participating CTA owns at
    // least one item: the merge counts every CTA between a unit's first and
    // last one
    const int n_cta = (int)(T < (long long)gridDim.x ? (T > 0 ? T : 1) : gridDim.x);
    const long long s = blockIdx.x < (unsigned)n_cta ? T * blockIdx.x / n_cta : T;
    const long long e = blockIdx.x < (unsigned)n_cta ? T * (blockIdx.x + 1) / n_cta : T;

    // units with nothing to attend (empty sequences): out = 0, lse = -inf
    if (blockIdx.x == 0) {
        for (int u = 0; u < units; ++u) {
            if (uoff[u + 1] != uoff[u]) continue;
            const int b = u / Hkv, g = u % Hkv;
            for (int i = tid; i < G * D; i += C::kThreads) {
                const int h = i / D, c = i % D;
                p.out[((size_t)b * Hq + (size_t)g * G + h) * D + c] = 0;
                if (c == 0 && p.lse) p.lse[(size_t)b * Hq + (size_t)g * G + h] = -INFINITY;
            }
        }
    }
    if (s >= e) return;

    // ---- resolve the physical page of every item of this CTA's slice
    for (long long x = s + tid; x < e; x += C::kThreads) {
        const int u = find_unit(uoff, units, x);
        const UnitPlan q = cached_plan(p, u, uinfo[u]);
        int page = 0;
        bool whole = true;
        int phys = -1;
        if (!plan_item(q, (int)(x - uoff[u]), page, whole)) {
            latch_flag(p.flags, CSA_DEVFLAG_BAD_SELECTION);
        } else {
            phys = p.page_table[(size_t)q.b * p.s.MP + page];
            if (phys < 0 || phys >= p.s.NPG) {
                latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
                phys = -1;
            }
        }
        items[x - s] = make_int2(phys, page * 2 + (whole ? 1 : 0));
    }
    if (tid == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        fence_barrier_init();
    }
    __syncthreads();

    const int u_first = find_unit(uoff, units, s);
    const int u_last = find_unit(uoff, units, e - 1);

    if (warp == C::kConsumers) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            int u = u_first;
            for (long long x = s; x < e; ++x) {
                while (x >= uoff[u + 1]) ++u;
                const int i = (int)(x - s);
                const int st = i % C::kStages, r = i / C::kStages;
                if (r > 0 && !mbar_wait(&empty[st], (r - 1) & 1)) {
                    latch_flag(p.flags, CSA_DEVFLAG_TIMEOUT);
                    s_abort = 1;
                }
                if (*(volatile int*)&s_abort) break;
                const int2 it = items[i];
                if (it.x >= 0) {
                    const int row = (it.x * Hkv + (u % Hkv)) * kPage;
                    uint8_t* dst = stages + (size_t)st * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[st], C::kStageBytes);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                        tma_tile_g2s(dst + bx * 2048, &tmK, bx * 64, row, &full[st]);
                        tma_tile_g2s(dst + C::kHalf + bx * 2048, &tmV, bx * 64, row, &full[st]);
                    }
                } else {
                    mbar_arrive(&full[st]);
                }
                s_issued = i + 1;
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int gq = lane >> 2, tq = lane & 3;
        const int mi = lane >> 3, ri = lane & 7;
        // per-lane ldmatrix geometry (128-byte swizzle: chunk c of row r sits at c ^ (r & 7))
        const int k_tok = ri + ((mi & 1) << 3), k_half = mi >> 1;
        const int v_tok = ri + ((mi >> 1) << 3), v_half = mi & 1;
        const float sl2 = p.scale_log2;

        for (int u = u_first; u <= u_last; ++u) {
            const long long a = s > uoff[u] ? s : uoff[u];
            const long long bnd = e < uoff[u + 1] ? e : uoff[u + 1];
            if (a >= bnd) continue;
            const int b = u / Hkv, g = u % Hkv;
            int L = p.seq_lens[b];
            if (L < 0 || L > p.s.MP * kPage) L = 0;
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

            for (long long x = a; x < bnd; ++x) {
                const int i = (int)(x - s);
                if (i % C::kConsumers != warp) continue;
                const int st = i % C::kStages, r = i / C::kStages;
                if (!*(volatile int*)&s_abort && !mbar_wait(&full[st], r & 1)) {
                    if (lane == 0) latch_flag(p.flags, CSA_DEVFLAG_TIMEOUT);
                    s_abort = 1;
                }
                const int2 it = items[i];
                bool wrote = false;
                if (!*(volatile int*)&s_abort && it.x >= 0) {
                    const int page = it.y >> 1;
                    const bool whole = it.y & 1;
                    const uint32_t kbase = smem_u32(stages + (size_t)st * C::kStageBytes);
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
                    const bool in0 = t0 < L && (whole || t0 < Pe || t0 >= Lw);
                    const bool in1 = t1 < L && (whole || t1 < Pe || t1 >= Lw);
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
                    // ---- slots past the end of the sequence may hold anything:
                    // zero those V rows so that P = 0 cannot meet a NaN
                    if (page == sg.np - 1 && (L & (kPage - 1))) {
                        const int r0 = L & (kPage - 1);
                        for (int c = lane; c < C::kBoxes * 128; c += 32) {
                            const int row = (c >> 3) & 15;
                            if (row >= r0) {
                                const uint32_t za = vbase + (c >> 7) * 2048 + row * 128 + (c & 7) * 16;
                                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(za),
                                             "r"(0u)
                                             : "memory");
                            }
                        }
                        __syncwarp();
                        wrote = true;
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
                __syncwarp();
                if (lane == 0) {
                    if (wrote) fence_proxy_async_smem();
                    mbar_arrive(&empty[st]);
                }
            }

            // ---- merge the four warps of this CTA
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
            consumer_sync();

            const int first_cta = cta_of(uoff[u], T, n_cta);
            const int last_cta = cta_of(uoff[u + 1] - 1, T, n_cta);
            const bool alone = first_cta == last_cta;
            const int ctid = tid;                      // 0 .. 127
            const size_t rec_stride = (size_t)G * (D + 2);
            float* rec = p.partials + ((size_t)blockIdx.x + u) * rec_stride;
            for (int idx = ctid; idx < G * D; idx += 128) {
                const int h = idx / D, c = idx % D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < C::kConsumers; ++w) M = fmaxf(M, ms[w * C::kHeads + h]);
                float acc = 0.f, lsum = 0.f;
#pragma unroll
                for (int w = 0; w < C::kConsumers; ++w) {
                    const float mw = ms[w * C::kHeads + h];
                    const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
                    acc += Ow[((size_t)w * C::kHeads + h) * D + c] * f;
                    lsum += ls[w * C::kHeads + h] * f;
                }
                const size_t oi = ((size_t)b * Hq + (size_t)g * G + h);
                if (alone) {
                    const float val = lsum > 0.f ? acc / lsum : 0.f;
                    p.out[oi * D + c] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
                    if (c == 0 && p.lse)
                        p.lse[oi] = lsum > 0.f ? (M + __log2f(lsum)) * 0.69314718055994531f
                                               : -INFINITY;
                } else {
                    rec[(size_t)h * (D + 2) + c] = acc;
                    if (c == 0) {
                        rec[(size_t)h * (D + 2) + D] = M;
                        rec[(size_t)h * (D + 2) + D + 1] = lsum;
                    }
                }
            }
            if (!alone) {
                __threadfence();
                consumer_sync();
                if (ctid == 0) {
                    const unsigned prev = atomicAdd(&p.tickets[u], 1u);
                    s_last = prev == (unsigned)(last_cta - first_cta);
                }
                consumer_sync();
                if (s_last) {
                    __threadfence();
                    merge_records<D>(p, b, g, u, first_cta, last_cta, rec_stride, Ow, ms, ls,
                                     ctid);
                    if (ctid == 0) atomicExch(&p.tickets[u], 0u);
                }
            }
            consumer_sync();   // Ow / ms / ls are reused by the next unit
        }
    }
    __syncthreads();
    if (tid == 0 && s_abort) {    // bounded drain of copies still in flight
        const int n = s_issued;
        for (int st = 0; st < C::kStages && st < n; ++st) {
            const int last = st + ((n - 1 - st) / C::kStages) * C::kStages;
            mbar_wait(&full[st], (last / C::kStages) & 1);
        }
    }
}

template <int D, int NB>
cudaError_t launch_decode_t(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            cudaStream_t st) {
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
    return launch_pdl(decode_kernel<D, NB>, dim3(grid), dim3(C::kThreads), smem, st, tmK, tmV, p);
}

}  // namespace

// Resident CTAs of the decode kernel for this shape, times the SM count, and
// at least enough CTAs that no slice exceeds the per-CTA item capacity.
template <int D, int NB>
static int resident_per_sm(int units) {
    const size_t per_cta = DecCfg<D, NB>::smem_bytes(units) + 1024;   // + per-CTA reserve
    int n = (int)((size_t)(228 * 1024) / per_cta);
    if (n > 2) n = 2;
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

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          cudaStream_t st) {
    const int nb = p.s.G > 8 ? 2 : 1;
    switch (p.s.D * 10 + nb) {
        case 641: return launch_decode_t<64, 1>(p, tmK, tmV, st);
        case 642: return launch_decode_t<64, 2>(p, tmK, tmV, st);
        case 1281: return launch_decode_t<128, 1>(p, tmK, tmV, st);
        case 1282: return launch_decode_t<128, 2>(p, tmK, tmV, st);
        case 2561: return launch_decode_t<256, 1>(p, tmK, tmV, st);
        case 2562: return launch_decode_t<256, 2>(p, tmK, tmV, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
