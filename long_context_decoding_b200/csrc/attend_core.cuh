// attend_core.cuh -- the page-attention core shared by the decode kernel and
// the fused selection + decode kernel.
//
// For one (sequence b, kv-head g) unit and a slice of its work items (pages,
// each with a token mask) the W warps of a CTA compute the unnormalised
// attention of the G query heads of the group over the slice:
//     m_h = max_t s_t,  l_h = sum_t 2^(s_t - m_h),  o_h = sum_t 2^(s_t - m_h) v_t,
// with s_t = scale * log2(e) * q_h . k_t over the slice's attended tokens
// ("Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs Without
// Retraining", abstract: each head attends to its prefix, window and
// selected pages), and write it as one partial record (o, m, l) that the
// combine kernel merges with the unit's other records.
//
// Every warp streams its own pages (round-robin over the slice) with 16-byte
// cp.async copies into a private ring of HALVES slots, each holding the K or
// the V tile of one page (16 tokens x D), laid out with the 128-byte XOR
// swizzle (16-byte chunk c of token row r at c ^ (r & 7)) so that ldmatrix
// reads them without bank conflicts; rows past the end of the sequence are
// zero-filled by the copy itself.  The tiles are consumed in the order K0,
// V0, K1, V1, ... and a slot is refilled with the tile HALVES places ahead
// as soon as its tile has been used, so HALVES - 1 tiles stay in flight while
// the warp computes (the attention is bound by the bytes in flight).  Per page: S^T = K Q^T (16 tokens x 8
// heads, mma.sync m16n8k16 with K fragments from ldmatrix and Q^T fragments
// in registers), the token mask, the fp32 online softmax in the exp2 domain,
// P turned into the B operand by movmatrix, and O^T += V^T P^T with
// ldmatrix.trans fragments of V.  The warps then merge through shared memory.
#pragma once

#include "common.cuh"

namespace csa {

// ------------------------------------------------------------ work items
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
__host__ __device__ constexpr __forceinline__ size_t record_stride(int G, int D) {
    return ((size_t)G * D + 2 * G + 3) & ~(size_t)3;
}

// Issues the cp.async copies of one tile (K or V) of a page (16 tokens x D)
// into a swizzled slot; token rows >= rows_valid are zero-filled.
template <int D>
__device__ __forceinline__ void load_half(uint32_t buf, const uint16_t* t, int rows_valid,
                                          int lane) {
    constexpr int kChunksPerRow = D / 8;
    constexpr int kChunks = 16 * kChunksPerRow;
#pragma unroll
    for (int i = 0; i < kChunks / 32; ++i) {
        const int idx = i * 32 + lane;
        const int r = idx / kChunksPerRow, c16 = idx % kChunksPerRow;
        const uint32_t off = (c16 >> 3) * 2048 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
        cp_async_16(buf + off, t + (size_t)r * D + c16 * 8, r < rows_valid ? 16u : 0u);
    }
}

// Shared-memory footprint of the core for W warps with HALVES tile slots each.
template <int D, int NB, int W, int HALVES>
struct TileCfg {
    static_assert(HALVES >= 2, "a page's K and V tiles both fit the ring");
    static constexpr int kHalf = 32 * D;                // bytes of one page's K (or V) tile
    static constexpr int kHeads = 8 * NB;               // query heads per CTA (padded)
    static constexpr int kMB = D / 16;                  // 16-channel blocks
    static constexpr size_t kStageArea = (size_t)W * HALVES * kHalf;
    static constexpr size_t kOw = (size_t)W * kHeads * D * 4;   // aliases the stage area
    static_assert(kOw <= kStageArea, "the merge buffer lives in the stage area");
    static constexpr size_t kMl = (size_t)2 * W * kHeads * 4;  // per-warp m and l
};

struct AttendArgs {
    const uint16_t* q;
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    int Hq, Hkv, G, prefix, window;
    float scale_log2;
};

// Attends unit u (sequence length L) over the work items x in [a, bnd) of a
// CTA whose resolved items start at flattened index s (items[x - s] =
// (physical page or -1 to skip, page * 4 + mask)) and writes the CTA's
// partial record of the unit to rec.  Called by all W warps of the CTA; the
// stage area, ms and ls are free on entry and again on return.
template <int D, int NB, int W, int HALVES>
__device__ void attend_unit(const AttendArgs& A, int u, int L, const int2* items, long long s,
                            long long a, long long bnd, uint8_t* stages, float* ms, float* ls,
                            float* rec) {
    using T = TileCfg<D, NB, W, HALVES>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    // per-lane ldmatrix geometry (chunk c of row r sits at c ^ (r & 7))
    const int k_tok = ri + ((mi & 1) << 3), k_half = mi >> 1;
    const int v_tok = ri + ((mi >> 1) << 3), v_half = mi & 1;
    const float sl2 = A.scale_log2;
    const int G = A.G, Hkv = A.Hkv;
    const int b = u / Hkv, g = u % Hkv;
    const SeqGeom sg = seq_geom(L, A.prefix, A.window);
    const int Pe = sg.Pe, Lw = L - sg.We;
    const uint32_t wbuf = smem_u32(stages) + (uint32_t)(warp * HALVES * T::kHalf);
    float* Ow = reinterpret_cast<float*>(stages);      // reused after the page loop

    // Q^T as the B operand: b0 = q[head][16kb + 2tq, +1], b1 = +8
    uint32_t qf[T::kMB][NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int head = nb * 8 + gq;
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(
            A.q + ((size_t)b * A.Hq + (size_t)g * G + (head < G ? head : 0)) * D);
#pragma unroll
        for (int kb = 0; kb < T::kMB; ++kb) {
            qf[kb][nb][0] = head < G ? __ldg(qw + 8 * kb + tq) : 0u;
            qf[kb][nb][1] = head < G ? __ldg(qw + 8 * kb + 4 + tq) : 0u;
        }
    }
    float m[NB][2], l[NB][2], o[T::kMB][NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        m[nb][0] = m[nb][1] = -INFINITY;
        l[nb][0] = l[nb][1] = 0.f;
#pragma unroll
        for (int mb = 0; mb < T::kMB; ++mb)
            o[mb][nb][0] = o[mb][nb][1] = o[mb][nb][2] = o[mb][nb][3] = 0.f;
    }

    // ---- S^T = K Q^T for the page in the buffer at kbase, the mask and the
    // online softmax (exp2 domain); leaves P^T as B fragments in pb
    auto qk_softmax = [&](uint32_t kbase, int page, int mask, uint32_t (&pb)[NB][2]) {
        // two accumulator chains (even and odd k steps) at D <= 128, summed at
        // the end (at D = 256 the second chain's registers cost more than the
        // shorter chain saves)
        constexpr bool kTwo = D <= 128;
        float sacc[NB][4], sacc2[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[nb][i] = sacc2[nb][i] = 0.f;
#pragma unroll
        for (int kb = 0; kb < T::kMB; ++kb) {
            const int chunk = 2 * kb + k_half;
            const uint32_t addr =
                kbase + (chunk >> 3) * 2048 + k_tok * 128 + (((chunk & 7) ^ ri) << 4);
            uint32_t af[4];
            ldsm_x4(af, addr);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                if (kTwo && (kb & 1)) mma_bf16_16816(sacc2[nb], af, qf[kb][nb][0], qf[kb][nb][1]);
                else mma_bf16_16816(sacc[nb], af, qf[kb][nb][0], qf[kb][nb][1]);
            }
        }
        if constexpr (kTwo) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int i = 0; i < 4; ++i) sacc[nb][i] += sacc2[nb][i];
        }
        const int t0 = page * kPage + gq, t1 = t0 + 8;
        const bool f0 = t0 < Pe || t0 >= Lw, f1 = t1 < Pe || t1 >= Lw;
        const bool in0 = t0 < L && (mask == kMaskAll || (mask == kMaskFixed) == f0);
        const bool in1 = t1 < L && (mask == kMaskAll || (mask == kMaskFixed) == f1);
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
            for (int mb = 0; mb < T::kMB; ++mb) {
                o[mb][nb][0] *= al0;
                o[mb][nb][1] *= al1;
                o[mb][nb][2] *= al0;
                o[mb][nb][3] *= al1;
            }
            pb[nb][0] = movmatrix_trans(P0);
            pb[nb][1] = movmatrix_trans(P1);
        }
    };
    // ---- O^T += V^T P^T for the page in the buffer at vbase
    auto pv = [&](uint32_t vbase, const uint32_t (&pb)[NB][2]) {
#pragma unroll
        for (int mb = 0; mb < T::kMB; ++mb) {
            const int chunk = 2 * mb + v_half;
            const uint32_t addr =
                vbase + (chunk >> 3) * 2048 + v_tok * 128 + (((chunk & 7) ^ ri) << 4);
            uint32_t af[4];
            ldsm_x4_trans(af, addr);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                mma_bf16_16816(o[mb][nb], af, pb[nb][0], pb[nb][1]);
        }
    };

    // this warp's items of the segment: a + warp, a + warp + W, ...; tile h of
    // the warp is the K (h even) or V (h odd) tile of item a + warp + (h / 2) W
    const long long first = a + warp;
    const int n_items = first < bnd ? (int)((bnd - first + W - 1) / W) : 0;
    auto issue = [&](int h, uint32_t slot) {   // one cp.async group per tile, always
        if (h < 2 * n_items) {
            const int2 it = items[first + (long long)(h >> 1) * W - s];
            if (it.x >= 0) {
                const int page = it.y >> 2;
                const size_t tile = ((size_t)it.x * Hkv + g) * kPage * D;
                const int rows = L - page * kPage < kPage ? L - page * kPage : kPage;
                load_half<D>(slot, ((h & 1) ? A.v_cache : A.k_cache) + tile, rows, lane);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int h = 0; h < HALVES; ++h) issue(h, wbuf + (uint32_t)(h * T::kHalf));
    uint32_t pb[NB][2];
    int slot = 0;
    for (int h = 0; h < 2 * n_items; ++h) {
        cp_async_wait<HALVES - 1>();   // tile h has landed
        __syncwarp();
        const uint32_t buf = wbuf + (uint32_t)(slot * T::kHalf);
        const int2 it = items[first + (long long)(h >> 1) * W - s];
        if (it.x >= 0) {
            if (h & 1) pv(buf, pb);
            else qk_softmax(buf, it.y >> 2, it.y & 3, pb);
        }
        __syncwarp();                  // the slot is refilled next
        issue(h + HALVES, buf);
        slot = slot + 1 == HALVES ? 0 : slot + 1;
    }
    cp_async_wait<0>();

    // ---- merge the warps of this CTA (Ow aliases the page buffers): each
    // warp's O^T goes to Ow[warp][column][head] (the fragment pairs of two
    // heads as one 8-byte store), m and l to ms and ls
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
            ms[warp * T::kHeads + nb * 8 + 2 * tq] = m[nb][0];
            ms[warp * T::kHeads + nb * 8 + 2 * tq + 1] = m[nb][1];
            ls[warp * T::kHeads + nb * 8 + 2 * tq] = l[nb][0];
            ls[warp * T::kHeads + nb * 8 + 2 * tq + 1] = l[nb][1];
        }
#pragma unroll
        for (int mb = 0; mb < T::kMB; ++mb) {
            float* ow = Ow + ((size_t)warp * D + mb * 16 + gq) * T::kHeads + nb * 8 + 2 * tq;
            *reinterpret_cast<float2*>(ow) = make_float2(o[mb][nb][0], o[mb][nb][1]);
            *reinterpret_cast<float2*>(ow + 8 * T::kHeads) = make_float2(o[mb][nb][2], o[mb][nb][3]);
        }
    }
    __syncthreads();
    // per head: M = max over the warps, each warp's factor 2^(m_w - M) in
    // place of its m, and the sum of l_w times the factor
    if (tid < G) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) M = fmaxf(M, ms[w * T::kHeads + tid]);
        float lsum = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float mw = ms[w * T::kHeads + tid];
            const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
            ms[w * T::kHeads + tid] = f;
            lsum += ls[w * T::kHeads + tid] * f;
        }
        rec[(size_t)G * D + tid] = M;
        rec[(size_t)G * D + G + tid] = lsum;
    }
    __syncthreads();
    // ---- this CTA's partial record of the unit (merged by the combine
    // kernel): a thread sums one column of four heads over the warps
    const int hq = (G + 3) / 4;
    for (int idx = tid; idx < hq * D; idx += 32 * W) {
        const int c = idx % D, h0 = 4 * (idx / D);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float4 f = *reinterpret_cast<const float4*>(ms + w * T::kHeads + h0);
            const float4 v =
                *reinterpret_cast<const float4*>(Ow + ((size_t)w * D + c) * T::kHeads + h0);
            acc.x += v.x * f.x;
            acc.y += v.y * f.y;
            acc.z += v.z * f.z;
            acc.w += v.w * f.w;
        }
        rec[(size_t)h0 * D + c] = acc.x;
        if (h0 + 1 < G) rec[(size_t)(h0 + 1) * D + c] = acc.y;
        if (h0 + 2 < G) rec[(size_t)(h0 + 2) * D + c] = acc.z;
        if (h0 + 3 < G) rec[(size_t)(h0 + 3) * D + c] = acc.w;
    }
    __syncthreads();   // Ow / ms / ls and the page buffers are reused next
}

}  // namespace csa
