// score.cu -- Quest page scores from the page metadata alone.
//
// "Methodology" (arxivlens analysis of "Accelerating Long-Context Decoding in
// Large-Scale Hybrid LLMs Without Retraining") and "The Move" (roboaidigest):
// the budgeted tokens are the query-aware top-k pages, Quest-style.  Quest's
// page score is the upper bound of q.k over the page's key box:
//     s_h(p) = sum_i max(q_i * max_{p,i}, q_i * min_{p,i})
//            = sum_i max(q_i, 0) * max_{p,i} + min(q_i, 0) * min_{p,i}
// (the two forms agree whenever min <= max).  The second form is a plain dot
// product of the page's [min | max] row with [q- | q+], so a tile of 16 pages
// against the 8 (or 16) query heads of a GQA group is a dense
// 16 x 2D x 8 contraction: it runs on the tensor cores (bf16 x bf16 products
// are exact in fp32; fp32 accumulation), and the kv-head score is the max
// over the group's heads.
//
// Data path.  The kernel streams 4*D bytes of metadata per candidate page
// from random physical pages and does ~2 flop per byte: it is HBM-bound, and
// what decides its speed is how many bytes are in flight.  Every warp of the
// grid loads its own tiles straight into the registers that feed the MMA:
// with the k index of the contraction permuted (the same permutation on the
// q side), lane (g, t) of a warp needs exactly the 16-byte chunks
// t, t+4, t+8, ... of rows g and g+8 of the tile, so a tile is 2D/16 plain
// 16-byte loads per lane (non-allocating in L1), with no shared-memory
// staging and no barriers.  Measured on B200 for 16 x 512-byte rows this
// sustains ~81% of the copy peak, where a TMA bulk copy per row (512 bytes)
// is limited by its per-copy issue cost to ~30%.
//   * the candidates of all (sequence, kv-head) units are flattened and split
//     evenly over a grid that fills every SM;
//   * each CTA copies its slice of the page table into shared memory once;
//   * warps take the CTA's 16-page tiles round-robin.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

template <int D, int NB>
struct ScoreCfg {
    static constexpr int kWarps = 8;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kKPairs = 2 * D / 32;        // 32-channel steps along [min | max]
    // page-table slice | 3 x [B + 1] ints
    static __host__ __device__ size_t smem_bytes(int B) {
        return (size_t)kScorePtCap * 4 + 3 * 4 * (size_t)(B + 1);
    }
};

struct TileInfo {
    int unit;      // b * Hkv + g
    int first;     // logical page of row 0
    int count;     // rows in use (1..16)
};

__device__ __forceinline__ uint32_t neg_part(uint32_t w) {   // min(q, 0) per bf16 half
    uint32_t r = 0;
    if (w & 0x00008000u) r |= (w & 0x0000ffffu);
    if (w & 0x80000000u) r |= (w & 0xffff0000u);
    return r;
}
__device__ __forceinline__ uint32_t pos_part(uint32_t w) {   // max(q, 0) per bf16 half
    uint32_t r = 0;
    if (!(w & 0x00008000u)) r |= (w & 0x0000ffffu);
    if (!(w & 0x80000000u)) r |= (w & 0xffff0000u);
    return r;
}

// Walks the CTA's range [x, e) of the flattened candidate list in tiles that
// never cross a (sequence, kv-head) unit.  One division at start-up; every
// step after that is a few integer adds.
struct TileWalker {
    int x, e;
    const int* seq_off;   // [B + 1]: first flattened index of sequence b
    const int* seq_n;     // candidates per (b, kv-head)
    const int* seq_clo;   // first candidate page of sequence b
    int Hkv, B;
    int b, g, idx;        // unit and candidate index of position x

    __device__ void start(int s, int end) {
        x = s;
        e = end;
        int lo = 0, hi = B;                   // last b with seq_off[b] <= x
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (seq_off[mid] <= x) lo = mid; else hi = mid;
        }
        b = lo;
        while (b < B - 1 && seq_n[b] == 0) ++b;
        const int n = seq_n[b] > 0 ? seq_n[b] : 1;
        const int rel = x - seq_off[b];
        g = rel / n;
        idx = rel - g * n;
    }
    // Next run of up to `cap` candidates inside one unit.
    __device__ bool next(TileInfo& t, int cap = 16) {
        if (x >= e) return false;
        const int n = seq_n[b];
        int cnt = n - idx;
        if (cnt > cap) cnt = cap;
        if (cnt > e - x) cnt = e - x;
        t.unit = b * Hkv + g;
        t.first = seq_clo[b] + idx;
        t.count = cnt;
        x += cnt;
        idx += cnt;
        if (idx == n) {
            idx = 0;
            if (++g == Hkv) {
                g = 0;
                do {
                    ++b;
                } while (b < B && seq_n[b] == 0);
            }
        }
        return true;
    }
};

// 16-byte load that does not allocate in L1 (the metadata is read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 4-byte load that does not allocate in L1 (the fp8 row exponent).
__device__ __forceinline__ int ld_stream_s32(const void* p) {
    int v;
    asm volatile("ld.global.nc.L1::no_allocate.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Two E4M3 values (bytes 0 and 1 of w) -> f16x2, exactly (hardware cvt).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"(w));
    return h2;
}
// 8 E4M3 channels -> 8 f16 channels in the order of a 16-byte chunk.
__device__ __forceinline__ uint4 e4m3x8_to_f16x8(uint32_t lo, uint32_t hi) {
    return make_uint4(e4m3x2_to_f16x2(lo), e4m3x2_to_f16x2(lo >> 16), e4m3x2_to_f16x2(hi),
                      e4m3x2_to_f16x2(hi >> 16));
}
// bf16x2 -> f16x2 (exact for |x| in [2^-17, 65504]; larger values saturate).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(bf16_hi(w)), "f"(bf16_lo(w)));
    return r;
}

// F8: the metadata is the fp8 copy (rows of 2D E4M3 bytes + a 16-byte trailer
// whose first int32 is the row's exponent e): 16 channels per 16-byte load,
// converted by the hardware to f16 (one instruction per two channels; the
// three-step route to bf16 made the conversions the bottleneck), multiplied
// with q in f16 on the tensor cores (products exact in fp32; q is exact in
// f16 for |q| >= 2^-17), and the row's sums scaled by 2^e.
template <int D, int NB, bool F8>
__global__ void __launch_bounds__(ScoreCfg<D, NB>::kThreads,
                                  ((NB == 1 && !(F8 && D == 256)) || D == 64) ? 2 : 1)
score_kernel(ScoreParams p) {
    using C = ScoreCfg<D, NB>;
    extern __shared__ __align__(16) int smem_i[];
    int* pt = smem_i;
    int* seq_n = pt + kScorePtCap;
    int* seq_clo = seq_n + (p.s.B + 1);
    int* seq_off = seq_clo + (p.s.B + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.s.B, Hkv = p.s.Hkv, G = p.s.G, MP = p.s.MP;

    // Candidates per sequence (caller inputs only before the dependency wait).
    for (int b = tid; b < B; b += C::kThreads) {
        int L = p.seq_lens[b];
        if (L < 0 || L > MP * kPage) {
            latch_flag(p.flags, CSA_DEVFLAG_BAD_SEQ_LEN);
            L = 0;
        }
        const SeqGeom sg = seq_geom(L, p.prefix, p.window);
        seq_n[b] = sg.c_hi - sg.c_lo;
        seq_clo[b] = sg.c_lo;
    }
    __syncthreads();
    if (warp == 0) {   // exclusive scan of Hkv * n_b
        int carry = 0;
        for (int base = 0; base < B; base += 32) {
            const int b = base + lane;
            int v = b < B ? seq_n[b] * Hkv : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (b < B) seq_off[b] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) seq_off[B] = carry;
    }
    __syncthreads();
    const long long N = seq_off[B];
    const int s = (int)(N * blockIdx.x / gridDim.x), e = (int)(N * (blockIdx.x + 1) / gridDim.x);

    TileWalker walk;
    walk.seq_off = seq_off;
    walk.seq_n = seq_n;
    walk.seq_clo = seq_clo;
    walk.Hkv = Hkv;
    walk.B = B;
    if (s < e) {
        // page-table slice (the grid is sized so that e - s <= cap), run by run:
        // every run is a contiguous piece of one page-table row
        TileWalker fill = walk;
        fill.start(s, e);
        TileInfo run;
        int at = 0;
        while (fill.next(run, 1 << 30)) {
            const int32_t* src = p.page_table + (size_t)(run.unit / Hkv) * MP + run.first;
            for (int i = tid; i < run.count; i += C::kThreads) pt[at + i] = __ldg(src + i);
            at += run.count;
        }
    }
    // the metadata was written by the previous kernel on the stream
    pdl_wait();
    pdl_launch_dependents();
    __syncthreads();
    if (s >= e) return;

    const int gq = lane >> 2, tq = lane & 3;
    uint32_t qf[C::kKPairs][NB][4];          // B fragments of [q- | q+] for the current unit
    int cur_unit = -1;
    int kr_unit = -1;                        // key range of this warp's current unit
    uint32_t kr_nmin = 0u, kr_max = 0u;
    if constexpr (F8) {
        // registers of one tile: rows g and g+8 of the fp8 copy as kKPairs / 2
        // 16-byte chunks of 16 channels each (lane (g, t) reads bytes
        // [64 m + 16 t, +16): the channel groups kp = 2m, first 8 channels, and
        // kp = 2m + 1, last 8)
        constexpr int NL = C::kKPairs / 2;
        struct Loaded {
            TileInfo t;
            int x0;
            bool ok0, ok8;
            uint4 a[NL], b[NL];
            int e0, e8;
        };

        walk.start(s, e);
        int jn = 0;
        // this warp's next tile: every kWarps-th tile of the CTA's range
        auto next_tile = [&](Loaded& L) -> bool {
            while (walk.next(L.t)) {
                if ((jn++ % C::kWarps) == warp) {
                    L.x0 = walk.x - L.t.count - s;       // slice index of row 0
                    return true;
                }
            }
            return false;
        };
        auto issue = [&](Loaded& L) {
            const int g = L.t.unit % Hkv;
            // rows g and g+8 of the tile (clamped inside the tile; extra rows are dropped)
            const int r0 = gq < L.t.count ? gq : L.t.count - 1;
            const int r8 = gq + 8 < L.t.count ? gq + 8 : L.t.count - 1;
            const int p0 = pt[L.x0 + r0], p8 = pt[L.x0 + r8];
            L.ok0 = p0 >= 0 && p0 < p.s.NPG;
            L.ok8 = p8 >= 0 && p8 < p.s.NPG;
            constexpr size_t kRow = 2 * D + 16;
            const uint8_t* b0 = p.meta8 + ((size_t)(L.ok0 ? p0 : 0) * Hkv + g) * kRow;
            const uint8_t* b8 = p.meta8 + ((size_t)(L.ok8 ? p8 : 0) * Hkv + g) * kRow;
#pragma unroll
            for (int m = 0; m < NL; ++m) {
                L.a[m] = ld_stream_v4(b0 + 64 * m + 16 * tq);
                L.b[m] = ld_stream_v4(b8 + 64 * m + 16 * tq);
            }
            L.e0 = ld_stream_s32(b0 + 2 * D);
            L.e8 = ld_stream_s32(b8 + 2 * D);
        };
        auto process = [&](const Loaded& L) {
            const TileInfo& t = L.t;
            const int b = t.unit / Hkv, g = t.unit % Hkv;
            if (t.unit != cur_unit) {
                cur_unit = t.unit;
    #pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int head = nb * 8 + gq;
                    const uint32_t* qw = reinterpret_cast<const uint32_t*>(
                        p.q + ((size_t)b * p.s.Hq + (size_t)g * G + (head < G ? head : 0)) * D);
    #pragma unroll
                    for (int kp = 0; kp < C::kKPairs; ++kp) {
                        // channels ch0 .. ch0+7 of the [min | max] row; min pairs with q-
                        const int ch0 = 64 * (kp >> 1) + 16 * tq + 8 * (kp & 1);
                        const bool is_max = ch0 >= D;
                        const int qc = is_max ? ch0 - D : ch0;
    #pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint32_t v = head < G ? __ldg(qw + qc / 2 + w) : 0u;
                            const uint32_t part = is_max ? pos_part(v) : neg_part(v);
                            qf[kp][nb][w] = bf16x2_to_f16x2(part);
                        }
                    }
                }
            }
            float acc[NB][4];
    #pragma unroll
            for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
    #pragma unroll
            for (int kp = 0; kp < C::kKPairs; ++kp) {
                const uint4 va = L.a[kp >> 1], vb = L.b[kp >> 1];
                const uint4 ta = (kp & 1) ? e4m3x8_to_f16x8(va.z, va.w) : e4m3x8_to_f16x8(va.x, va.y);
                const uint4 tb = (kp & 1) ? e4m3x8_to_f16x8(vb.z, vb.w) : e4m3x8_to_f16x8(vb.x, vb.y);
                const uint32_t a0[4] = {ta.x, tb.x, ta.y, tb.y};
                const uint32_t a1[4] = {ta.z, tb.z, ta.w, tb.w};
    #pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_f16_16816(acc[nb], a0, qf[kp][nb][0], qf[kp][nb][1]);
                    mma_f16_16816(acc[nb], a1, qf[kp][nb][2], qf[kp][nb][3]);
                }
            }
            const float sc0 = ldexpf(1.f, L.e0), sc8 = ldexpf(1.f, L.e8);
    #pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                acc[nb][0] *= sc0;
                acc[nb][1] *= sc0;
                acc[nb][2] *= sc8;
                acc[nb][3] *= sc8;
            }
            // max over the group's heads: this lane holds heads 8nb + 2tq, +1
            float m0 = -INFINITY, m8 = -INFINITY;
    #pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int h = nb * 8 + 2 * tq;
                if (h < G) {
                    m0 = fmaxf(m0, acc[nb][0]);
                    m8 = fmaxf(m8, acc[nb][2]);
                }
                if (h + 1 < G) {
                    m0 = fmaxf(m0, acc[nb][1]);
                    m8 = fmaxf(m8, acc[nb][3]);
                }
            }
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
            m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 1));
            m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 2));
            const int row = tq == 0 ? gq : gq + 8;
            const bool has = tq < 2 && row < t.count;
            const bool ok = tq == 0 ? L.ok0 : L.ok8;
            const float v = ok ? (tq == 0 ? m0 : m8) : -INFINITY;
            if (has) {
                if (!ok) latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
                const size_t o = (size_t)t.unit * MP + t.first + row;
                p.scores_ws[o] = v;
                if (p.scores_out) p.scores_out[o] = v;
            }
            // the unit's key range for the selection (min kept as ~key, so that
            // both ends merge with atomicMax from a zeroed word), published once
            // per warp and unit: per-tile atomics on one word serialise in L2
            const uint32_t key = order_key(v);
            if (t.unit != kr_unit) {
                if (lane == 0 && kr_unit >= 0) {
                    atomicMax(&p.keyrange[kr_unit].x, kr_nmin);
                    atomicMax(&p.keyrange[kr_unit].y, kr_max);
                }
                kr_unit = t.unit;
                kr_nmin = kr_max = 0u;
            }
            kr_nmin = max(kr_nmin, __reduce_max_sync(0xffffffffu, has ? ~key : 0u));
            kr_max = max(kr_max, __reduce_max_sync(0xffffffffu, has ? key : 0u));
        };
        // two tiles in flight per warp: the next tile's loads go out before
        // the current tile is processed (the fp8 tile needs half the registers)
        Loaded A, Bt;
        bool ha = next_tile(A);
        if (ha) issue(A);
        while (ha) {
            const bool hb = next_tile(Bt);
            if (hb) issue(Bt);
            process(A);
            if (!hb) break;
            ha = next_tile(A);
            if (ha) issue(A);
            process(Bt);
        }
    } else {
        // bf16: one tile in flight per warp (its registers allow no more)
        walk.start(s, e);
        TileInfo t;
        for (int j = 0; walk.next(t); ++j) {
            if (j % C::kWarps != warp) continue;
            const int b = t.unit / Hkv, g = t.unit % Hkv;
            const int x0 = walk.x - t.count - s;           // slice index of row 0
            // rows g and g+8 of the tile (clamped inside the tile; extra rows are dropped)
            const int r0 = gq < t.count ? gq : t.count - 1;
            const int r8 = gq + 8 < t.count ? gq + 8 : t.count - 1;
            const int p0 = pt[x0 + r0], p8 = pt[x0 + r8];
            const bool ok0 = p0 >= 0 && p0 < p.s.NPG, ok8 = p8 >= 0 && p8 < p.s.NPG;
            const char* row0 = reinterpret_cast<const char*>(
                p.meta + ((size_t)(ok0 ? p0 : 0) * Hkv + g) * 2 * D) + 16 * tq;
            const char* row8 = reinterpret_cast<const char*>(
                p.meta + ((size_t)(ok8 ? p8 : 0) * Hkv + g) * 2 * D) + 16 * tq;
            uint4 xa[C::kKPairs], xb[C::kKPairs];
    #pragma unroll
            for (int kp = 0; kp < C::kKPairs; ++kp) {
                xa[kp] = ld_stream_v4(row0 + 64 * kp);
                xb[kp] = ld_stream_v4(row8 + 64 * kp);
            }
            if (t.unit != cur_unit) {
                cur_unit = t.unit;
    #pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int head = nb * 8 + gq;
                    const uint32_t* qw = reinterpret_cast<const uint32_t*>(
                        p.q + ((size_t)b * p.s.Hq + (size_t)g * G + (head < G ? head : 0)) * D);
    #pragma unroll
                    for (int kp = 0; kp < C::kKPairs; ++kp) {
                        // channels ch0 .. ch0+7 of the [min | max] row; min pairs with q-
                        const int ch0 = 32 * kp + 8 * tq;
                        const bool is_max = ch0 >= D;
                        const int qc = is_max ? ch0 - D : ch0;
    #pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint32_t v = head < G ? __ldg(qw + qc / 2 + w) : 0u;
                            qf[kp][nb][w] = is_max ? pos_part(v) : neg_part(v);
                        }
                    }
                }
            }
            float acc[NB][4];
    #pragma unroll
            for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
    #pragma unroll
            for (int kp = 0; kp < C::kKPairs; ++kp) {
                const uint32_t a0[4] = {xa[kp].x, xb[kp].x, xa[kp].y, xb[kp].y};
                const uint32_t a1[4] = {xa[kp].z, xb[kp].z, xa[kp].w, xb[kp].w};
    #pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_bf16_16816(acc[nb], a0, qf[kp][nb][0], qf[kp][nb][1]);
                    mma_bf16_16816(acc[nb], a1, qf[kp][nb][2], qf[kp][nb][3]);
                }
            }
            // max over the group's heads: this lane holds heads 8nb + 2tq, +1
            float m0 = -INFINITY, m8 = -INFINITY;
    #pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int h = nb * 8 + 2 * tq;
                if (h < G) {
                    m0 = fmaxf(m0, acc[nb][0]);
                    m8 = fmaxf(m8, acc[nb][2]);
                }
                if (h + 1 < G) {
                    m0 = fmaxf(m0, acc[nb][1]);
                    m8 = fmaxf(m8, acc[nb][3]);
                }
            }
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
            m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 1));
            m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 2));
            const int row = tq == 0 ? gq : gq + 8;
            const bool has = tq < 2 && row < t.count;
            const bool ok = tq == 0 ? ok0 : ok8;
            const float v = ok ? (tq == 0 ? m0 : m8) : -INFINITY;
            if (has) {
                if (!ok) latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
                const size_t o = (size_t)t.unit * MP + t.first + row;
                p.scores_ws[o] = v;
                if (p.scores_out) p.scores_out[o] = v;
            }
            // the unit's key range for the selection (min kept as ~key, so that
            // both ends merge with atomicMax from a zeroed word), published once
            // per warp and unit: per-tile atomics on one word serialise in L2
            const uint32_t key = order_key(v);
            if (t.unit != kr_unit) {
                if (lane == 0 && kr_unit >= 0) {
                    atomicMax(&p.keyrange[kr_unit].x, kr_nmin);
                    atomicMax(&p.keyrange[kr_unit].y, kr_max);
                }
                kr_unit = t.unit;
                kr_nmin = kr_max = 0u;
            }
            kr_nmin = max(kr_nmin, __reduce_max_sync(0xffffffffu, has ? ~key : 0u));
            kr_max = max(kr_max, __reduce_max_sync(0xffffffffu, has ? key : 0u));
        }
    }
    if (lane == 0 && kr_unit >= 0) {
        atomicMax(&p.keyrange[kr_unit].x, kr_nmin);
        atomicMax(&p.keyrange[kr_unit].y, kr_max);
    }
}

template <int D, int NB, bool F8>
cudaError_t launch_score_t(const ScoreParams& p, cudaStream_t st) {
    using C = ScoreCfg<D, NB>;
    auto kern = score_kernel<D, NB, F8>;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)C::smem_bytes(kMaxUnits));
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    const size_t smem = C::smem_bytes(p.s.B);
    const long long ub = (long long)p.s.B * p.s.Hkv * p.s.MP;
    long long grid = 2LL * device_sm_count();      // two resident CTAs of 8 warps per SM
    const long long need = (ub + kScorePtCap - 1) / kScorePtCap;
    if (need > grid) grid = need;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(C::kThreads), smem, st, p);
}

}  // namespace

cudaError_t launch_score(const ScoreParams& p, cudaStream_t st) {
    const int nb = p.s.G > 8 ? 2 : 1;
    switch (p.s.D * 10 + nb) {
        case 641: return p.meta8 ? launch_score_t<64, 1, true>(p, st)
                          : launch_score_t<64, 1, false>(p, st);
        case 642: return p.meta8 ? launch_score_t<64, 2, true>(p, st)
                          : launch_score_t<64, 2, false>(p, st);
        case 1281: return p.meta8 ? launch_score_t<128, 1, true>(p, st)
                          : launch_score_t<128, 1, false>(p, st);
        case 1282: return p.meta8 ? launch_score_t<128, 2, true>(p, st)
                          : launch_score_t<128, 2, false>(p, st);
        case 2561: return p.meta8 ? launch_score_t<256, 1, true>(p, st)
                          : launch_score_t<256, 1, false>(p, st);
        case 2562: return p.meta8 ? launch_score_t<256, 2, true>(p, st)
                          : launch_score_t<256, 2, false>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
