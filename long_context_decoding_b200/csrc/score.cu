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
// Data path.  The kernels stream one metadata row per candidate (page,
// kv-head) from random physical pages and do ~2 flop per byte: they are
// bound by memory, and on B200 the rate of random row requests (~12 G rows/s
// for rows of 256 to 512 bytes) matters as much as the bytes.  Three load
// paths, chosen per shape by measurement:
//   * direct (bf16 metadata, D <= 128): every warp loads its own tiles
//     straight into the registers that feed the MMA.  With the k index of the
//     contraction permuted (the same permutation on the q side), lane (g, t)
//     needs exactly the 16-byte chunks t, t+4, ... of rows g and g+8, so a
//     tile is 2D/16 plain 16-byte loads per lane, with no staging and no
//     barriers.
//   * ring (bf16 metadata at D = 256, and the fp8 copy of other shapes):
//     each warp copies whole rows of its tiles into a private shared-memory
//     ring with 16-byte cp.async (one 512-byte row per instruction), keeps
//     several tiles in flight, and reads a landed tile into MMA fragments
//     with ldmatrix.
//   * page-major (the fp8 copy at 4 or 8 kv-heads): the CTA copies whole
//     pages, all kv-heads' rows of a page as one contiguous run (one bulk
//     copy per page, counted on the stage's mbarrier), into a shared ring;
//     warp g scores kv-head g.
// All: the candidates of all (sequence, kv-head) units -- of all sequences,
// for the page-major path -- are flattened and split evenly over the grid;
// each CTA copies its slice of the page table into shared memory once,
// before the dependency wait.  A TMA bulk copy per
// row (512 bytes) is limited by its per-copy issue cost to ~30% of the copy
// peak on B200, so neither path uses one.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

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

// Four E4M3 values (the bytes of w) -> two f16x2: bytes 0, 1 to lo and 2, 3
// to hi, exactly (hardware cvt on each 16-bit half).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// mbarrier and bulk-copy wrappers (the page-major kernel's shared ring).
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ unsigned long long gtimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 2^e as a normal float, e clamped to [-126, 127] (built from its exponent bits).
__device__ __forceinline__ float pow2_normal(int e) {
    e = e < -126 ? -126 : (e > 127 ? 127 : e);
    return __int_as_float((e + 127) << 23);
}
// x * 2^e, exact while the result stays in the normal range, for e in
// [-252, 254] (two power-of-two factors, each a normal float).
__device__ __forceinline__ float scale_pow2(float x, int e) {
    const int e1 = e / 2;
    return x * pow2_normal(e1) * pow2_normal(e - e1);
}

// 16-byte load that does not allocate in L1 (the metadata is read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Walks a range [x, e) of the flattened candidate list in tiles that never
// cross a (sequence, kv-head) unit.  One division at start-up; every step
// after that is a few integer adds.
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

// Shared memory common to the kernels: page-table slice (cap entries) |
// 3 x [B + 1] ints.
__host__ __device__ __forceinline__ size_t score_common_bytes(int B, int cap = kScorePtCap) {
    return (size_t)cap * 4 + 12 * (size_t)(B + 1);
}

// The prologue of the kernels: candidates per sequence, their exclusive scan
// over (sequence, kv-head) -- or over sequences alone when Hkv is passed as 1
// (the page-major kernel, whose items are pages) -- this CTA's range [s, e)
// of the flattened list and its page-table slice (at most cap entries, which
// the grid guarantees) -- all from caller inputs,
// before the dependency wait -- then the wait (the metadata was written by
// the previous kernel on the stream).  Returns the walker template (range not
// started).
__device__ __forceinline__ TileWalker score_setup(const ScoreParams& p, int* smem_i, int& s,
                                                  int& e, int Hkv, int cap = kScorePtCap) {
    const int B = p.s.B, MP = p.s.MP;
    const int tid = threadIdx.x, lane = tid & 31, nthr = blockDim.x;
    int* pt = smem_i;
    int* seq_n = pt + cap;
    int* seq_clo = seq_n + (B + 1);
    int* seq_off = seq_clo + (B + 1);
    for (int b = tid; b < B; b += nthr) {
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
    if (tid < 32) {   // exclusive scan of Hkv * n_b
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
    s = (int)(N * blockIdx.x / gridDim.x);
    e = (int)(N * (blockIdx.x + 1) / gridDim.x);

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
            for (int i = tid; i < run.count; i += nthr) pt[at + i] = __ldg(src + i);
            at += run.count;
        }
    }
    pdl_wait();
    pdl_launch_dependents();
    __syncthreads();
    return walk;
}

// The unit's key range for the selection: each lane keeps the largest ~key
// (the minimum, complemented so that both ends merge with atomicMax from a
// zeroed word) and the largest key of its rows; the warp reduces them and
// publishes once per warp and unit (per-tile atomics on one word serialise
// in L2).  Called by whole warps.
struct KeyRange {
    int unit = -1;
    uint32_t nmin = 0u, max = 0u;
    __device__ void flush(const ScoreParams& p, int lane) {
        const uint32_t n = __reduce_max_sync(0xffffffffu, nmin);
        const uint32_t m = __reduce_max_sync(0xffffffffu, max);
        if (lane == 0 && unit >= 0) {
            atomicMax(&p.keyrange[unit].x, n);
            atomicMax(&p.keyrange[unit].y, m);
        }
    }
};

// Tile epilogue of both kernels.  acc holds the MMA results (rows g, g+8 x
// heads 8 nb + 2t, +1); the kv-head score of a row is the max over the
// group's heads.  Rows with a bad page id score -inf and raise the flag.
template <int NB>
__device__ __forceinline__ void score_store(const ScoreParams& p, const TileInfo& t,
                                            const float (&acc)[NB][4], bool ok0, bool ok8,
                                            KeyRange& kr, int lane) {
    const int gq = lane >> 2, tq = lane & 3, G = p.s.G;
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
        const size_t o = (size_t)t.unit * p.s.MP + t.first + row;
        p.scores_ws[o] = v;
        if (p.scores_out) p.scores_out[o] = v;
    }
    const uint32_t key = order_key(v);
    if (t.unit != kr.unit) {
        kr.flush(p, lane);
        kr.unit = t.unit;
        kr.nmin = kr.max = 0u;
    }
    kr.nmin = max(kr.nmin, has ? ~key : 0u);
    kr.max = max(kr.max, has ? key : 0u);
}

// Whether row r of a tile starting at slice index x0 has a valid page id (ph:
// the id of row min(r, count - 1)).
__device__ __forceinline__ bool row_ok(const ScoreParams& p, const int* pt, int x0, int r,
                                       int count, int& ph) {
    ph = pt[x0 + (r < count ? r : count - 1)];
    return ph >= 0 && ph < p.s.NPG;
}

// ------------------------------------------------------------ direct path
// bf16 metadata; tiles round-robin over the CTA's warps: 4 CTAs of 4 warps
// per SM at D = 128 with up to 8 heads per group (measured 0.2-0.7 us faster
// per 256k layer's scoring call than 2 CTAs of 8 warps: smaller slices end
// closer together), else 2 (or 1) CTAs of 8 warps.
template <int D, int NB>
struct DirectCfg {
    static constexpr int kWarps = (NB == 1 && D == 128) ? 4 : 8;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kKPairs = 2 * D / 32;        // 32-channel steps along [min | max]
    static constexpr int kMinBlocks =
        (NB == 1 && D == 128) ? 4 : ((NB == 1 || D == 64) ? 2 : 1);
    static __host__ __device__ size_t smem_bytes(int B) { return score_common_bytes(B); }
};

template <int D, int NB>
__global__ void __launch_bounds__(DirectCfg<D, NB>::kThreads, DirectCfg<D, NB>::kMinBlocks)
score_direct_kernel(ScoreParams p) {
    using C = DirectCfg<D, NB>;
    extern __shared__ __align__(16) int smem_i[];
    int s, e;
    TileWalker walk = score_setup(p, smem_i, s, e, p.s.Hkv);
    if (s >= e) return;
    const int* pt = smem_i;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hkv = p.s.Hkv, G = p.s.G;
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t qf[C::kKPairs][NB][4];          // B fragments of [q- | q+] for the current unit
    int cur_unit = -1;
    KeyRange kr;

    walk.start(s, e);
    TileInfo t;
    for (int j = 0; walk.next(t); ++j) {
        if (j % C::kWarps != warp) continue;
        const int b = t.unit / Hkv, g = t.unit % Hkv;
        const int x0 = walk.x - t.count - s;           // slice index of row 0
        // rows g and g+8 of the tile (clamped inside the tile; extra rows are dropped)
        int p0, p8;
        const bool ok0 = row_ok(p, pt, x0, gq, t.count, p0);
        const bool ok8 = row_ok(p, pt, x0, gq + 8, t.count, p8);
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
        score_store<NB>(p, t, acc, ok0, ok8, kr, lane);
    }
    kr.flush(p, lane);
}

// B fragments of [q- | q+] for unit (b, g): MMA kk covers the 16 channels
// [16 kk, 16 kk + 16) of the [min | max] row (min pairs with q-).  F8: each
// head's q scaled by 2^-f and converted to f16 (see score_ring_kernel), with
// qexp[nb] = the exponents f of the heads of accumulator columns 2t, 2t + 1.
template <int D, int NB, bool F8>
__device__ __forceinline__ void load_q_frags(const ScoreParams& p, int b, int g, int lane,
                                             uint32_t (&qf)[D / 8][NB][2], int (&qexp)[NB][2]) {
    const int gq = lane >> 2, tq = lane & 3, G = p.s.G;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int head = nb * 8 + gq;
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(
            p.q + ((size_t)b * p.s.Hq + (size_t)g * G + (head < G ? head : 0)) * D);
#pragma unroll
        for (int kk = 0; kk < D / 8; ++kk) {
            const bool is_max = 16 * kk >= D;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // channel pair of k slots (2t, 2t+1) [h = 0] or (2t+8, 2t+9) [h = 1]
                const int ch = F8 ? 16 * kk + 4 * tq + 2 * h : 16 * kk + 8 * h + 2 * tq;
                const int qc = is_max ? ch - D : ch;
                const uint32_t v = head < G ? __ldg(qw + qc / 2) : 0u;
                qf[kk][nb][h] = is_max ? pos_part(v) : neg_part(v);
            }
        }
    }
    if constexpr (F8) {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            // largest |q| of head nb * 8 + g: this lane holds a quarter
            // of its channels (each once in the q- and once in the q+ half)
            float amax = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(qf[kk][nb][h])),
                                             fabsf(bf16_hi(qf[kk][nb][h]))));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const int f = amax > 0.f ? ilogbf(amax) - 14 : 0;
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w = qf[kk][nb][h];
                    uint32_t r;
                    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;"
                        : "=r"(r)
                        : "f"(scale_pow2(bf16_hi(w), -f)), "f"(scale_pow2(bf16_lo(w), -f)));
                    qf[kk][nb][h] = r;
                }
            // accumulator columns 2t and 2t + 1 belong to the heads
            // loaded by the lanes with g = 2t and g = 2t + 1
            qexp[nb][0] = __shfl_sync(0xffffffffu, f, 8 * tq);
            qexp[nb][1] = __shfl_sync(0xffffffffu, f, 8 * tq + 4);
        }
    }
}

// ------------------------------------------------------------ ring path
// Shared-memory rings, one per warp, of kStages tiles of 16 rows; each warp
// takes a contiguous 1/kWarps of the CTA's range.
template <int D, bool F8>
struct RingCfg {
    static constexpr int kRowBytes = F8 ? 2 * D + 16 : 4 * D;   // one (page, kv-head) row
    static constexpr int kRowChunks = kRowBytes / 16;
    // shared-memory row stride: an odd number of 16-byte chunks, so that the 8
    // row addresses of an ldmatrix phase fall in distinct banks
    static constexpr int kStride = F8 ? kRowBytes : kRowBytes + 16;
    static constexpr int kTileSmem = 16 * kStride;
    static constexpr int kTileChunks = 16 * kRowChunks;
    static constexpr int kCopyIters = (kTileChunks + 31) / 32;
    static constexpr int kWarps = kTileSmem > 12 * 1024 ? 2 : 4;
    static constexpr int kRingBudget = 70 * 1024;    // per CTA; two CTAs per SM
    static constexpr int kStagesFit = kRingBudget / (kWarps * kTileSmem);
    static constexpr int kStages = kStagesFit < 2 ? 2 : (kStagesFit > 6 ? 6 : kStagesFit);
    static constexpr int kThreads = 32 * kWarps;
    // common part | per-warp tile descriptors | per-warp rings
    static __host__ __device__ size_t desc_offset(int B) {
        return (score_common_bytes(B) + 15) & ~(size_t)15;
    }
    static __host__ __device__ size_t ring_offset(int B) {
        return (desc_offset(B) + (size_t)kWarps * kStages * 16 + 127) & ~(size_t)127;
    }
    static __host__ __device__ size_t smem_bytes(int B) {
        return ring_offset(B) + (size_t)kWarps * kStages * kTileSmem;
    }
};

// F8: the rows are the fp8 copy (2D E4M3 bytes + a 16-byte trailer whose
// first int32 is the row's exponent e).  An ldmatrix of 8 rows x 16 bytes
// gives lane (g, t) the four channels 4t .. 4t+3 of row g's 16-channel chunk;
// the hardware converts each pair to f16 (exact), the pairs become the k
// slots (2t, 2t+1) and (2t+8, 2t+9) of an f16 MMA whose q side takes the same
// channels.  Each head's q is scaled by 2^-f, f chosen so that its largest
// component lands in [2^14, 2^15), and converted to f16: exact for every
// component within 2^-31 of the head's largest (the rest, which move the sum
// by less than its fp32 rounding, round to the f16 grid), and never
// saturated, whatever the magnitude of q.  The row's sums are scaled back by
// 2^(e + f), exactly (two power-of-two factors: exact for |e + f| up to
// about 250, which covers every exponent bf16 keys and queries produce).
template <int D, int NB, bool F8>
__global__ void __launch_bounds__(RingCfg<D, F8>::kThreads, (F8 && D <= 128) ? 4 : 2)
score_ring_kernel(ScoreParams p) {
    using C = RingCfg<D, F8>;
    extern __shared__ __align__(16) int smem_i[];
    int s, e;
    TileWalker walk = score_setup(p, smem_i, s, e, p.s.Hkv);
    if (s >= e) return;
    const int* pt = smem_i;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = p.s.B, Hkv = p.s.Hkv;
    const int gq = lane >> 2;
    uint8_t* ring = reinterpret_cast<uint8_t*>(smem_i) + C::ring_offset(B) +
                    (size_t)warp * C::kStages * C::kTileSmem;
    int4* desc = reinterpret_cast<int4*>(reinterpret_cast<uint8_t*>(smem_i) + C::desc_offset(B)) +
                 warp * C::kStages;
    const uint8_t* mbase = F8 ? p.meta8 : reinterpret_cast<const uint8_t*>(p.meta);
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    // ldmatrix row address of this lane: matrices (rows 0-7 | rows 8-15) x (chunk c | c+1)
    const uint32_t lm_off = (uint32_t)(((lane & 7) + 8 * ((lane >> 3) & 1)) * C::kStride +
                                       16 * (lane >> 4));

    // copies of one tile's rows into ring stage `stage`; rows past the tile and
    // rows with a bad page id are zero-filled (their scores are dropped)
    auto issue = [&](const TileInfo& t, int x0, int stage) {
        // lane r < 16 resolves row r of the tile: its metadata row, or -1
        int row_of_lane = -1;
        if (lane < t.count) {
            const int ph = pt[x0 + lane];
            if (ph >= 0 && ph < p.s.NPG) row_of_lane = ph * Hkv + t.unit % Hkv;
        }
        const uint32_t dst = ring_s + (uint32_t)(stage * C::kTileSmem);
#pragma unroll
        for (int i = 0; i < C::kCopyIters; ++i) {
            const int id = i * 32 + lane;
            const int r = id / C::kRowChunks < 16 ? id / C::kRowChunks : 15;
            const int c = id - r * C::kRowChunks;
            const int mrow = __shfl_sync(0xffffffffu, row_of_lane, r);
            if (C::kTileChunks % 32 == 0 || id < C::kTileChunks) {
                const uint8_t* src =
                    mbase + (size_t)(mrow >= 0 ? mrow : 0) * C::kRowBytes + 16 * c;
                cp_async_16(dst + (uint32_t)(r * C::kStride + 16 * c), src, mrow >= 0 ? 16u : 0u);
            }
        }
    };

    // B fragments of [q- | q+] for the current unit: MMA kk covers the 16
    // channels [16 kk, 16 kk + 16) of the [min | max] row (min pairs with q-)
    uint32_t qf[D / 8][NB][2];
    int qexp[NB][2];       // F8: exponent f of the heads of accumulator columns 2t, 2t + 1
    int cur_unit = -1;
    KeyRange kr;

    auto process = [&](const TileInfo& t, int x0, int stage) {
        const int b = t.unit / Hkv, g = t.unit % Hkv;
        if (t.unit != cur_unit) {
            cur_unit = t.unit;
            load_q_frags<D, NB, F8>(p, b, g, lane, qf, qexp);
        }
        const uint32_t tile = ring_s + (uint32_t)(stage * C::kTileSmem) + lm_off;
        // two accumulator chains (even and odd MMAs), summed at the end
        float acc[NB][4], acc2[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nb][i] = acc2[nb][i] = 0.f;
        if constexpr (!F8) {
#pragma unroll
            for (int kk = 0; kk < D / 8; ++kk) {          // chunks 2kk (k 0-7), 2kk+1 (k 8-15)
                uint32_t a[4];
                ldsm_x4(a, tile + 32 * kk);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    if (kk & 1) mma_bf16_16816(acc2[nb], a, qf[kk][nb][0], qf[kk][nb][1]);
                    else mma_bf16_16816(acc[nb], a, qf[kk][nb][0], qf[kk][nb][1]);
                }
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[nb][i] += acc2[nb][i];
        } else {
#pragma unroll
            for (int kp = 0; kp < D / 16; ++kp) {         // chunks 2kp and 2kp+1, one MMA each
                uint32_t m[4];
                ldsm_x4(m, tile + 32 * kp);
                uint32_t a0[4], a1[4];
                e4m3x4_to_f16x2x2(m[0], a0[0], a0[2]);
                e4m3x4_to_f16x2x2(m[1], a0[1], a0[3]);
                e4m3x4_to_f16x2x2(m[2], a1[0], a1[2]);
                e4m3x4_to_f16x2x2(m[3], a1[1], a1[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_f16_16816(acc[nb], a0, qf[2 * kp][nb][0], qf[2 * kp][nb][1]);
                    mma_f16_16816(acc2[nb], a1, qf[2 * kp + 1][nb][0], qf[2 * kp + 1][nb][1]);
                }
            }
            const uint8_t* rows = ring + stage * C::kTileSmem;
            const int e0 = *reinterpret_cast<const int*>(rows + gq * C::kStride + 2 * D);
            const int e8 = *reinterpret_cast<const int*>(rows + (gq + 8) * C::kStride + 2 * D);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                acc[nb][0] = scale_pow2(acc[nb][0] + acc2[nb][0], e0 + qexp[nb][0]);
                acc[nb][1] = scale_pow2(acc[nb][1] + acc2[nb][1], e0 + qexp[nb][1]);
                acc[nb][2] = scale_pow2(acc[nb][2] + acc2[nb][2], e8 + qexp[nb][0]);
                acc[nb][3] = scale_pow2(acc[nb][3] + acc2[nb][3], e8 + qexp[nb][1]);
            }
        }
        int p0, p8;
        const bool ok0 = row_ok(p, pt, x0, gq, t.count, p0);
        const bool ok8 = row_ok(p, pt, x0, gq + 8, t.count, p8);
        score_store<NB>(p, t, acc, ok0, ok8, kr, lane);
    };

    // this warp's tiles: a contiguous 1/kWarps of the CTA's range, walked once;
    // copies run kStages - 1 tiles ahead of the processing, and each stage's
    // tile descriptor waits in shared memory
    const int ws = s + (int)((long long)(e - s) * warp / C::kWarps);
    const int we = s + (int)((long long)(e - s) * (warp + 1) / C::kWarps);
    walk.start(ws, we);
    auto issue_next = [&](int stage) -> bool {
        TileInfo t;
        if (!walk.next(t)) return false;
        const int x0 = walk.x - t.count - s;            // slice index of row 0
        if (lane == 0) desc[stage] = make_int4(t.unit, t.first, t.count, x0);
        issue(t, x0, stage);
        return true;
    };
    int pending = 0;
#pragma unroll
    for (int k = 0; k < C::kStages - 1; ++k) {
        if (issue_next(k)) ++pending;
        cp_async_commit();
    }
    for (int stage = 0; pending > 0; stage = stage + 1 == C::kStages ? 0 : stage + 1) {
        if (issue_next(stage == 0 ? C::kStages - 1 : stage - 1)) ++pending;   // the stage freed last
        cp_async_commit();
        cp_async_wait<C::kStages - 1>();
        __syncwarp();
        const int4 d = desc[stage];
        process(TileInfo{d.x, d.y, d.z}, d.w, stage);
        __syncwarp();
        --pending;
    }
    cp_async_wait<0>();
    kr.flush(p, lane);
}

// ------------------------------------------------------------ page-major fp8 path
// The fp8 rows of all kv-heads of a page lie side by side (Hkv x (2D + 16)
// bytes), so the CTA copies whole pages: one contiguous run per page instead
// of Hkv separate rows, which raises the rate of random requests for these
// short rows.  A CTA of HKV warps takes a range of the candidate pages of all
// sequences (flattened over sequences); each stage of its shared ring holds
// up to 16 consecutive candidate pages of one sequence, all kv-heads: one
// thread per page issues a bulk copy of the page's run into the page's slot
// (the slot stride an odd number of 16-byte chunks, so that ldmatrix reads
// the rows of one kv-head without bank conflicts), counted on the stage's
// mbarrier, and warp g scores the 16 x 2D tile of kv-head g with its own q
// fragments (the same MMAs, operand order and scaling as the ring kernel, so
// the scores agree with it bit for bit).  One CTA barrier per stage; the
// wait for a stage is bounded (20 ms, then CSA_DEVFLAG_TIMEOUT).  Bulk copies
// took the fp8 scoring call of a 256k layer from 22.0 to 21.2 us against
// 16-byte cp.async by every thread (fewer instructions per byte).
template <int D, int NB, int HKV>
struct PmCfg {
    static constexpr int kRowBytes = 2 * D + 16;             // one (page, kv-head) row
    static constexpr int kPageBytes = HKV * kRowBytes;       // one page, every kv-head
    static constexpr int kSlot = kPageBytes + 16;            // a page's slot in a stage (odd chunks)
    static constexpr int kStageSmem = 16 * kSlot;
    static constexpr int kWarps = HKV;
    static constexpr int kThreads = 32 * kWarps;
    // CTAs per SM: at 4 kv-heads and D <= 128, four (three stages each;
    // measured faster than two or three CTAs with deeper rings), three where
    // four would spill registers (16-head groups at D = 128); else two
    static constexpr int kCtasPerSm =
        (HKV == 4 && D <= 128) ? ((NB == 1 || D == 64) ? 4 : 3) : 2;
    static constexpr int kRingBudget = (kCtasPerSm == 4 ? 52 : 70) * 1024;   // per CTA
    static constexpr int kStagesFit = kRingBudget / kStageSmem;
    static constexpr int kStages = kStagesFit > 6 ? 6 : kStagesFit;
    static_assert((kSlot / 16) % 2 == 1, "odd slot stride: conflict-free ldmatrix");
    // page-table slice: a CTA's share of the candidate pages, at most
    // ceil(B * MP / grid) (the grid keeps it within kScorePtCap)
    static __host__ __device__ int pt_cap(int B, int MP, int grid) {
        const long long c = ((long long)B * MP + grid - 1) / grid;
        return (int)((c + 3) & ~3ll);
    }
    static __host__ __device__ size_t desc_offset(int B, int cap) {
        return (score_common_bytes(B, cap) + 15) & ~(size_t)15;
    }
    static __host__ __device__ size_t bar_offset(int B, int cap) {
        return desc_offset(B, cap) + (size_t)kStages * 16;
    }
    static __host__ __device__ size_t ring_offset(int B, int cap) {
        return (bar_offset(B, cap) + (size_t)kStages * 8 + 127) & ~(size_t)127;
    }
    static __host__ __device__ size_t smem_bytes(int B, int cap) {
        return ring_offset(B, cap) + (size_t)kStages * kStageSmem;
    }
};

template <int D, int NB, int HKV>
__global__ void __launch_bounds__(PmCfg<D, NB, HKV>::kThreads, PmCfg<D, NB, HKV>::kCtasPerSm)
    score_pm_kernel(ScoreParams p) {
    using C = PmCfg<D, NB, HKV>;
    static_assert(C::kStages >= 2, "two stages at least");
    extern __shared__ __align__(16) int smem_i[];
    const int cap = C::pt_cap(p.s.B, p.s.MP, (int)gridDim.x);
    int s, e;
    TileWalker walk = score_setup(p, smem_i, s, e, 1, cap);   // items: candidate pages
    if (s >= e) return;
    const int* pt = smem_i;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2;
    uint8_t* ring = reinterpret_cast<uint8_t*>(smem_i) + C::ring_offset(p.s.B, cap);
    int4* desc = reinterpret_cast<int4*>(reinterpret_cast<uint8_t*>(smem_i) +
                                         C::desc_offset(p.s.B, cap));
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    const uint32_t bar_s =
        (uint32_t)__cvta_generic_to_shared(reinterpret_cast<uint8_t*>(smem_i) + C::bar_offset(p.s.B, cap));
    const uint32_t lm_off = (uint32_t)(((lane & 7) + 8 * ((lane >> 3) & 1)) * C::kSlot +
                                       16 * (lane >> 4));
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < C::kStages; ++i) mbar_init(bar_s + 8 * i, 16);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // copies of a stage: the thread of page r (warp r % HKV, lane r / HKV)
    // copies the page's rows of every kv-head, one contiguous run, with one
    // bulk copy counted on the stage's barrier (16 arrivals); a slot past the
    // group or with a bad page id gets page 0 (its scores are dropped)
    const int my_r = lane < 16 / HKV ? warp + HKV * lane : -1;
    auto issue = [&](const TileInfo& t, int x0, int stage) {
        if (my_r >= 0) {
            const int ph = my_r < t.count ? pt[x0 + my_r] : -1;
            const bool ok = ph >= 0 && ph < p.s.NPG;
            const uint32_t bar = bar_s + 8 * stage;
            mbar_arrive_expect_tx(bar, (uint32_t)C::kPageBytes);
            bulk_g2s(ring_s + (uint32_t)(stage * C::kStageSmem + my_r * C::kSlot),
                     p.meta8 + (size_t)(ok ? ph : 0) * C::kPageBytes, (uint32_t)C::kPageBytes, bar);
        }
    };
    uint32_t parity = 0u, inflight = 0u;       // per stage: next phase parity, copies issued
    auto wait_stage = [&](int stage) -> bool {
        const uint32_t bar = bar_s + 8 * stage, par = (parity >> stage) & 1u;
        bool done = mbar_try_wait(bar, par);
        if (!done) {
            const unsigned long long t0 = gtimer_ns();
            while (!(done = mbar_try_wait(bar, par)) && gtimer_ns() - t0 < 20000000ull) {
            }
        }
        if (done) {
            parity ^= 1u << stage;
            inflight &= ~(1u << stage);
        }
        return done;
    };

    uint32_t qf[D / 8][NB][2];
    int qexp[NB][2];
    int cur_b = -1;
    KeyRange kr;
    const int g = warp;

    auto process = [&](const TileInfo& t, int x0, int stage) {
        const int b = t.unit;                               // walker over sequences
        if (b != cur_b) {
            cur_b = b;
            load_q_frags<D, NB, true>(p, b, g, lane, qf, qexp);
        }
        const uint32_t tile =
            ring_s + (uint32_t)(stage * C::kStageSmem + g * C::kRowBytes) + lm_off;
        float acc[NB][4], acc2[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nb][i] = acc2[nb][i] = 0.f;
#pragma unroll
        for (int kp = 0; kp < D / 16; ++kp) {
            uint32_t m[4];
            ldsm_x4(m, tile + 32 * kp);
            uint32_t a0[4], a1[4];
            e4m3x4_to_f16x2x2(m[0], a0[0], a0[2]);
            e4m3x4_to_f16x2x2(m[1], a0[1], a0[3]);
            e4m3x4_to_f16x2x2(m[2], a1[0], a1[2]);
            e4m3x4_to_f16x2x2(m[3], a1[1], a1[3]);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                mma_f16_16816(acc[nb], a0, qf[2 * kp][nb][0], qf[2 * kp][nb][1]);
                mma_f16_16816(acc2[nb], a1, qf[2 * kp + 1][nb][0], qf[2 * kp + 1][nb][1]);
            }
        }
        const uint8_t* rows = ring + stage * C::kStageSmem + g * C::kRowBytes;
        const int e0 = *reinterpret_cast<const int*>(rows + gq * C::kSlot + 2 * D);
        const int e8 = *reinterpret_cast<const int*>(rows + (gq + 8) * C::kSlot + 2 * D);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            acc[nb][0] = scale_pow2(acc[nb][0] + acc2[nb][0], e0 + qexp[nb][0]);
            acc[nb][1] = scale_pow2(acc[nb][1] + acc2[nb][1], e0 + qexp[nb][1]);
            acc[nb][2] = scale_pow2(acc[nb][2] + acc2[nb][2], e8 + qexp[nb][0]);
            acc[nb][3] = scale_pow2(acc[nb][3] + acc2[nb][3], e8 + qexp[nb][1]);
        }
        int p0, p8;
        const bool ok0 = row_ok(p, pt, x0, gq, t.count, p0);
        const bool ok8 = row_ok(p, pt, x0, gq + 8, t.count, p8);
        score_store<NB>(p, TileInfo{b * HKV + g, t.first, t.count}, acc, ok0, ok8, kr, lane);
    };

    walk.start(s, e);
    auto issue_next = [&](int stage) -> bool {
        TileInfo t;
        if (!walk.next(t)) return false;
        const int x0 = walk.x - t.count - s;                // slice index of page 0
        if (tid == 0) desc[stage] = make_int4(t.unit, t.first, t.count, x0);
        issue(t, x0, stage);
        inflight |= 1u << stage;
        return true;
    };
    int pending = 0;
#pragma unroll
    for (int k = 0; k < C::kStages - 1; ++k)
        if (issue_next(k)) ++pending;
    for (int stage = 0; pending > 0; stage = stage + 1 == C::kStages ? 0 : stage + 1) {
        const bool ok = wait_stage(stage);
        // every thread saw the stage land (or none continues); the previous
        // stage is free
        if (__syncthreads_or(!ok)) {
            latch_flag(p.flags, CSA_DEVFLAG_TIMEOUT);
            break;
        }
        if (issue_next(stage == 0 ? C::kStages - 1 : stage - 1)) ++pending;
        const int4 d = desc[stage];
        process(TileInfo{d.x, d.y, d.z}, d.w, stage);
        --pending;
    }
    // copies still in flight (only after a wait ran out): let them land, bounded
    for (int stage = 0; stage < C::kStages; ++stage)
        if (inflight & (1u << stage)) wait_stage(stage);
    kr.flush(p, lane);
}

// ------------------------------------------------------------ launch
// Raises a kernel's dynamic shared-memory limit to `bytes` unless done[dev]
// (the caller's per-kernel record of the largest limit set on each device)
// already covers it.
template <typename K>
cudaError_t ensure_smem(K kern, size_t bytes, size_t (&done)[64]) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && done[dev] >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e == cudaSuccess && dev < 64) done[dev] = bytes;
    return e;
}

// Grid: `per_sm` CTAs per SM, or more when the candidates would overflow the
// CTAs' page-table slices.
inline unsigned score_grid(const ScoreParams& p, int per_sm) {
    const long long ub = (long long)p.s.B * p.s.Hkv * p.s.MP;
    long long grid = (long long)per_sm * device_sm_count();
    const long long need = (ub + kScorePtCap - 1) / kScorePtCap;
    if (need > grid) grid = need;
    return (unsigned)(grid < 1 ? 1 : grid);
}

template <int D, int NB>
cudaError_t launch_direct(const ScoreParams& p, cudaStream_t st) {
    using C = DirectCfg<D, NB>;
    auto kern = score_direct_kernel<D, NB>;
    static size_t smem_set[64] = {0};
    const size_t smem = C::smem_bytes(p.s.B);
    cudaError_t e = ensure_smem(kern, smem, smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(score_grid(p, C::kMinBlocks)), dim3(C::kThreads), smem, st, p);
}

template <int D, int NB, bool F8>
cudaError_t launch_ring(const ScoreParams& p, cudaStream_t st) {
    using C = RingCfg<D, F8>;
    auto kern = score_ring_kernel<D, NB, F8>;
    static size_t smem_set[64] = {0};
    const size_t smem = C::smem_bytes(p.s.B);
    cudaError_t e = ensure_smem(kern, smem, smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(score_grid(p, 2)), dim3(C::kThreads), smem, st, p);
}

// bf16 metadata: the direct path at D <= 128, the ring at D = 256; the fp8
// copy: page-major at 4 or 8 kv-heads, else the ring.  Measured on B200: a
// 256k layer's scoring (D = 128, 262k rows) took 28.5 us direct against
// 30.2 us in the ring, and 90 against 100 us at four times the rows; the 64k
// layer (D = 256) took 37.4 us per layer step with the ring against 39.6 us
// direct; the fp8 copy, 24.7 us in the ring against 29.5 us direct, and one
// 256k layer's fp8 scoring call after an L2 flush 27.8 us page-major (four
// CTAs per SM) against 30.7 us in the ring.
template <int D, int NB, int HKV>
cudaError_t launch_pm(const ScoreParams& p, cudaStream_t st) {
    using C = PmCfg<D, NB, HKV>;
    auto kern = score_pm_kernel<D, NB, HKV>;
    static size_t smem_set[64] = {0};
    // kCtasPerSm CTAs per SM, or more when a CTA's share of the candidate
    // pages would overflow kScorePtCap
    const long long pages = (long long)p.s.B * p.s.MP;
    long long grid = (long long)C::kCtasPerSm * device_sm_count();
    const long long need = (pages + kScorePtCap - 1) / kScorePtCap;
    if (need > grid) grid = need;
    const size_t smem = C::smem_bytes(p.s.B, C::pt_cap(p.s.B, p.s.MP, (int)grid));
    cudaError_t e = ensure_smem(kern, smem, smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(C::kThreads), smem, st, p);
}

template <int D, int NB>
cudaError_t launch_score_d(const ScoreParams& p, cudaStream_t st) {
    if (p.meta8) {
        // whole pages of 4 or 8 kv-heads (not 8 at D = 256, whose stage
        // would not fit twice, nor 8 with 16-head groups, which spills)
        if (p.s.Hkv == 4) return launch_pm<D, NB, 4>(p, st);
        if constexpr (D <= 128 && NB == 1)
            if (p.s.Hkv == 8) return launch_pm<D, NB, 8>(p, st);
        return launch_ring<D, NB, true>(p, st);
    }
    if constexpr (D == 256) return launch_ring<D, NB, false>(p, st);
    else return launch_direct<D, NB>(p, st);
}

}  // namespace

cudaError_t launch_score(const ScoreParams& p, cudaStream_t st) {
    const int nb = p.s.G > 8 ? 2 : 1;
    switch (p.s.D * 10 + nb) {
        case 641: return launch_score_d<64, 1>(p, st);
        case 642: return launch_score_d<64, 2>(p, st);
        case 1281: return launch_score_d<128, 1>(p, st);
        case 1282: return launch_score_d<128, 2>(p, st);
        case 2561: return launch_score_d<256, 1>(p, st);
        case 2562: return launch_score_d<256, 2>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
