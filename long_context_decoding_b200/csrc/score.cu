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
// Data path (the kernel is HBM-bound: it streams 4*D bytes of metadata per
// candidate page and does ~2 flop per byte):
//   * the candidates of all (sequence, kv-head) units are flattened and split
//     evenly over a grid sized to fill every SM;
//   * each CTA copies its slice of the page table into shared memory once;
//   * a producer warp issues one TMA bulk copy (cp.async.bulk) per page into
//     a ring of 16-page stages tracked by mbarriers with byte counts; rows are
//     padded to 4*D+16 bytes so that the fragment loads are bank-conflict free;
//   * four consumer warps each take whole stages: 2D/16 mma.sync m16n8k16 per
//     tile, a quad-shuffle max over heads, fp32 scores out.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

template <int D, int NB>
struct ScoreCfg {
    static constexpr int kConsumers = 4;
    static constexpr int kThreads = 32 * (kConsumers + 1);
    static constexpr int kTile = 16;                  // pages per stage (one m16 tile)
    static constexpr int kRowBytes = 4 * D;           // [min | max] bf16 of one (page, kv-head)
    static constexpr int kRowStride = 4 * D + 16;     // padded shared-memory row
    static constexpr int kStageBytes = kTile * kRowStride;
    static constexpr int kStages = D >= 256 ? 4 : 8;
    // a stage's previous use must belong to the same consumer warp, so that a
    // parity wait can never be two phases ahead of the barrier
    static_assert(kStages % kConsumers == 0, "stages must be a multiple of consumers");
    static constexpr int kKPairs = 2 * D / 32;        // 32-channel steps along [min | max]
    // stages | page-table slice | full/empty barriers | tile infos | 3 x [B + 1] ints
    static __host__ __device__ size_t smem_bytes(int B) {
        return (size_t)kStages * kStageBytes + (size_t)kScorePtCap * 4 + 16 * (size_t)kStages +
               16 * (size_t)kStages + 3 * 4 * (size_t)(B + 1);
    }
};

struct TileInfo {
    int unit;      // b * Hkv + g
    int first;     // logical page of row 0
    int count;     // rows in use (1..16)
    uint32_t valid;
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

// After a timed-out wait (the CTA unwinds with CSA_DEVFLAG_TIMEOUT latched),
// keep the CTA alive, again for a bounded time, until every copy it issued
// has landed, so that no TMA write targets shared memory of a finished CTA.
template <int kStages>
__device__ void drain_issued(uint64_t* full, int issued) {
    for (int st = 0; st < kStages && st < issued; ++st) {
        const int last = st + ((issued - 1 - st) / kStages) * kStages;   // last use of st
        mbar_wait(&full[st], (last / kStages) & 1);
    }
}

// Consumer warps: score whole 16-page stages on the tensor cores.
template <int D, int NB>
__device__ __forceinline__ void consume(const ScoreParams& p, TileWalker walk, uint8_t* stages,
                                        uint64_t* full, uint64_t* empty, const TileInfo* info,
                                        int* s_abort, int warp, int lane) {
    using C = ScoreCfg<D, NB>;
    const int Hkv = p.s.Hkv, G = p.s.G, MP = p.s.MP;
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t qf[C::kKPairs][NB][4];          // B fragments of [q- | q+] for the current unit
    int cur_unit = -1;
    TileInfo t;
    for (int j = 0; walk.next(t); ++j) {
        if (j % C::kConsumers != warp) continue;
        const int st = j % C::kStages;
        const int r = j / C::kStages;
        if (!mbar_wait(&full[st], r & 1)) {
            if (lane == 0) latch_flag(p.flags, CSA_DEVFLAG_TIMEOUT);
            *s_abort = 1;
            break;
        }
        if (*(volatile int*)s_abort) break;
        const TileInfo ti = info[st];
        if (ti.unit != cur_unit) {
            cur_unit = ti.unit;
            const int b = ti.unit / Hkv, g = ti.unit % Hkv;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int head = nb * 8 + gq;
                const uint32_t* qw = reinterpret_cast<const uint32_t*>(
                    p.q + ((size_t)b * p.s.Hq + (size_t)g * G + head) * D);
#pragma unroll
                for (int kp = 0; kp < C::kKPairs; ++kp) {
                    // channels ch0 .. ch0+7 of the [min | max] row; min pairs with q-
                    const int ch0 = 32 * kp + 8 * tq;
                    const bool is_max = ch0 >= D;
                    const int qc = is_max ? ch0 - D : ch0;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t v = head < G ? __ldg(qw + qc / 2 + w) : 0u;
                        qf[kp][nb][w] = is_max ? pos_part(v) : neg_part(v);
                    }
                }
            }
        }
        float acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
            acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
        const uint32_t base = smem_u32(stages + (size_t)st * C::kStageBytes);
        const uint32_t row0 = base + gq * C::kRowStride + 16 * tq;
        const uint32_t row8 = row0 + 8 * C::kRowStride;
#pragma unroll
        for (int kp = 0; kp < C::kKPairs; ++kp) {
            const uint4 x = ld_shared_v4(row0 + 64 * kp);
            const uint4 y = ld_shared_v4(row8 + 64 * kp);
            const uint32_t a0[4] = {x.x, y.x, x.y, y.y};
            const uint32_t a1[4] = {x.z, y.z, x.w, y.w};
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                mma_bf16_16816(acc[nb], a0, qf[kp][nb][0], qf[kp][nb][1]);
                mma_bf16_16816(acc[nb], a1, qf[kp][nb][2], qf[kp][nb][3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);   // stage free once fragments are loaded
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
        if (tq < 2 && row < ti.count) {
            float v = tq == 0 ? m0 : m8;
            if (!((ti.valid >> row) & 1u)) v = -INFINITY;
            const size_t o = (size_t)ti.unit * MP + ti.first + row;
            p.scores_ws[o] = v;
            if (p.scores_out) p.scores_out[o] = v;
        }
    }
}

template <int D, int NB>
__global__ void __launch_bounds__(ScoreCfg<D, NB>::kThreads)
score_kernel(ScoreParams p) {
    using C = ScoreCfg<D, NB>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* stages = smem;
    int* pt = reinterpret_cast<int*>(stages + (size_t)C::kStages * C::kStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(pt + kScorePtCap);
    uint64_t* empty = full + C::kStages;
    TileInfo* info = reinterpret_cast<TileInfo*>(empty + C::kStages);
    int* seq_n = reinterpret_cast<int*>(info + C::kStages);
    int* seq_clo = seq_n + (p.s.B + 1);
    int* seq_off = seq_clo + (p.s.B + 1);
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.s.B, Hkv = p.s.Hkv, G = p.s.G, MP = p.s.MP;

    // Candidates per sequence.
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
    if (tid == 0) s_abort = 0;
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
    const long long s = N * blockIdx.x / gridDim.x, e = N * (blockIdx.x + 1) / gridDim.x;
    if (s >= e) {
        pdl_wait();
        pdl_launch_dependents();
        return;
    }

    // Page-table slice of this CTA (the grid is sized so that e - s <= cap),
    // copied run by run: every run is a contiguous piece of one page-table row.
    TileWalker walk;
    walk.seq_off = seq_off;
    walk.seq_n = seq_n;
    walk.seq_clo = seq_clo;
    walk.Hkv = Hkv;
    walk.B = B;
    {
        TileWalker fill = walk;
        fill.start((int)s, (int)e);
        TileInfo run;
        int at = 0;
        while (fill.next(run, 1 << 30)) {
            const int32_t* src = p.page_table + (size_t)(run.unit / Hkv) * MP + run.first;
            for (int i = tid; i < run.count; i += C::kThreads) pt[at + i] = __ldg(src + i);
            at += run.count;
        }
    }
    walk.start((int)s, (int)e);
    __shared__ int s_issued;
    if (tid == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        fence_barrier_init();
        s_issued = 0;
    }
    // the metadata was written by the previous kernel on the stream
    pdl_wait();
    pdl_launch_dependents();
    __syncthreads();

    if (warp == C::kConsumers) {
        // ------------------------------------------------------------ producer
        TileInfo t;
        for (int j = 0; walk.next(t); ++j) {
            const int st = j % C::kStages;
            const int r = j / C::kStages;
            if (lane == 0 && r > 0 && !mbar_wait(&empty[st], (r - 1) & 1)) {
                latch_flag(p.flags, CSA_DEVFLAG_TIMEOUT);
                s_abort = 1;
            }
            __syncwarp();
            if (*(volatile int*)&s_abort) break;
            const int g = t.unit % Hkv;
            const int x0 = walk.x - t.count - (int)s;    // slice index of row 0
            int phys = -1;
            bool ok = false;
            if (lane < t.count) {
                phys = pt[x0 + lane];
                ok = phys >= 0 && phys < p.s.NPG;
                if (!ok) latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
            }
            const uint32_t valid = __ballot_sync(0xffffffffu, ok);
            if (lane == 0) {
                t.valid = valid;
                info[st] = t;
                mbar_arrive_expect_tx(&full[st], (uint32_t)__popc(valid) * C::kRowBytes);
            }
            __syncwarp();
            if (ok) {
                const uint16_t* src = p.meta + ((size_t)phys * Hkv + g) * 2 * D;
                tma_bulk_g2s(stages + (size_t)st * C::kStageBytes + lane * C::kRowStride, src,
                             C::kRowBytes, &full[st]);
            }
            if (lane == 0) s_issued = j + 1;
        }
    } else {
        consume<D, NB>(p, walk, stages, full, empty, info, &s_abort, warp, lane);
    }
    __syncthreads();
    if (tid == 0 && s_abort) drain_issued<C::kStages>(full, s_issued);
}

template <int D, int NB>
cudaError_t launch_score_t(const ScoreParams& p, cudaStream_t st) {
    using C = ScoreCfg<D, NB>;
    auto kern = score_kernel<D, NB>;
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
    // resident CTAs per SM: registers allow several; shared memory decides
    int occ = (int)((size_t)(228 * 1024) / (smem + 1024));
    if (occ > 4) occ = 4;
    if (occ < 1) occ = 1;
    const long long ub = (long long)p.s.B * p.s.Hkv * p.s.MP;
    long long grid = (long long)occ * device_sm_count();
    const long long need = (ub + kScorePtCap - 1) / kScorePtCap;
    if (need > grid) grid = need;
    if (grid < 1) grid = 1;
    return launch_pdl(score_kernel<D, NB>, dim3((unsigned)grid), dim3(C::kThreads), smem, st, p);
}

}  // namespace

cudaError_t launch_score(const ScoreParams& p, cudaStream_t st) {
    const int nb = p.s.G > 8 ? 2 : 1;
    switch (p.s.D * 10 + nb) {
        case 641: return launch_score_t<64, 1>(p, st);
        case 642: return launch_score_t<64, 2>(p, st);
        case 1281: return launch_score_t<128, 1>(p, st);
        case 1282: return launch_score_t<128, 2>(p, st);
        case 2561: return launch_score_t<256, 1>(p, st);
        case 2562: return launch_score_t<256, 2>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
