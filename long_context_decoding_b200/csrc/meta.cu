// meta.cu -- token append and page-metadata maintenance.
//
// The KV cache stays full size ("Why It Matters", roboaidigest post), and
// the Quest-style selection ("Methodology", arxivlens analysis) scores a page
// from its per-channel key minimum and maximum.  This kernel writes the new
// tokens into their page slots and brings the min/max of every touched page
// up to date: from the new keys alone when the page starts inside the new
// tokens, else by folding the new keys into the stored min/max (exact, since
// min and max of bf16 values are bf16 values).  In rebuild mode (no new
// tokens) it recomputes the touched pages' min/max from the cache.
//
// One CTA per (sequence, kv-head, touched page), D/2 threads, each owning a
// bf16x2 channel pair: every global access is a coalesced 4-byte word per
// thread.  The work is tiny (a few KB per layer per step); it is a latency
// kernel, not a bandwidth one.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

struct Pair {
    uint32_t lo, hi;   // bf16x2 minimum / maximum, channel 2c in bits 0..15
};

__device__ __forceinline__ uint32_t sel_half(uint32_t cur, uint32_t v, int half, bool take) {
    const uint32_t m = half ? 0xffff0000u : 0x0000ffffu;
    return take ? ((cur & ~m) | (v & m)) : cur;
}

// Fold key word v into the running min/max (strict comparisons: on equal
// values the earlier token's bits stay).
__device__ __forceinline__ void fold(Pair& p, uint32_t v) {
    const float v0 = bf16_lo(v), v1 = bf16_hi(v);
    p.lo = sel_half(p.lo, v, 0, v0 < bf16_lo(p.lo));
    p.lo = sel_half(p.lo, v, 1, v1 < bf16_hi(p.lo));
    p.hi = sel_half(p.hi, v, 0, v0 > bf16_lo(p.hi));
    p.hi = sel_half(p.hi, v, 1, v1 > bf16_hi(p.hi));
}

// ---------------------------------------------------------------- fp8 copy
// The optional fp8 copy of a metadata row pair: 2*D bytes of E4M3 (OCP FP8:
// bias 7, 3 mantissa bits, largest value 448, subnormals k * 2^-9) holding
// min * 2^-e rounded toward -inf and max * 2^-e rounded toward +inf, then a
// 16-byte trailer {e, 0, 0, 0} (int32).  e is the smallest integer with
// max |value| * 2^-e <= 448 over the row pair (0 when it is all zero), so
// the decoded box contains the exact one and the Quest bound stays an upper
// bound.  All steps below are exact in fp32: scaling by powers of two and
// floor/ceil of quotients by powers of two.

// Largest (up = false) / smallest (up = true) E4M3 value <= / >= y, |y| <= 448.
__device__ float fp8_round(float y, bool up) {
    const bool neg = y < 0.f;
    if (neg) {
        y = -y;
        up = !up;
    }
    float quantum = 0.001953125f;                    // 2^-9 below 2^-6
    if (y >= 0.015625f) {
        int ex;
        frexpf(y, &ex);                              // y in [2^(ex-1), 2^ex)
        quantum = ldexpf(1.f, ex - 4);               // 3 mantissa bits
    }
    const float k = up ? ceilf(y / quantum) : floorf(y / quantum);
    const float r = k * quantum;
    return neg ? -r : r;
}

// E4M3 bits of a value on the grid; zero is 0x00.
__device__ uint32_t fp8_encode(float v) {
    if (v == 0.f) return 0u;
    const uint32_t s = v < 0.f ? 0x80u : 0u;
    const float a = fabsf(v);
    if (a < 0.015625f) return s | (uint32_t)(a * 512.f);
    int ex;
    frexpf(a, &ex);
    const int E = ex - 1;
    const int m = (int)ldexpf(a, 3 - E);             // 8 .. 15
    return s | ((uint32_t)(E + 7) << 3) | (uint32_t)(m - 8);
}

__device__ uint32_t fp8_outward(float x, int e, bool up) {
    float y = ldexpf(x, -e);
    // below 2^-10 only the sign decides (and fp32 may have underflowed)
    if (x != 0.f && fabsf(y) < 0.0009765625f) y = copysignf(0.0009765625f, x);
    return fp8_encode(fp8_round(y, up));
}

// Called by all D/2 threads of the CTA (thread c owns channels 2c, 2c+1).
__device__ void write_fp8_row(const MetaParams& p, int phys, int g, int c, const Pair& acc) {
    __shared__ uint32_t s_max[4];
    const int D = p.s.D;
    const int warp = c >> 5, lane = c & 31;
    const float mn0 = bf16_lo(acc.lo), mn1 = bf16_hi(acc.lo);
    const float mx0 = bf16_lo(acc.hi), mx1 = bf16_hi(acc.hi);
    const float a = fmaxf(fmaxf(fabsf(mn0), fabsf(mn1)), fmaxf(fabsf(mx0), fabsf(mx1)));
    // non-negative floats order like their bit patterns
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
    if (lane == 0) s_max[warp] = wmax;
    __syncthreads();
    uint32_t amax_bits = 0;
    for (int w = 0; w < (D / 2 + 31) / 32; ++w) amax_bits = max(amax_bits, s_max[w]);
    __syncthreads();            // s_max is reused by the next page of this CTA
    const float amax = __uint_as_float(amax_bits);
    int e = 0;
    if (amax > 0.f) {
        int ex;
        const float f = frexpf(amax, &ex);           // amax = (2f) * 2^(ex-1)
        e = ex - 1 - 8 + (2.f * f > 1.75f ? 1 : 0);
    }
    uint8_t* row = p.meta8 + ((size_t)phys * p.s.Hkv + g) * (size_t)(2 * D + 16);
    const uint32_t lo = fp8_outward(mn0, e, false) | (fp8_outward(mn1, e, false) << 8);
    const uint32_t hi = fp8_outward(mx0, e, true) | (fp8_outward(mx1, e, true) << 8);
    reinterpret_cast<uint16_t*>(row)[c] = (uint16_t)lo;
    reinterpret_cast<uint16_t*>(row + D)[c] = (uint16_t)hi;
    if (c == 0) *reinterpret_cast<int4*>(row + 2 * D) = make_int4(e, 0, 0, 0);
}

// Append the new tokens of logical page `page` and refresh its min/max.
// phys is the page's physical id (page_table[b][page]).
__device__ void update_page(const MetaParams& p, int b, int g, int c, int L, int start, int page,
                            int phys) {
    const int Hkv = p.s.Hkv, D = p.s.D;
    const bool append = p.new_k != nullptr;
    const int t0 = page * kPage;
    const int t_end = t0 + kPage < L ? t0 + kPage : L;
    if (phys < 0 || phys >= p.s.NPG) {
        if (c == 0) latch_flag(p.flags, CSA_DEVFLAG_BAD_PAGE_ID);
        return;
    }
    const int W = D / 2;                                    // words per key row
    const size_t tile = ((size_t)phys * Hkv + g) * kPage * W;
    uint32_t* kc = reinterpret_cast<uint32_t*>(p.k_cache) + tile;
    uint32_t* vc = reinterpret_cast<uint32_t*>(p.v_cache) + tile;
    uint32_t* mt = reinterpret_cast<uint32_t*>(p.meta) + ((size_t)phys * Hkv + g) * 2 * W;
    const int first_new = t0 > start ? t0 : start;

    Pair acc;
    bool have = false;
    if (append) {
        const uint32_t* nk = reinterpret_cast<const uint32_t*>(p.new_k);
        const uint32_t* nv = reinterpret_cast<const uint32_t*>(p.new_v);
        if (first_new > t0) {                 // older tokens: stored min/max
            acc.lo = mt[c];
            acc.hi = mt[W + c];
            have = true;
        }
        for (int t = first_new; t < t_end; ++t) {
            const size_t src = (((size_t)b * p.n_new + (t - start)) * Hkv + g) * W + c;
            const uint32_t kw = nk[src];
            kc[(size_t)(t - t0) * W + c] = kw;
            vc[(size_t)(t - t0) * W + c] = nv[src];
            if (have) {
                fold(acc, kw);
            } else {
                acc.lo = acc.hi = kw;
                have = true;
            }
        }
    } else {
        for (int t = t0; t < t_end; ++t) {
            const uint32_t kw = kc[(size_t)(t - t0) * W + c];
            if (have) {
                fold(acc, kw);
            } else {
                acc.lo = acc.hi = kw;
                have = true;
            }
        }
    }
    mt[c] = acc.lo;
    mt[W + c] = acc.hi;
    if (p.meta8) write_fp8_row(p, phys, g, c, acc);
}

__global__ void meta_update_kernel(MetaParams p) {
    const int u = blockIdx.x;
    const int Hkv = p.s.Hkv, D = p.s.D, MP = p.s.MP;
    const int b = u / Hkv, g = u % Hkv;
    const int c = threadIdx.x;                  // channel pair
    // seq_lens and page_table are caller inputs, read before the dependency
    // wait; the cache, the metadata and the new tokens only after it
    const int L = p.seq_lens[b];
    const bool append = p.new_k != nullptr;
    const bool bad_len = L < 0 || L > MP * kPage || (append && L < p.n_new);
    const int start = bad_len ? 0 : (L - p.n_new > 0 ? L - p.n_new : 0);   // first new token
    const int n_touched = bad_len || L == 0 ? 0 : (L - 1) / kPage - start / kPage + 1;
    const int j0 = (int)blockIdx.y;
    const int phys0 = j0 < n_touched ? p.page_table[(size_t)b * MP + start / kPage + j0] : -1;
    // the next grid may start now: whatever follows an append reads only
    // caller inputs before its own dependency wait, which covers this kernel
    pdl_launch_dependents();
    pdl_wait();
    if (bad_len) {
        if (c == 0 && blockIdx.y == 0) latch_flag(p.flags, CSA_DEVFLAG_BAD_SEQ_LEN);
        return;
    }
    if (c >= D / 2) return;
    for (int j = j0; j < n_touched; j += (int)gridDim.y) {
        const int page = start / kPage + j;
        const int phys = j == j0 ? phys0 : p.page_table[(size_t)b * MP + page];
        update_page(p, b, g, c, L, start, page, phys);
    }
}

}  // namespace

cudaError_t launch_meta_update(const MetaParams& p, cudaStream_t st) {
    const int units = p.s.B * p.s.Hkv;
    int pages = (p.n_new + kPage - 1) / kPage + 1;          // pages one chunk can touch
    if (pages > p.s.MP) pages = p.s.MP;
    if (pages > 65535) pages = 65535;                       // grid.y limit; the kernel strides
    if (units == 0 || pages <= 0) return cudaSuccess;
    dim3 grid(units, pages);
    return launch_pdl(meta_update_kernel, grid, dim3(p.s.D / 2), 0, st, p);
}

}  // namespace csa
