// context.cu -- the kernels of the context-parallel step: one sequence's
// pages split over ranks, with one exchange (all-gather of the page scores,
// then of the partial attention results).
//
// The method ("Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs
// Without Retraining", abstract; "Methodology") attends each query head to
// prefix, window and the query-aware top-k pages of the full cache.  Split by
// pages over ranks, the top-k of the union is the top-k of the concatenated
// per-rank scores (selected on every rank by the selection kernels over the
// gathered scores), and the attention over the union of the ranks' disjoint
// token sets is the log-sum-exp merge of the per-rank attentions:
//     lse = log sum_r e^(lse_r),   out = sum_r e^(lse_r - lse) out_r.
// This file holds the two steps that have no single-GPU counterpart: taking a
// rank's pages out of the global selection, and the merge.
#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

// One CTA per (sequence, kv-head) unit.  The selection is ascending, so the
// pages in [lo, hi) are a contiguous run that starts after the pages below lo.
__global__ void __launch_bounds__(128) shard_selection_kernel(const int32_t* sel,
                                                              const int32_t* n_sel, int max_sel,
                                                              int lo, int hi, int max_local,
                                                              int32_t* sel_local,
                                                              int32_t* n_local) {
    __shared__ int below, inside;
    const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    int n = n_sel[u];
    n = n < 0 ? 0 : (n > max_sel ? max_sel : n);
    const int32_t* s = sel + (size_t)u * max_sel;
    if (tid == 0) below = inside = 0;
    __syncthreads();
    int a = 0, c = 0;
    for (int j = tid; j < n; j += blockDim.x) {
        const int v = s[j];
        a += v < lo;
        c += v >= lo && v < hi;
    }
    a = __reduce_add_sync(0xffffffffu, a);
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) {
        atomicAdd(&below, a);
        atomicAdd(&inside, c);
    }
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x) {
        const int v = s[j];
        const int at = j - below;            // in range only for an ascending selection
        if (v >= lo && v < hi && at >= 0 && at < max_local)
            sel_local[(size_t)u * max_local + at] = v - lo;
    }
    if (tid == 0) n_local[u] = inside < max_local ? inside : max_local;
}

// One CTA per (sequence, query head); fp32 throughout, bf16 out rounded to
// nearest even.
template <int D>
__global__ void __launch_bounds__(64) merge_kernel(int parts, int bh_count,
                                                   const __nv_bfloat16* out_parts,
                                                   const float* lse_parts, __nv_bfloat16* out,
                                                   float* lse) {
    const int bh = blockIdx.x, tid = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < parts; ++r) M = fmaxf(M, lse_parts[(size_t)r * bh_count + bh]);
    if (M == -INFINITY) {                    // no part attended a token
        for (int c = tid; c < D; c += blockDim.x)
            out[(size_t)bh * D + c] = __float2bfloat16_rn(0.f);
        if (lse && tid == 0) lse[bh] = -INFINITY;
        return;
    }
    float wsum = 0.f;
    for (int r = 0; r < parts; ++r) wsum += expf(lse_parts[(size_t)r * bh_count + bh] - M);
    for (int c = tid; c < D; c += blockDim.x) {
        float acc = 0.f;
        for (int r = 0; r < parts; ++r) {
            const float w = expf(lse_parts[(size_t)r * bh_count + bh] - M);
            acc += w * __bfloat162float(out_parts[((size_t)r * bh_count + bh) * D + c]);
        }
        out[(size_t)bh * D + c] = __float2bfloat16_rn(acc / wsum);
    }
    if (lse && tid == 0) lse[bh] = M + logf(wsum);
}

}  // namespace

cudaError_t launch_shard_selection(const Shape& s, const int32_t* sel, const int32_t* n_sel,
                                   int lo, int hi, int max_local, int32_t* sel_local,
                                   int32_t* n_local, cudaStream_t st) {
    const int units = s.B * s.Hkv;
    shard_selection_kernel<<<units, 128, 0, st>>>(sel, n_sel, s.max_sel, lo, hi, max_local,
                                                  sel_local, n_local);
    return cudaGetLastError();
}

cudaError_t launch_merge(int parts, int bh_count, int D, const void* out_parts,
                         const float* lse_parts, void* out, float* lse, cudaStream_t st) {
    const auto* op = static_cast<const __nv_bfloat16*>(out_parts);
    auto* o = static_cast<__nv_bfloat16*>(out);
    switch (D) {
        case 64: merge_kernel<64><<<bh_count, 64, 0, st>>>(parts, bh_count, op, lse_parts, o, lse); break;
        case 128: merge_kernel<128><<<bh_count, 64, 0, st>>>(parts, bh_count, op, lse_parts, o, lse); break;
        case 256: merge_kernel<256><<<bh_count, 64, 0, st>>>(parts, bh_count, op, lse_parts, o, lse); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace csa
