// common.cuh -- device helpers shared by the libcsa kernels (sm_100a).
//
// bf16 bit helpers, an order-preserving float -> key map, inline-PTX wrappers
// for the warp-level bf16 tensor-core MMA and the ldmatrix / movmatrix
// fragment moves, programmatic dependent launch, and the per-sequence token
// geometry (prefix, window, candidate pages) every kernel shares.  No kernel
// of the library spins on a flag or barrier of its own.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/csa.h"

namespace csa {

constexpr int kPage = 16;                       // tokens per page
constexpr int kMaxUnits = 2048;                 // B * Hkv supported per call
constexpr int kScorePtCap = 4096;               // page-table entries staged per scoring CTA
constexpr int kDecodeItemCap = 1024;            // pages staged per decode CTA

// ------------------------------------------------------------ bf16 / keys
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
}

// Pack two floats into a bf16x2 word, round-to-nearest-even (lo in bits 0..15).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Order-preserving map fp32 -> uint32 (larger float -> larger key).  -0 and
// +0 map to the same key; NaN maps to 0, below every number.
__device__ __forceinline__ uint32_t order_key(float s) {
    if (s != s) return 0u;
    uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------ misc PTX
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float ex2(float x) {     // 2^x, hardware approximation
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void latch_flag(uint32_t* flags, uint32_t bit) {
    if (flags) atomicOr(flags, bit);
}

// Programmatic dependent launch: wait for the preceding grid's memory, or
// let the next grid start its prologue.  No-ops without the launch attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ tensor core
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
//   A (16x16 row): a0 (g, 2t..2t+1) a1 (g+8, 2t..) a2 (g, 2t+8..) a3 (g+8, 2t+8..)
//   B (16x8 col):  b0 (k 2t..2t+1, n g) b1 (k 2t+8.., n g)
//   D (16x8):      d0 (g, 2t) d1 (g, 2t+1) d2 (g+8, 2t) d3 (g+8, 2t+1)
// with g = lane / 4, t = lane % 4.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same with f16 inputs.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
// 16-byte global -> shared copies that bypass L1; src_bytes < 16 zero-fills the rest.
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

// Transpose an 8x8 b16 matrix held one fragment row-pair per lane.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// ------------------------------------------------------------ sequence geometry
// Token ranges of one sequence for one call: effective prefix Pe and window
// We, logical pages np, and the top-k candidate pages [c_lo, c_hi): the
// pages holding at least one token of [Pe, L - We) (empty when prefix and
// window cover every token).
struct SeqGeom {
    int L, Pe, We, np, c_lo, c_hi;
};
__host__ __device__ __forceinline__ SeqGeom seq_geom(int L, int prefix, int window) {
    SeqGeom s;
    s.L = L;
    s.Pe = prefix < L ? prefix : L;
    s.We = window < L ? window : L;
    s.np = (L + kPage - 1) / kPage;
    if (s.Pe < L - s.We) {
        s.c_lo = s.Pe / kPage;
        s.c_hi = (L - s.We + kPage - 1) / kPage;
    } else {
        s.c_lo = 0;
        s.c_hi = 0;
    }
    return s;
}

// ------------------------------------------------------------ launches
// Launch with programmatic stream serialization: the grid may start while
// the previous kernel on the stream is still running.  Every kernel of this
// library reads only caller inputs before pdl_wait(), with two exceptions
// that also read library-written data early: the prefix/window work of the
// fused kernel (after the scoring kernel) and of the early decode (after the
// selection kernel).  The kernels ahead of those two call
// pdl_launch_dependents() only after their own wait, so that when either
// starts, every kernel two or more launches earlier has completed.  The
// append kernel, which neither of those two can follow, lets the next grid
// start at its own start.

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace csa
