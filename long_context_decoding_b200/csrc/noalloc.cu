// noalloc.cu -- csa_decode_noalloc: the sparse decode of csa_decode with its
// scratch memory built into the library.
//
// Some callers cannot allocate device memory at all: a plugin hosted inside
// another runtime that owns every device buffer and hands the plugin only
// its inputs and outputs, or a serving process that reserves the whole GPU
// for its KV cache at start-up and forbids any allocation afterwards.  Such a
// caller cannot provide the workspace csa_decode needs for its split-K
// partial results.  This entry point runs the same decode kernel, but its
// scratch (flag word, record ranges and partial records) lives in one
// file-scope __device__ array of kNoAllocScratchBytes that every GPU which
// loads the library keeps until the process exits.  The call itself
// allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
//
// The host name of that array is only a stand-in; the kernels get its device
// address, looked up once per device (with that device current) through
// cudaGetSymbolAddress on the first call made on the device.  Make that first
// call before any stream capture.
//
// All calls share the one array and it keeps whatever the previous call left:
// the flag word is cleared on the caller's stream at the start of every call;
// the record ranges and partial records are rewritten by every call before
// they are read.  Two calls whose
// kernels overlap on a GPU therefore race on the array: issue them on one
// stream, or order them.
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace csa {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;   // 8 MiB per GPU
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (nullptr on error).
void* scratch_address(int dev) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

bool ok16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" int csa_decode_noalloc(const csa_dims* d, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* page_table,
                                  const int32_t* seq_lens, const int32_t* sel_pages,
                                  const int32_t* n_sel, int prefix, int window, float scale,
                                  void* out, float* lse, void* stream) {
    Shape s;
    const int rc = check_dims(d, &s);
    if (rc != CSA_OK) return rc;
    if (!ok16(q) || !ok16(k_cache) || !ok16(v_cache) || !ok16(page_table) || !ok16(seq_lens) ||
        !ok16(sel_pages) || !ok16(n_sel) || !ok16(out) || (lse && !ok16(lse)))
        return CSA_ERR_INVALID_ARG;
    if (prefix < 0 || window < 0 || !(scale == scale) || isinf(scale)) return CSA_ERR_INVALID_ARG;

    // scratch: [flag word | record ranges | partial records of the two
    // decode phases], each 256-byte aligned
    const size_t units = (size_t)s.B * s.Hkv;
    const size_t ranges_off = 256;
    const size_t partials_off = ranges_off + up256(16 * units);
    const size_t slots = (size_t)decode_grid(s) + units;
    const size_t need = partials_off + 2 * 4 * slots * decode_record_floats(s);
    if (need > kNoAllocScratchBytes) return CSA_ERR_WORKSPACE;   // shape needs more scratch

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    uint8_t* scratch = static_cast<uint8_t*>(scratch_address(dev));
    if (!scratch) return CSA_ERR_CUDA;

    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(scratch, 0, 4, st) != cudaSuccess) {   // flag word
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    DecodeParams p;
    p.q = static_cast<const uint16_t*>(q);
    p.k_cache = static_cast<const uint16_t*>(k_cache);
    p.v_cache = static_cast<const uint16_t*>(v_cache);
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.sel = sel_pages;
    p.n_sel = n_sel;
    p.prefix = prefix;
    p.window = window;
    p.dense = 0;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)s.D);
    p.scale_log2 = sc * 1.4426950408889634f;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.flags = reinterpret_cast<uint32_t*>(scratch);
    p.rec_range = reinterpret_cast<int4*>(scratch + ranges_off);
    p.partials = reinterpret_cast<float*>(scratch + partials_off);
    p.phase_floats = slots * decode_record_floats(s);
    // as csa_decode: right after a selection call on this stream, the prefix
    // and window pages stream before the dependency wait and the selection is
    // read after it; otherwise the caller inputs are read before the wait and
    // the scratch is touched only after it
    p.early = last_stream_call(stream) == kCallScoreSelect ? 1 : 0;
    p.s = s;
    note_stream_call(stream, kCallOther);
    if (launch_decode(p, st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    return CSA_OK;
}
