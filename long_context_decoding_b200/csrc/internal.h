// internal.h -- host-side interface between the C ABI (csa_api.cu) and the
// kernel translation units.  Not installed; the public ABI is include/csa.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// Workspace layout (byte offsets into the caller's workspace).
struct WsLayout {
    size_t flags;          // uint32 device flag word
    size_t rec_range;      // int4 [units]
    size_t keyrange;       // uint2 [units]: ~min and max order key of the scores
    size_t scores;         // fp32 [B][Hkv][max_pages]
    size_t partials;       // fp32 [2][dec_slots][decode_record_floats]
    size_t dec_slots;      // partial records available per decode phase
    size_t total;
};

struct Shape {
    int B, Hq, Hkv, G, D, MP, NPG, max_sel;
};

// ---------------------------------------------------------------- meta
struct MetaParams {
    uint16_t* k_cache;
    uint16_t* v_cache;
    uint16_t* meta;
    const int32_t* page_table;
    const int32_t* seq_lens;
    const uint16_t* new_k;   // nullable (rebuild)
    const uint16_t* new_v;
    uint8_t* meta8;          // nullable: fp8 copy [num_pages][Hkv][2D + 16] to keep current
    int n_new;
    uint32_t* flags;
    Shape s;
};
cudaError_t launch_meta_update(const MetaParams& p, cudaStream_t st);

// ---------------------------------------------------------------- score
struct ScoreParams {
    const uint16_t* q;
    const uint16_t* meta;
    const int32_t* page_table;
    const int32_t* seq_lens;
    int prefix, window;
    float* scores_ws;       // [B][Hkv][MP]
    float* scores_out;      // nullable
    const uint8_t* meta8;   // non-null: score from the fp8 copy instead of meta
    uint2* keyrange;        // [units] merged with atomicMax: ~min key, max key
    uint32_t* flags;
    Shape s;
};
cudaError_t launch_score(const ScoreParams& p, cudaStream_t st);

// ---------------------------------------------------------------- select
struct SelectParams {
    float* scores_ws;       // read; rewritten in place as order keys
    const int32_t* seq_lens;
    int prefix, window, k_pages;
    int32_t* sel;
    int32_t* n_sel;
    uint2* keyrange;        // [units] from the scoring kernel; reset to zero here
    uint32_t* flags;
    int smem_keys;          // keys that fit in the dynamic shared memory (set by the launcher)
    Shape s;
};
cudaError_t launch_select(const SelectParams& p, cudaStream_t st);

// ---------------------------------------------------------------- decode
struct DecodeParams {
    const uint16_t* q;
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    const int32_t* page_table;
    const int32_t* seq_lens;
    const int32_t* sel;     // nullable when dense
    const int32_t* n_sel;
    int prefix, window;
    int dense;
    float scale_log2;       // softmax scale * log2(e)
    uint16_t* out;
    float* lse;             // nullable
    uint32_t* flags;
    int4* rec_range;        // [units]: first/last CTA with a record, per phase (x,y | z,w)
    float* partials;        // [2][dec_slots][record]: o[G][D] | m[G] | l[G]
    size_t phase_floats;    // floats of one phase's record region (dec_slots * record)
    int early;              // 1: the prefix/window phase runs before the dependency wait
    Shape s;
};
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t st);

// ---------------------------------------------------------------- fused
// Selection + decode in one launch (csa_sparse_attention): clusters of 8
// CTAs select the top-k pages of one unit each and attend over them; more
// CTAs of the same grid attend over the prefix and window pages meanwhile.
struct FusedParams {
    DecodeParams d;          // q, caches, geometry, outputs, workspace records
    const float* scores_ws;  // [units][MP] Quest scores of the candidates
    int k_pages;
    int32_t* sel;            // [units][max_sel] selected pages (output)
    int32_t* n_sel;          // [units] (output)
    uint2* keyrange;         // [units] from the scoring kernel; reset to zero here
    int n0;                  // CTAs of the prefix/window role (a multiple of 8)
};
bool fused_eligible(const Shape& s, int prefix, int window, int k_pages);
int fused_phase0_ctas(const Shape& s);
int fused_phase0_ctas(const Shape& s, long long prefix, long long window);
cudaError_t launch_fused(const FusedParams& p, cudaStream_t st);

// Kind of the last kernel-launching call issued on a stream (host side).
// csa_decode streams the prefix/window pages before the dependency wait only
// when the call before it on the stream was csa_score_select: its kernels
// wait in a chain, so every earlier kernel on the stream (the appends of
// csa_meta_update, the previous decode's combine) has finished by then.
enum CallKind { kCallOther = 0, kCallScoreSelect = 1 };
void note_stream_call(const void* stream, CallKind kind);
CallKind last_stream_call(const void* stream);

// Grid sizes (shared by the workspace sizing and the launches).
// ---------------------------------------------------------------- context parallelism
cudaError_t launch_shard_selection(const Shape& s, const int32_t* sel, const int32_t* n_sel,
                                   int lo, int hi, int max_local, int32_t* sel_local,
                                   int32_t* n_local, cudaStream_t st);
cudaError_t launch_merge(int parts, int bh_count, int D, const void* out_parts,
                         const float* lse_parts, void* out, float* lse, cudaStream_t st);

// Validates a csa_dims (sizes, supported head dims and group sizes, index
// ranges) and fills the kernel-side shape; CSA_OK or the status to return.
int check_dims(const ::csa_dims* d, Shape* s);

int device_sm_count();
int decode_grid(const Shape& s);
size_t decode_record_floats(const Shape& s);   // floats per split-K partial record
WsLayout workspace_layout(const Shape& s);

}  // namespace csa
