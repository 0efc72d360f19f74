// pisa_internal.h -- parameter blocks and launchers shared between the C-ABI
// layer (api.cu) and the kernel translation units. Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "pisa.h"
#include "pisa_device.cuh"

namespace pisa {

struct PoolParams {
    int B, Hkv, N, C;
    int64_t k_rows;      // rows per head in K (N for prefill, capacity for caches)
    const int32_t* len;  // optional per-sequence key count (device), else N
    Geom geom;           // pyramid layout (for N or for the capacity)
};

struct SelectParams {
    int B, Hq, Hkv, N, C, K, causal, forced_mask;
    float qscale;  // log2(e) / sqrt(d)
    Geom geom;
    int variant;   // enum pisa_score
};

struct AttnParams {
    int B, Hq, Hkv, N, C, K, causal;
    float qscale;  // log2(e) / sqrt(d)
};

struct DecodeParams {
    int B, Hq, Hkv, N, C, K, forced_mask;
    float qscale;  // log2(e) / sqrt(d)
    Geom geom;     // layout for the capacity N
    int variant;   // enum pisa_score
};

// block-major tensor-core path (bf16, d = 128, C = 64)
struct BmShape {
    int B, Hq, Hkv, N, G;
    int64_t M1;    // leaves per sequence
    int64_t rows;  // pyramid rows per (b, kv-head)
    int variant;   // enum pisa_score (the ranking scores need their own region unless 0)
};
struct BmLayout {  // byte offsets of the workspace regions
    size_t cand, lse, vscore, z2, counts, slots, offsets, entries, tiles, bsum, phl, resume, misc, oacc, total;
};
struct PhaseEvents {  // optional caller events recorded at phase boundaries
    void* const* events;
    int n;
};
BmLayout blockmajor_layout(const BmShape& s);
cudaError_t launch_select_bm(const void* Q, const void* K, const float* pyr, int32_t* idx, const SelectParams& sp,
                             const BmShape& s, void* ws, const PhaseEvents* ev, cudaStream_t st);
cudaError_t launch_attn_bm(const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                           const SelectParams& sp, const BmShape& s, void* ws, bool have_z2, const PhaseEvents* ev,
                           cudaStream_t st);
// backward with the selection fixed: its workspace is the forward's plus D per (query, head)
size_t blockmajor_bwd_bytes(const BmShape& s);
cudaError_t launch_attn_bwd_bm(const void* Q, const void* K, const void* V, const int32_t* idx, const void* dO,
                               float* dQ, float* dK, float* dV, const SelectParams& sp, const BmShape& s, void* ws,
                               bool saved, const PhaseEvents* ev, cudaStream_t st);

// The parameter blocks of a problem statement (the public pisa_cfg), built
// in one place for every entry point that launches the block-major path.
inline SelectParams select_params_of(const pisa_cfg* c) {
    SelectParams p;
    p.B = c->B; p.Hq = c->Hq; p.Hkv = c->Hkv; p.N = c->N; p.C = c->C; p.K = c->K;
    p.causal = c->causal; p.forced_mask = c->forced_mask;
    p.qscale = (float)(1.4426950408889634 / sqrt((double)c->d));
    make_geom(c->N, c->C, &p.geom);
    p.variant = c->score_variant;
    return p;
}
inline BmShape bm_shape_of(const pisa_cfg* c) {
    BmShape s;
    s.B = c->B; s.Hq = c->Hq; s.Hkv = c->Hkv; s.N = c->N; s.G = c->Hq / c->Hkv;
    s.M1 = ((int64_t)c->N + c->C - 1) / c->C;
    Geom g;
    make_geom(c->N, c->C, &g);
    s.rows = g.rows;
    s.variant = c->score_variant;
    return s;
}

// Stage 1 on the tensor cores (walk_tc.cu): tiles of consecutive positions
// walk the coarse levels, scoring the union of their kept parents'
// grandchildren. A tile that finishes every level writes the level-1
// candidates and bucket counts itself (resume[unit] = 0); otherwise each
// position's kept nodes go to the candidate region (slots 0..15) and
// resume[unit] = resume level << 8 | count, for the one-warp walk to finish.
// pyr_hl holds the bf16 high and low parts of the pyramid (walk_tc_pyramid_bytes).
bool walk_tc_fits(const SelectParams& sp);
size_t walk_tc_pyramid_bytes(int64_t units_bh, int64_t rows);
cudaError_t launch_walk_tc(const void* Q, const float* pyr, void* pyr_hl, int32_t* cand, int32_t* resume,
                           int32_t* counts, int32_t* slots, int* err, const SelectParams& sp, int G, int sms,
                           cudaStream_t st);

// the bf16 high / low parts of the fp32 pyramid (elems floats -> 2 x elems bf16 at pyr_hl)
cudaError_t launch_split_pyramid(const float* pyr, void* pyr_hl, int64_t elems, int sms, cudaStream_t st);
// flat Eq.(1) selection on the tensor cores (bsa_tc.cu); pyr_hl as for the tile walk
cudaError_t launch_bsa_tc(const void* Q, const float* pyr, void* pyr_hl, int32_t* idx, int* err,
                          const SelectParams& sp, int G, int sms, cudaStream_t st);

cudaError_t launch_pool(int dtype, int d, const void* K, float* pyr, const PoolParams& p, cudaStream_t st);
cudaError_t launch_attn_bwd(int dtype, int d, const void* Q, const void* K, const void* V, const int32_t* idx,
                            const void* dO, float* dQ, float* dK, float* dV, const AttnParams& p, cudaStream_t st);
cudaError_t launch_pyramid_grow(const float* old_pyr, float* new_pyr, int64_t units, int d, const Geom& go,
                                const Geom& gn, cudaStream_t st);
cudaError_t launch_cache_grow(const void* src, void* dst, int64_t units, int64_t rows_old, int64_t rows_new,
                              int row_bytes, cudaStream_t st);
cudaError_t launch_select(int dtype, int d, const void* Q, const void* K, const float* pyr, int32_t* idx,
                          const SelectParams& p, cudaStream_t st);
cudaError_t launch_attn(int dtype, int d, const void* Q, const void* K, const void* V, const int32_t* idx,
                        void* O, const AttnParams& p, cudaStream_t st);
cudaError_t launch_bsa(int dtype, int d, const void* Q, const float* pyr, int32_t* idx, const SelectParams& p,
                       cudaStream_t st);
cudaError_t launch_append(int dtype, int d, void* Kc, void* Vc, float* pyr, const void* k_new, const void* v_new,
                          const int32_t* pos, const DecodeParams& p, cudaStream_t st);
cudaError_t launch_decode(int dtype, int d, const void* q_new, void* Kc, void* Vc, float* pyr, const int32_t* pos,
                          int32_t* idx, void* o, const void* k_new, const void* v_new, const DecodeParams& p,
                          cudaStream_t st);

}  // namespace pisa
