// pisa_stage1.cuh -- the internal levels of the pyramid walk for one query,
// one warp, laid out for few instructions per scored level (close reading
// §04 4.2-4.4, Eq.(5)-(7), (11)).
//
// A scored level has at most 32 candidates (lane c owns candidate c) and needs
// the dot products of q with both children of each: 64 fp32 summary rows of
// 128 elements (512 bytes, four 128-byte lines). Lanes are split into 8 groups
// of 4: group g handles the two children of candidates 4g..4g+3 (8 rows, 1 KB
// contiguous per candidate); inside a group lane j reads the 32-byte chunks j,
// j+4, j+8, j+12 of each row with 256-bit loads, so one load instruction
// covers one whole line of each of 8 rows (the fewest L1 wavefronts for its
// 1 KB), and keeps the matching 32 elements of q in shared memory. A 2-stage
// reduce-scatter over the 4 lanes of the group leaves lane 4g+j with both
// children of candidate 4g+j, so the candidate's LSE over its children needs
// no further exchange.
#pragma once

#include "pisa_walk.cuh"

namespace pisa {

// 256-bit read-only global load (sm_100); p must be 32-byte aligned.
__device__ __forceinline__ void ldg_nc_v8(const float* p, float (&x)[8]) {
    asm("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]), "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7])
        : "l"(p));
}

// q is held in shared memory (one 128 x G float slot per warp) and the row loop
// sits inside the chunk loop: each lane keeps 8 independent row loads in
// flight per chunk and needs few registers, so more warps fit on an SM.
template <int G>
struct Walk4S {
    static_assert(G == 1 || G == 2, "Walk4S serves group sizes 1 and 2");
    static constexpr int D = 128;
    static constexpr int kChunk = 8;  // floats per lane per load (32 bytes)
    float* qs;  // this warp's slot: qs[h * 128 + e], scaled, natural order

    __device__ __forceinline__ void load_q(const __nv_bfloat16* const* qrow, float scale, int lane) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float x[4];
            Ld<__nv_bfloat16, 4>::run(qrow[h] + lane * 4, x);
            *reinterpret_cast<float4*>(qs + h * 128 + lane * 4) =
                make_float4(x[0] * scale, x[1] * scale, x[2] * scale, x[3] * scale);
        }
        __syncwarp();
    }

    __device__ __forceinline__ float score_internal(int cand, unsigned need, const float* child_lvl,
                                                    int64_t span_child, int64_t n_keys, int lane,
                                                    int variant = 0) const {
        const int g = lane >> 2, j = lane & 3;
        int cbase[4];      // first-child row offset (floats) of the group's 4 candidates, chunk j
        unsigned okm = 0;  // bit r: row r of the group exists and is wanted
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int c = 4 * g + jj;
            const int cc = __shfl_sync(kFull, cand, c);
            const bool want = (need >> c) & 1u;
            const int64_t row0 = 2 * (int64_t)cc;
            const bool ok0 = want && row0 * span_child < n_keys;
            const bool ok1 = want && (row0 + 1) * span_child < n_keys;
            okm |= (ok0 ? 1u : 0u) << (2 * jj);
            okm |= (ok1 ? 1u : 0u) << (2 * jj + 1);
            cbase[jj] = (int)((ok0 ? row0 : 0) * D) + j * kChunk;
        }
        // row r of the group: child r & 1 of candidate r >> 1 (a row that does
        // not exist reads an existing one; its dot is discarded)
        auto row_off = [&](int r) { return cbase[r >> 1] + ((((okm >> r) & 1u) && (r & 1)) ? D : 0); };
        auto row_ok = [&](int r) { return ((okm >> r) & 1u) != 0; };
        // two interleaved partial sums per (row, head), packed fp32x2 FMAs
        float2 acc[8 * G];
#pragma unroll
        for (int i = 0; i < 8 * G; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < D / (4 * kChunk); ++k) {
            const int e0 = (j + 4 * k) * kChunk;  // first element of this lane's chunk
            float4 qa[G], qb[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                qa[h] = *reinterpret_cast<const float4*>(qs + h * D + e0);
                qb[h] = *reinterpret_cast<const float4*>(qs + h * D + e0 + 4);
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float x[8];
                ldg_nc_v8(child_lvl + row_off(r) + 4 * kChunk * k, x);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float2 a = acc[r * G + h];
                    a = __ffma2_rn(make_float2(qa[h].x, qa[h].y), make_float2(x[0], x[1]), a);
                    a = __ffma2_rn(make_float2(qa[h].z, qa[h].w), make_float2(x[2], x[3]), a);
                    a = __ffma2_rn(make_float2(qb[h].x, qb[h].y), make_float2(x[4], x[5]), a);
                    a = __ffma2_rn(make_float2(qb[h].z, qb[h].w), make_float2(x[6], x[7]), a);
                    acc[r * G + h] = a;
                }
            }
        }
        float part[8 * G];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int h = 0; h < G; ++h) part[r * G + h] = row_ok(r) ? acc[r * G + h].x + acc[r * G + h].y : 0.f;
        constexpr int R = 2 * G;
        {
            const bool hi = (lane & 2) != 0;
#pragma unroll
            for (int i = 0; i < 2 * R; ++i) {
                const float send = hi ? part[i] : part[i + 2 * R];
                const float keep = hi ? part[i + 2 * R] : part[i];
                part[i] = keep + __shfl_xor_sync(kFull, send, 2);
            }
        }
        {
            const bool hi = (lane & 1) != 0;
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float send = hi ? part[i] : part[i + R];
                const float keep = hi ? part[i + R] : part[i];
                part[i] = keep + __shfl_xor_sync(kFull, send, 1);
            }
        }
        const bool mine = (need >> lane) & 1u;
        const bool has1 = (2 * (int64_t)cand + 1) * span_child < n_keys;
        float score = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) score += pair_score(part[h], has1 ? part[G + h] : -INFINITY, variant);
        return mine ? score : -INFINITY;
    }
};

}  // namespace pisa
