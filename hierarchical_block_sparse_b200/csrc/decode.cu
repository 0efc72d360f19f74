// decode.cu -- decode path (close reading §5.1 last paragraph; §5.3 "decode
// cache").
//
// append_kernel: one CTA (4 warps) per (b, kv-head) writes the new key/value
// row at pos[b], recomputes that leaf's mean from its cached rows and the new
// key, then each ancestor as the mean of its existing children: O(C + L) rows.
//
// decode_kernel: the single-stage fused step, one CTA (8 warps) per
// (b, kv-head). Warp 0 carries the walk's bookkeeping; at every scored level
// all warps compute the child dot products together (one round of gathers
// per level), all warps then split the leaf scoring (exact LSE over raw keys)
// and, after warp 0's final Top-K, the attention over the kept blocks;
// partial softmax states are merged through shared memory.
#include "pisa_internal.h"
#include "pisa_walk.cuh"
#include "tc.cuh"

namespace pisa {

// named barrier over `count` threads (a multiple of 32)
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}

// Summaries' update of one (b, kv-head) for the row at n: NWA warps (wi =
// this warp's index among them) write the new key/value row, fetch the leaf's
// cached rows before n (summed per warp, INFLIGHT loads in flight per lane)
// and the sibling of each ancestor into `scratch` ((NWA + kMaxLevels) x D
// floats of shared memory) -- none of which depends on the new row -- meet on
// named barrier `bar`, and warp 0 of them runs the chain leaf -> root.
template <typename T, int D, int NWA>
__device__ __forceinline__ void append_unit(T* Kh, T* Vh, float* P, const T* krow, const T* vrow, int64_t n,
                                            const DecodeParams& p, int wi, int lane, float* scratch, int bar) {
    constexpr int VD = D / 32;
    constexpr int INFLIGHT = 8;
    float* s_part = scratch;            // [NWA][D]
    float* s_sib = scratch + NWA * D;   // [kMaxLevels][D]
    float kn[VD];
    Ld<T, VD>::run(krow + lane * VD, kn);
    if (wi == 0) {
        float vn[VD];
        Ld<T, VD>::run(vrow + lane * VD, vn);
        store_vec<T, VD>(Kh + n * D + lane * VD, kn);
        store_vec<T, VD>(Vh + n * D + lane * VD, vn);
    }
    const int64_t leaf = n / p.C, lo = leaf * p.C;
    float acc[VD];
#pragma unroll
    for (int e = 0; e < VD; ++e) acc[e] = 0.f;
    for (int64_t r0 = lo + wi; r0 < n; r0 += NWA * INFLIGHT) {
        float x[INFLIGHT][VD];
#pragma unroll
        for (int i = 0; i < INFLIGHT; ++i) {
            const int64_t r = r0 + (int64_t)i * NWA;
            if (r < n) {
                Ld<T, VD>::run(Kh + r * D + lane * VD, x[i]);
            } else {
#pragma unroll
                for (int e = 0; e < VD; ++e) x[i][e] = 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < INFLIGHT; ++i)
#pragma unroll
            for (int e = 0; e < VD; ++e) acc[e] += x[i][e];
    }
#pragma unroll
    for (int e = 0; e < VD; ++e) s_part[wi * D + lane * VD + e] = acc[e];
    const int64_t len = n + 1;
    for (int l = 1 + wi; l < p.geom.L; l += NWA) {
        const int64_t sib = (leaf >> (l - 1)) ^ 1;
        if (sib * ((int64_t)p.C << (l - 1)) < len) {
            float sv[VD];
            Ld<float, VD>::run(P + (p.geom.off[l] + sib) * D + lane * VD, sv);
#pragma unroll
            for (int e = 0; e < VD; ++e) s_sib[(l - 1) * D + lane * VD + e] = sv[e];
        }
    }
    bar_sync(bar, NWA * 32);
    if (wi != 0) return;
    // leaf mean over [leaf*C, n]
    float m[VD];
    const float inv = 1.f / (float)(n - lo + 1);
#pragma unroll
    for (int e = 0; e < VD; ++e) {
        float sum = kn[e];
#pragma unroll
        for (int w = 0; w < NWA; ++w) sum += s_part[w * D + lane * VD + e];
        m[e] = sum * inv;
    }
    store_vec<float, VD>(P + (p.geom.off[1] + leaf) * D + lane * VD, m);
    // ancestors: mean of the existing children at length n + 1
    int64_t node = leaf;
    for (int l = 1; l < p.geom.L; ++l) {
        const int64_t sib = node ^ 1;
        if (sib * ((int64_t)p.C << (l - 1)) < len) {
#pragma unroll
            for (int e = 0; e < VD; ++e) m[e] = (m[e] + s_sib[(l - 1) * D + lane * VD + e]) * 0.5f;
        }
        node >>= 1;
        store_vec<float, VD>(P + (p.geom.off[l + 1] + node) * D + lane * VD, m);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(128) append_kernel(T* __restrict__ Kc, T* __restrict__ Vc,
                                                     float* __restrict__ pyr, const T* __restrict__ k_new,
                                                     const T* __restrict__ v_new, const int32_t* __restrict__ pos,
                                                     DecodeParams p) {
    __shared__ __align__(16) float scratch[(4 + kMaxLevels) * D];
    const int64_t unit = blockIdx.x;  // b * Hkv + kvh
    const int64_t b = unit / p.Hkv;
    const int64_t n = pos[b];
    if (n < 0 || n >= p.N) return;
    append_unit<T, D, 4>(Kc + unit * p.N * D, Vc + unit * p.N * D, pyr + unit * p.geom.rows * D, k_new + unit * D,
                         v_new + unit * D, n, p, threadIdx.x >> 5, threadIdx.x & 31, scratch, 0);
}

// Layout of the decode step. One CTA (8 warps) per (b, kv-head); every phase
// gives each thread a fixed slice of a row, so a row's dot product needs only
// a short shuffle reduction across the few threads that share the row:
//  * walk: pyramid rows (fp32) are gathered straight from global memory, TPRW
//    threads per row, 4 chunks of 16 bytes each;
//  * leaf scoring: the keys of every level-1 candidate leaf stream through a
//    CTA-wide cp.async pipeline of kDecStages tiles of kDecStageBytes; TPR
//    threads per row read 4 chunks each;
//  * attention: tiles of RowsC key rows and the same value rows; TPRC threads
//    per row read 2 key chunks and 2 value chunks each. The per-head
//    normaliser is known from the leaf LSEs, so p = 2^(z - Z) needs no
//    running max, and each thread accumulates p * v for its value chunks.
// Tile rows keep their 16-byte chunks XOR-swizzled so that the 8 threads of a
// shared-memory access phase hit distinct banks.
constexpr int kDecStageBytes = 16384;

template <typename T, int D>
struct DecLayout {
    static constexpr int EPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    static constexpr int CH = D / EPC;               // chunks per cache row (8, 16 or 32)
    static constexpr int RowBytes = D * (int)sizeof(T);
    static constexpr int TPR = CH / 4;               // leaf scoring: threads per row
    static constexpr int RowsB = 256 / TPR;          // rows per scoring tile
    static constexpr int TPRC = 2 * TPR;             // attention: threads per row
    static constexpr int RowsC = 256 / TPRC;         // rows per attention tile (keys; values alike)
    static constexpr int TPRW = D / 16;              // walk: threads per fp32 pyramid row
    static constexpr int RowsW = 256 / TPRW;         // pyramid rows per pass
    static_assert(RowsB * RowBytes == kDecStageBytes, "a scoring tile fills a stage");
    static_assert(2 * RowsC * RowBytes == kDecStageBytes, "an attention tile fills a stage");
    // byte offset of chunk c of row r in a tile whose rows are read by `tpr` threads
    __device__ __forceinline__ static int off(int r, int c, int tpr) {
        const int sw = tpr < 8 ? (8 / tpr) : 1;
        return r * RowBytes + ((c ^ ((r % sw) * tpr)) << 4);
    }
};

// 16 bytes of T widened to EPC floats
template <typename T>
__device__ __forceinline__ void widen16(const uint4& v, float* o) {
    if constexpr (sizeof(T) == 4) {
        o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
    } else {
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
}

// cp.async of `nrows` cache rows into a swizzled tile read by `tpr` threads per row
template <typename T, int D>
__device__ __forceinline__ void stage_rows(uint32_t dst, const T* src, int nrows, int tpr, int tid) {
    using Lo = DecLayout<T, D>;
    const uint8_t* s = reinterpret_cast<const uint8_t*>(src);
    for (int i = tid; i < nrows * Lo::CH; i += 256) {
        const int r = i / Lo::CH, c = i - r * Lo::CH;
        tc::cp_async16(dst + Lo::off(r, c, tpr), s + (size_t)i * 16);
    }
}

// merge two (max, sum) log2-domain softmax states
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
    const float mn = fmaxf(m, m2);
    s = (mn == -INFINITY) ? 0.f : s * exp2f(m - mn) + s2 * exp2f(m2 - mn);
    m = mn;
}

// CTAs per SM the decode kernel is sized for: with G <= 2 four CTAs of 8
// warps fit (64 registers a thread, under 57 KB of shared memory each), so a
// step of up to 4 * 148 (b, kv-head) units runs in one wave.
template <int G>
constexpr int decode_min_blocks() { return G <= 2 ? 4 : (G <= 4 ? 2 : 1); }

// With one head per group (G = 1) and leaves of at most kDecCacheKeys keys, the
// scoring pass keeps every candidate key's logit in shared memory
// ([32 leaves][kDecCacheKeys]), so the attention streams only the values of
// the kept leaves; that variant runs a 2-stage pipeline to make room (still
// 8 stages of 16 KB in flight per SM).
constexpr int kDecCacheKeys = 64;
template <int G>
constexpr bool decode_caches() { return G == 1; }
template <int G>
constexpr int decode_stages() { return decode_caches<G>() ? 2 : 3; }

template <typename T, int D, int G>
__global__ void __launch_bounds__(256, decode_min_blocks<G>()) decode_kernel(
    const T* __restrict__ q_new, T* __restrict__ Kc, T* __restrict__ Vc, float* __restrict__ pyr,
    const int32_t* __restrict__ pos, int32_t* __restrict__ idx, T* __restrict__ out, const T* __restrict__ k_new,
    const T* __restrict__ v_new, DecodeParams p) {
    using Lo = DecLayout<T, D>;
    constexpr int NW = 8;
    constexpr int kDecStages = decode_stages<G>();
    constexpr int EPC = Lo::EPC, TPR = Lo::TPR, TPRC = Lo::TPRC, TPRW = Lo::TPRW;
    extern __shared__ __align__(16) uint8_t dsm[];  // pipeline stages, then [NW][G][D] partial outputs
    __shared__ __align__(16) float s_q[G][D];       // scaled queries of the group
    __shared__ int s_cand[32];
    __shared__ float s_dot[64][G];
    __shared__ float s_lse[32][G];                  // per candidate slot and head (log2)
    __shared__ int s_sel[32], s_slot[32];
    __shared__ unsigned s_need;
    __shared__ int s_level, s_nlist;
    __shared__ float s_Z[G];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // per-warp states of the listed leaves, after the pipeline stages: the LSE
    // (max, sum) and, for the PISA-1 / PISA-2 ranking, the logits' moments
    using Part = float[32][NW][G];
    Part& s_pm = *reinterpret_cast<Part*>(dsm + kDecStages * kDecStageBytes);
    Part& s_ps = *reinterpret_cast<Part*>(dsm + kDecStages * kDecStageBytes + sizeof(Part));
    Part& s_vn = *reinterpret_cast<Part*>(dsm + kDecStages * kDecStageBytes + 2 * sizeof(Part));
    Part& s_vmean = *reinterpret_cast<Part*>(dsm + kDecStages * kDecStageBytes + 3 * sizeof(Part));
    Part& s_vm2 = *reinterpret_cast<Part*>(dsm + kDecStages * kDecStageBytes + 4 * sizeof(Part));
    // cached logits [32][kDecCacheKeys] (G = 1, C <= kDecCacheKeys), after the leaf states
    float* s_logit = reinterpret_cast<float*>(dsm + kDecStages * kDecStageBytes + 5 * sizeof(Part));
    const bool cached = decode_caches<G>() && p.C <= kDecCacheKeys;
    __shared__ int s_kj[32];  // for each kept leaf, its index in the scored list
    const int64_t unit = blockIdx.x;  // b * Hkv + kvh
    const int64_t b = unit / p.Hkv;
    const int kvh = (int)(unit - b * p.Hkv);
    const int64_t t = pos[b];
    if (t < 0 || t >= p.N) {
        if (tid < p.K) idx[unit * p.K + tid] = -1;
        for (int i = tid; i < G * D; i += blockDim.x) out[((b * p.Hq + (int64_t)kvh * G) * D) + i] = (T)0.f;
        return;
    }
    const int64_t n_keys = t + 1;
    const T* Kh = Kc + unit * p.N * D;
    const T* Vh = Vc + unit * p.N * D;
    const float* P = pyr + unit * p.geom.rows * D;
    const Forced F(t, p.C, 1, p.forced_mask);
    for (int i = tid; i < G * D; i += blockDim.x) {
        const int h = i / D;
        s_q[h][i - h * D] = (float)q_new[(b * p.Hq + (int64_t)kvh * G + h) * D + (i - h * D)] * p.qscale;
    }
    __syncthreads();
    // Fused append (k_new given): warps 1..7 write the new row and update the
    // current leaf's summary and its ancestors, in the stage buffers' space,
    // while warp 0 passes the first levels of the walk. The walk never reads
    // those rows: they are the forced path (never scored), and the parent of
    // an ancestor is an ancestor. The new key/value row is read back only by
    // the attention, after later barriers.
    if (k_new != nullptr && warp >= 1)
        append_unit<T, D, NW - 1>(Kc + unit * p.N * D, Vc + unit * p.N * D, pyr + unit * p.geom.rows * D,
                                  k_new + unit * D, v_new + unit * D, t, p, warp - 1, lane,
                                  reinterpret_cast<float*>(dsm), 1);

    // ---- internal levels. Warp 0 carries the walk (lane c = candidate c,
    // valid candidates in ascending node order) and passes alone through the
    // levels that need no dot products; at a scored level all threads compute
    // the <= 64 child dots into s_dot.
    int cand = lane == 0 ? 0 : -1;  // warp 0's walk state
    int l = p.geom.L;
    for (;;) {
        if (warp == 0) {
            unsigned need = 0;
            for (; l >= 2; --l) {
                const LevelState s = level_state(cand, l, p.C, n_keys, t, 1, F);
                if (s.n <= p.K) {
                    const int parent = compact_by_rank(cand, s.vmask, lane >> 1);
                    cand = lane < 2 * s.n ? 2 * parent + (lane & 1) : -1;
                    continue;
                }
                const unsigned fmask = __ballot_sync(kFull, s.forced);
                if (__popc(fmask) >= p.K) {  // the forced nodes fill the budget
                    int id = cand;
                    const int kept = keep_topk_lane(id, s.forced ? INFINITY : -INFINITY, s.valid, p.K, lane);
                    const int parent = __shfl_sync(kFull, id, lane >> 1);
                    cand = lane < 2 * kept ? 2 * parent + (lane & 1) : -1;
                    continue;
                }
                need = s.vmask & ~fmask;
                break;
            }
            s_cand[lane] = cand;
            if (lane == 0) {
                s_level = l;
                s_need = need;
            }
        }
        __syncthreads();
        const int lv = s_level;
        if (lv < 2) break;
        {
            const unsigned need = s_need;
            const int64_t span_child = (int64_t)p.C << (lv - 2);
            const float* child_lvl = P + p.geom.off[lv - 1] * D;
            const int sl = tid % TPRW;
#pragma unroll
            for (int r0 = 0; r0 < 64; r0 += Lo::RowsW) {
                const int rho = r0 + tid / TPRW, c = rho >> 1;
                const int64_t child = 2 * (int64_t)s_cand[c] + (rho & 1);
                const bool ok = ((need >> c) & 1u) && child * span_child < n_keys;
                float acc[G];
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = 0.f;
                if (ok) {
                    const float4* row = reinterpret_cast<const float4*>(child_lvl + child * D);
                    float4 x[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) x[k] = __ldg(row + sl + TPRW * k);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int e0 = (sl + TPRW * k) * 4;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float4 qv = *reinterpret_cast<const float4*>(&s_q[h][e0]);
                            acc[h] = fmaf(qv.x, x[k].x, fmaf(qv.y, x[k].y, fmaf(qv.z, x[k].z, fmaf(qv.w, x[k].w, acc[h]))));
                        }
                    }
                }
#pragma unroll
                for (int o = 1; o < TPRW; o <<= 1)
#pragma unroll
                    for (int h = 0; h < G; ++h) acc[h] += __shfl_xor_sync(kFull, acc[h], o);
                if (sl == 0)
#pragma unroll
                    for (int h = 0; h < G; ++h) s_dot[rho][h] = acc[h];
            }
        }
        __syncthreads();
        if (warp == 0) {  // scores (Eq.7, summed over the group: Eq.11) and the keep
            const LevelState s = level_state(cand, l, p.C, n_keys, t, 1, F);
            const bool mine = (s_need >> lane) & 1u;
            float score = -INFINITY;
            if (mine) {
                const bool has1 = (2 * (int64_t)cand + 1) * ((int64_t)p.C << (l - 2)) < n_keys;
                score = 0.f;
#pragma unroll
                for (int h = 0; h < G; ++h)
                    score += pair_score(s_dot[2 * lane][h], has1 ? s_dot[2 * lane + 1][h] : -INFINITY, p.variant);
            }
            int id = cand;
            const int kept = keep_topk_lane(id, s.forced ? INFINITY : score, s.valid, p.K, lane);
            const int parent = __shfl_sync(kFull, id, lane >> 1);
            cand = lane < 2 * kept ? 2 * parent + (lane & 1) : -1;
            --l;
        }
    }

    // ---- leaves: exact LSE (per head) over the raw keys of every valid
    // candidate -- the non-forced ones are ranked by it, and the kept ones
    // give the attention's normaliser.
    uint8_t* stage = dsm;
    const uint32_t stage0 = tc::smem_u32(stage);
    if (warp == 0) {
        const LevelState s = level_state(cand, 1, p.C, n_keys, t, 1, F);
        if (s.valid) {
            const int j = __popc(s.vmask & ((1u << lane) - 1u));
            s_sel[j] = cand;
            s_slot[j] = lane;
        }
        if (lane == 0) s_nlist = s.n;
    }
    __syncthreads();
    {
        const int nlist = s_nlist;
        const int tpl = (p.C + Lo::RowsB - 1) / Lo::RowsB;  // tiles per leaf
        const int ntiles = nlist * tpl;
        auto rows_of = [&](int tile, int64_t& lo) {
            const int64_t leaf = s_sel[tile / tpl];
            lo = leaf * p.C + (int64_t)(tile % tpl) * Lo::RowsB;
            return (int)(min(min(leaf * p.C + p.C, n_keys), lo + Lo::RowsB) - lo);
        };
        auto issue = [&](int tile) {
            if (tile < ntiles) {
                int64_t lo;
                const int n = rows_of(tile, lo);
                stage_rows<T, D>(stage0 + (tile % kDecStages) * kDecStageBytes, Kh + lo * D, n, TPR, tid);
            }
            tc::cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < kDecStages - 1; ++i) issue(i);
        const int r = tid / TPR, sl = tid % TPR;
        for (int tile = 0; tile < ntiles; ++tile) {
            // tile's copies have landed; after the barrier every warp is done
            // with the buffer of tile - 1, which the next issue refills
            tc::cp_async_wait_group<kDecStages - 2>();
            __syncthreads();
            issue(tile + kDecStages - 1);
            const int j = tile / tpl;
            int64_t lo;
            const int nrows = rows_of(tile, lo);
            const uint8_t* buf = stage + (tile % kDecStages) * kDecStageBytes;
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
            if (r < nrows) {
                uint4 raw[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) raw[k] = *reinterpret_cast<const uint4*>(buf + Lo::off(r, sl + TPR * k, TPR));
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float x[EPC];
                    widen16<T>(raw[k], x);
                    const int e0 = (sl + TPR * k) * EPC;
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < EPC; e += 4) {
                            const float4 qv = *reinterpret_cast<const float4*>(&s_q[h][e0 + e]);
                            acc[h] = fmaf(qv.x, x[e], fmaf(qv.y, x[e + 1], fmaf(qv.z, x[e + 2], fmaf(qv.w, x[e + 3], acc[h]))));
                        }
                }
            }
#pragma unroll
            for (int o = 1; o < TPR; o <<= 1)
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] += __shfl_xor_sync(kFull, acc[h], o);
            if (cached && sl == 0 && r < nrows) s_logit[j * kDecCacheKeys + (tile % tpl) * Lo::RowsB + r] = acc[0];
            // this warp's rows: max and sum of 2^(z - max) per head, one lane per row counting
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float z = r < nrows ? acc[h] : -INFINITY;
                float m = z;
#pragma unroll
                for (int o = TPR; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
                float e = (sl == 0 && z != -INFINITY) ? exp2f(z - m) : 0.f;
#pragma unroll
                for (int o = TPR; o < 32; o <<= 1) e += __shfl_xor_sync(kFull, e, o);
                if (lane == 0) {  // this warp's running state of leaf j (its tiles come in order)
                    float mm = m, ss = e;
                    if (tile % tpl != 0) lse_merge(mm, ss, s_pm[j][warp][h], s_ps[j][warp][h]);
                    s_pm[j][warp][h] = mm;
                    s_ps[j][warp][h] = ss;
                }
                if (p.variant) {  // moments of this warp's logits (two passes), merged likewise
                    const bool live = z != -INFINITY && sl == 0;
                    float cnt = live ? 1.f : 0.f, sum = live ? z : 0.f;
#pragma unroll
                    for (int o = TPR; o < 32; o <<= 1) {
                        cnt += __shfl_xor_sync(kFull, cnt, o);
                        sum += __shfl_xor_sync(kFull, sum, o);
                    }
                    const float mean = cnt > 0.f ? sum / cnt : 0.f;
                    float dev = live ? (z - mean) * (z - mean) : 0.f;
#pragma unroll
                    for (int o = TPR; o < 32; o <<= 1) dev += __shfl_xor_sync(kFull, dev, o);
                    if (lane == 0) {
                        Moments mo;
                        if (tile % tpl != 0) {
                            mo.n = s_vn[j][warp][h];
                            mo.mean = s_vmean[j][warp][h];
                            mo.m2 = s_vm2[j][warp][h];
                        }
                        mo.merge(cnt, mean, dev);
                        s_vn[j][warp][h] = mo.n;
                        s_vmean[j][warp][h] = mo.mean;
                        s_vm2[j][warp][h] = mo.m2;
                    }
                }
            }
        }
        tc::cp_async_wait_all();
        __syncthreads();
        if (tid < nlist * G) {  // leaf LSE per head (and the PISA-1 / PISA-2 score in s_dot)
            const int j = tid / G, h = tid - j * G;
            float m = -INFINITY, sm = 0.f;
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) lse_merge(m, sm, s_pm[j][ww][h], s_ps[j][ww][h]);
            s_lse[s_slot[j]][h] = m + log2f(sm);
            if (p.variant) {
                Moments mo;
#pragma unroll
                for (int ww = 0; ww < NW; ++ww) mo.merge(s_vn[j][ww][h], s_vmean[j][ww][h], s_vm2[j][ww][h]);
                s_dot[s_slot[j]][h] = mo.score(p.variant);
            }
        }
    }
    __syncthreads();

    if (warp == 0) {  // final Top-K (kept leaves come out in ascending order), then Z per head
        const LevelState s = level_state(cand, 1, p.C, n_keys, t, 1, F);
        float score = 0.f;  // ranking: the LSE or the PISA-1 / PISA-2 score, summed over the group (Eq.11)
#pragma unroll
        for (int h = 0; h < G; ++h) score += s.valid ? (p.variant ? s_dot[lane][h] : s_lse[lane][h]) : 0.f;
        int id = cand, kept;
        unsigned kmask;
        if (s.n <= p.K) {
            kmask = s.vmask;
            id = compact_by_rank(cand, s.vmask, lane);
            kept = s.n;
        } else {
            kept = keep_topk_lane(id, s.forced ? INFINITY : score, s.valid, p.K, lane);
            // kept-ness per candidate lane: the kept ids are in lanes 0..kept-1
            bool mine = false;
            for (int i = 0; i < kept; ++i) mine |= (__shfl_sync(kFull, id, i) == cand) && s.valid;
            kmask = __ballot_sync(kFull, mine);
        }
        const int out_id = lane < kept ? id : -1;
        if (lane < p.K) idx[unit * p.K + lane] = out_id;
        if ((kmask >> lane) & 1u)  // kept candidate lane -> (its rank among the kept, among the scored)
            s_kj[__popc(kmask & ((1u << lane) - 1u))] = __popc(s.vmask & ((1u << lane) - 1u));
        s_sel[lane] = lane < p.K ? out_id : -1;
        if (lane == 0) s_nlist = min(kept, p.K);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float x = ((kmask >> lane) & 1u) ? s_lse[lane][h] : -INFINITY;
            float m = x;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
            float e = x == -INFINITY ? 0.f : exp2f(x - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(kFull, e, o);
            if (lane == 0) s_Z[h] = m + log2f(e);
        }
    }
    __syncthreads();

    // ---- attention over the kept leaves
    constexpr int VE = 2 * EPC;  // value elements per thread per row
    float o[G][VE], lsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        lsum[h] = 0.f;
#pragma unroll
        for (int e = 0; e < VE; ++e) o[h][e] = 0.f;
    }
    const int rc = tid / TPRC, sc = tid % TPRC;
    {
        float Z[G];
#pragma unroll
        for (int h = 0; h < G; ++h) Z[h] = s_Z[h];
        const int nkept = s_nlist;
        const int tpl = (p.C + Lo::RowsC - 1) / Lo::RowsC;
        const int ntiles = nkept * tpl;
        auto rows_of = [&](int tile, int64_t& lo) {
            const int64_t blk = s_sel[tile / tpl];
            lo = blk * p.C + (int64_t)(tile % tpl) * Lo::RowsC;
            const int64_t hi = min(min(blk * p.C + p.C, n_keys), lo + Lo::RowsC);
            return (int)max(hi - lo, (int64_t)0);
        };
        auto issue = [&](int tile) {
            if (tile < ntiles) {
                int64_t lo;
                const int n = rows_of(tile, lo);
                const uint32_t dst = stage0 + (tile % kDecStages) * kDecStageBytes;
                if (!cached) stage_rows<T, D>(dst, Kh + lo * D, n, TPRC, tid);
                stage_rows<T, D>(dst + kDecStageBytes / 2, Vh + lo * D, n, TPRC, tid);
            }
            tc::cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < kDecStages - 1; ++i) issue(i);
        for (int tile = 0; tile < ntiles; ++tile) {
            tc::cp_async_wait_group<kDecStages - 2>();
            __syncthreads();
            issue(tile + kDecStages - 1);
            int64_t lo;
            const int nrows = rows_of(tile, lo);
            const uint8_t* kbuf = stage + (tile % kDecStages) * kDecStageBytes;
            const uint8_t* vbuf = kbuf + kDecStageBytes / 2;
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
            const bool live = rc < nrows;
            if (cached) {  // the logit from the scoring pass (every lane of the row reads it)
                if (live) acc[0] = s_logit[s_kj[tile / tpl] * kDecCacheKeys + (tile % tpl) * Lo::RowsC + rc];
            } else if (live) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float x[EPC];
                    widen16<T>(*reinterpret_cast<const uint4*>(kbuf + Lo::off(rc, sc + TPRC * k, TPRC)), x);
                    const int e0 = (sc + TPRC * k) * EPC;
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < EPC; e += 4) {
                            const float4 qv = *reinterpret_cast<const float4*>(&s_q[h][e0 + e]);
                            acc[h] = fmaf(qv.x, x[e], fmaf(qv.y, x[e + 1], fmaf(qv.z, x[e + 2], fmaf(qv.w, x[e + 3], acc[h]))));
                        }
                }
            }
            if (!cached) {
#pragma unroll
                for (int o2 = 1; o2 < TPRC; o2 <<= 1)
#pragma unroll
                    for (int h = 0; h < G; ++h) acc[h] += __shfl_xor_sync(kFull, acc[h], o2);
            }
            if (live) {
                float pr[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    pr[h] = exp2f(acc[h] - Z[h]);
                    lsum[h] += pr[h];
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float x[EPC];
                    widen16<T>(*reinterpret_cast<const uint4*>(vbuf + Lo::off(rc, sc + TPRC * k, TPRC)), x);
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < EPC; ++e) o[h][k * EPC + e] = fmaf(pr[h], x[e], o[h][k * EPC + e]);
                }
            }
        }
        tc::cp_async_wait_all();
    }
    // sum over the rows a warp holds (lanes with the same slice), then over warps
#pragma unroll
    for (int off = TPRC; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h) {
            lsum[h] += __shfl_xor_sync(kFull, lsum[h], off);
#pragma unroll
            for (int e = 0; e < VE; ++e) o[h][e] += __shfl_xor_sync(kFull, o[h][e], off);
        }
    __syncthreads();  // the stage buffers are free: reuse them for the partial outputs
    float* part = reinterpret_cast<float*>(dsm);  // [NW][G][D + 1]: outputs, then the row sum
    if (lane < TPRC) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
                for (int e = 0; e < EPC; ++e) part[(warp * G + h) * (D + 1) + (sc + TPRC * k) * EPC + e] = o[h][k * EPC + e];
            if (sc == 0) part[(warp * G + h) * (D + 1) + D] = lsum[h];
        }
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += blockDim.x) {
        const int h = i / D, d = i - h * D;
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) {
            num += part[(ww * G + h) * (D + 1) + d];
            den += part[(ww * G + h) * (D + 1) + D];
        }
        out[((b * p.Hq + (int64_t)kvh * G) * D) + i] = (T)(den > 0.f ? num / den : 0.f);
    }
}

template <typename T, int D>
static cudaError_t launch_append_t(void* Kc, void* Vc, float* pyr, const void* k_new, const void* v_new,
                                   const int32_t* pos, const DecodeParams& p, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Hkv;
    append_kernel<T, D><<<(unsigned)units, 128, 0, st>>>((T*)Kc, (T*)Vc, pyr, (const T*)k_new, (const T*)v_new,
                                                          pos, p);
    return cudaGetLastError();
}

cudaError_t launch_append(int dtype, int d, void* Kc, void* Vc, float* pyr, const void* k_new, const void* v_new,
                          const int32_t* pos, const DecodeParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_append_t<__nv_bfloat16, 128>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
        if (d == 64) return launch_append_t<__nv_bfloat16, 64>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
    } else {
        if (d == 128) return launch_append_t<float, 128>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
        if (d == 64) return launch_append_t<float, 64>(Kc, Vc, pyr, k_new, v_new, pos, p, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int D, int G>
static cudaError_t launch_decode_t(const void* q, void* Kc, void* Vc, float* pyr, const int32_t* pos, int32_t* idx,
                                   void* o, const void* k_new, const void* v_new, const DecodeParams& p,
                                   cudaStream_t st) {
    const size_t out_bytes = sizeof(float) * 8 * G * (D + 1);
    // pipeline stages + five per-warp arrays [32][8][G] of leaf states (+ the cached logits)
    const size_t stage_bytes = (size_t)decode_stages<G>() * kDecStageBytes + 5 * sizeof(float) * 32 * 8 * G +
                               (decode_caches<G>() ? sizeof(float) * 32 * kDecCacheKeys : 0);
    const size_t smem = out_bytes > stage_bytes ? out_bytes : stage_bytes;
    auto kern = decode_kernel<T, D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // the pipeline stages of decode_min_blocks<G>() CTAs must fit in one SM's shared memory
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((int64_t)p.B * p.Hkv), 256, smem, st>>>((const T*)q, (T*)Kc, (T*)Vc, pyr, pos, idx, (T*)o,
                                                               (const T*)k_new, (const T*)v_new, p);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_decode_d(const void* q, void* Kc, void* Vc, float* pyr, const int32_t* pos, int32_t* idx,
                                   void* o, const void* k_new, const void* v_new, const DecodeParams& p,
                                   cudaStream_t st) {
    switch (p.Hq / p.Hkv) {
        case 1: return launch_decode_t<T, D, 1>(q, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
        case 2: return launch_decode_t<T, D, 2>(q, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
        case 4: return launch_decode_t<T, D, 4>(q, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
        case 8: return launch_decode_t<T, D, 8>(q, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
        case 16: return launch_decode_t<T, D, 16>(q, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
    }
    return cudaErrorInvalidValue;
}

// k_new / v_new null: decode only (the row at pos was appended before);
// otherwise the append runs inside the same kernel.
cudaError_t launch_decode(int dtype, int d, const void* q_new, void* Kc, void* Vc, float* pyr, const int32_t* pos,
                          int32_t* idx, void* o, const void* k_new, const void* v_new, const DecodeParams& p,
                          cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_decode_d<__nv_bfloat16, 128>(q_new, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
        if (d == 64) return launch_decode_d<__nv_bfloat16, 64>(q_new, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
    } else {
        if (d == 128) return launch_decode_d<float, 128>(q_new, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
        if (d == 64) return launch_decode_d<float, 64>(q_new, Kc, Vc, pyr, pos, idx, o, k_new, v_new, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
