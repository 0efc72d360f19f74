// api.cu -- the extern "C" boundary declared in include/pisa.h: argument
// validation on the host, geometry, and dispatch to the kernel launchers.
// Nothing is enqueued unless every check passes; no call allocates memory.
#include <math.h>
#include <stdint.h>

#include "pisa.h"
#include "pisa_internal.h"

using namespace pisa;

namespace {

// checks that need no device: the problem statement itself
int check_cfg(const pisa_cfg* c) {
    if (!c) return PISA_E_INVALID;
    if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->N < 0 || c->d < 1 || c->C < 1 || c->K < 1 || c->g < 2)
        return PISA_E_INVALID;
    if (c->Hq % c->Hkv != 0) return PISA_E_INVALID;
    if (c->causal != 0 && c->causal != 1) return PISA_E_INVALID;
    if (c->forced_mask < 0 || c->forced_mask > 7) return PISA_E_INVALID;
    if (c->dtype != PISA_DTYPE_F32 && c->dtype != PISA_DTYPE_BF16) return PISA_E_INVALID;
    if (c->score_variant < PISA_SCORE_LSE || c->score_variant > PISA_SCORE_MEAN_VAR) return PISA_E_INVALID;
    const int forced = c->forced_mask | (c->causal ? 4 : 0);
    const int nf = (forced & 1) + ((forced >> 1) & 1) + ((forced >> 2) & 1);
    if (c->K < nf) return PISA_E_INVALID;  // forced leaves count against K (Eq.6)
    return PISA_OK;
}

// limits of the GPU kernels
int check_gpu(const pisa_cfg* c) {
    int s = check_cfg(c);
    if (s) return s;
    if (c->g != 2) return PISA_E_UNSUPPORTED;
    if (c->d != 64 && c->d != 128) return PISA_E_UNSUPPORTED;
    if (c->K > 16) return PISA_E_UNSUPPORTED;
    if (c->C > 1024) return PISA_E_UNSUPPORTED;
    const int G = c->Hq / c->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return PISA_E_UNSUPPORTED;
    Geom g;
    if (make_geom(c->N, c->C, &g) < 0) return PISA_E_UNSUPPORTED;
    return PISA_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
// the block-major stage 1 reads pyramid rows with 256-bit loads
bool aligned32(const void* p) { return ((uintptr_t)p & 31u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PISA_OK : PISA_E_CUDA; }

// generic geometry for any g >= 2 (host only)
int geom_any(const pisa_cfg* c, int64_t* M, int64_t* off, int maxl) {
    if (c->N == 0) return 0;
    int L = 1;
    M[1] = ((int64_t)c->N + c->C - 1) / c->C;
    off[1] = 0;
    while (M[L] > 1) {
        if (L + 1 > maxl) return -1;
        M[L + 1] = (M[L] + c->g - 1) / c->g;
        off[L + 1] = off[L] + M[L];
        ++L;
    }
    return L;
}

SelectParams select_params(const pisa_cfg* c, const Geom& g) {
    SelectParams p = select_params_of(c);
    p.geom = g;
    return p;
}

PoolParams pool_params(const pisa_cfg* c, const Geom& g, const int32_t* len) {
    PoolParams p;
    p.B = c->B; p.Hkv = c->Hkv; p.N = c->N; p.C = c->C;
    p.k_rows = c->N;
    p.len = len;
    p.geom = g;
    return p;
}

// limits of the block-major tensor-core path
int check_bm(const pisa_cfg* c) {
    int s = check_gpu(c);
    if (s) return s;
    if (c->dtype != PISA_DTYPE_BF16 || c->d != 128 || c->C != 64) return PISA_E_UNSUPPORTED;
    if (c->N >= (1 << 27)) return PISA_E_UNSUPPORTED;
    if ((int64_t)c->B * c->Hkv * c->N * 32 >= ((int64_t)1 << 31)) return PISA_E_UNSUPPORTED;
    if ((int64_t)c->B * c->Hkv > 65535) return PISA_E_UNSUPPORTED;  // one grid row per (b, kv-head)
    return PISA_OK;
}

BmShape bm_shape(const pisa_cfg* c) { return bm_shape_of(c); }

int check_ws(const pisa_cfg* c, const void* ws, size_t bytes) {
    if (!ws) return PISA_E_INVALID;
    if (((uintptr_t)ws & 255u) != 0) return PISA_E_ALIGNMENT;
    if (bytes < blockmajor_layout(bm_shape(c)).total) return PISA_E_INVALID;
    return PISA_OK;
}

// every check pisa_forward_ws makes, before anything is enqueued
int check_forward_ws(const pisa_cfg* c, const void* Q, const void* K, const void* V, const float* pyr,
                     const int32_t* idx, const void* O, const void* ws, size_t bytes) {
    int s = check_bm(c);
    if (s) return s;
    if (c->N == 0) return PISA_OK;
    if (!Q || !K || !V || !pyr || !idx || !O) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned32(pyr) || !aligned16(idx) || !aligned16(O))
        return PISA_E_ALIGNMENT;
    return check_ws(c, ws, bytes);
}

// checks of a pyramid re-layout from cfg_old's capacity to cfg_new's
int check_grow(const pisa_cfg* o, const pisa_cfg* n) {
    int s = check_gpu(o);
    if (s) return s;
    s = check_gpu(n);
    if (s) return s;
    if (o->B != n->B || o->Hq != n->Hq || o->Hkv != n->Hkv || o->d != n->d || o->C != n->C || o->g != n->g ||
        o->dtype != n->dtype || n->N < o->N)
        return PISA_E_INVALID;
    return PISA_OK;
}
int check_grow_pyramids(const float* pyr_old, const float* pyr_new) {
    if (!pyr_old || !pyr_new || pyr_old == pyr_new) return PISA_E_INVALID;
    if (!aligned16(pyr_old) || !aligned16(pyr_new)) return PISA_E_ALIGNMENT;
    return PISA_OK;
}

DecodeParams decode_params(const pisa_cfg* c, const Geom& g) {
    DecodeParams p;
    p.B = c->B; p.Hq = c->Hq; p.Hkv = c->Hkv; p.N = c->N; p.C = c->C; p.K = c->K;
    p.forced_mask = c->forced_mask;
    p.qscale = (float)(1.4426950408889634 / sqrt((double)c->d));
    p.geom = g;
    p.variant = c->score_variant;
    return p;
}

}  // namespace

extern "C" {

int pisa_num_levels(const pisa_cfg* cfg) {
    int s = check_cfg(cfg);
    if (s) return s;
    int64_t M[65], off[65];
    int L = geom_any(cfg, M, off, 64);
    return L < 0 ? PISA_E_UNSUPPORTED : L;
}

int64_t pisa_level_nodes(const pisa_cfg* cfg, int level) {
    int s = check_cfg(cfg);
    if (s) return s;
    int64_t M[65], off[65];
    int L = geom_any(cfg, M, off, 64);
    if (L < 0) return PISA_E_UNSUPPORTED;
    if (level < 1 || level > L) return PISA_E_INVALID;
    return M[level];
}

int64_t pisa_level_offset(const pisa_cfg* cfg, int level) {
    int s = check_cfg(cfg);
    if (s) return s;
    int64_t M[65], off[65];
    int L = geom_any(cfg, M, off, 64);
    if (L < 0) return PISA_E_UNSUPPORTED;
    if (level < 1 || level > L) return PISA_E_INVALID;
    return off[level];
}

int64_t pisa_pyramid_rows(const pisa_cfg* cfg) {
    int s = check_cfg(cfg);
    if (s) return s;
    int64_t M[65], off[65];
    int L = geom_any(cfg, M, off, 64);
    if (L < 0) return PISA_E_UNSUPPORTED;
    return L == 0 ? 0 : off[L] + M[L];
}

int pisa_build_pyramid(const pisa_cfg* cfg, const void* K, float* pyr, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!K || !pyr) return PISA_E_INVALID;
    if (!aligned16(K) || !aligned16(pyr)) return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_pool(cfg->dtype, cfg->d, K, pyr, pool_params(cfg, g, nullptr), (cudaStream_t)stream));
}

int pisa_select(const pisa_cfg* cfg, const void* Q, const void* K, const float* pyr, int32_t* idx, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !pyr || !idx) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(pyr) || !aligned16(idx)) return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_select(cfg->dtype, cfg->d, Q, K, pyr, idx, select_params(cfg, g), (cudaStream_t)stream));
}

int pisa_sparse_attn(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                     void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !V || !idx || !O) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(O)) return PISA_E_ALIGNMENT;
    AttnParams p;
    p.B = cfg->B; p.Hq = cfg->Hq; p.Hkv = cfg->Hkv; p.N = cfg->N; p.C = cfg->C; p.K = cfg->K;
    p.causal = cfg->causal;
    p.qscale = (float)(1.4426950408889634 / sqrt((double)cfg->d));
    return cuda_status(launch_attn(cfg->dtype, cfg->d, Q, K, V, idx, O, p, (cudaStream_t)stream));
}

int pisa_sparse_attn_backward(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, const int32_t* idx,
                              const void* dO, float* dQ, float* dK, float* dV, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !V || !idx || !dO || !dQ || !dK || !dV) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV))
        return PISA_E_ALIGNMENT;
    const size_t kv_bytes = (size_t)cfg->B * cfg->Hkv * cfg->N * cfg->d * sizeof(float);
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(dK, 0, kv_bytes, st) != cudaSuccess || cudaMemsetAsync(dV, 0, kv_bytes, st) != cudaSuccess)
        return PISA_E_CUDA;
    AttnParams p;
    p.B = cfg->B; p.Hq = cfg->Hq; p.Hkv = cfg->Hkv; p.N = cfg->N; p.C = cfg->C; p.K = cfg->K;
    p.causal = cfg->causal;
    p.qscale = (float)(1.4426950408889634 / sqrt((double)cfg->d));
    return cuda_status(launch_attn_bwd(cfg->dtype, cfg->d, Q, K, V, idx, dO, dQ, dK, dV, p, st));
}

int pisa_forward(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, float* pyr, int32_t* idx, void* O,
                 void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !V || !pyr || !idx || !O) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(pyr) || !aligned16(idx) || !aligned16(O))
        return PISA_E_ALIGNMENT;
    s = pisa_build_pyramid(cfg, K, pyr, stream);
    if (s) return s;
    s = pisa_select(cfg, Q, K, pyr, idx, stream);
    if (s) return s;
    return pisa_sparse_attn(cfg, Q, K, V, idx, O, stream);
}

int pisa_bsa_select(const pisa_cfg* cfg, const void* Q, const float* pyr, int32_t* idx, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !pyr || !idx) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(pyr) || !aligned16(idx)) return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_bsa(cfg->dtype, cfg->d, Q, pyr, idx, select_params(cfg, g), (cudaStream_t)stream));
}

int pisa_bsa_select_ws(const pisa_cfg* cfg, const void* Q, const float* pyr, int32_t* idx, void* workspace,
                       size_t workspace_bytes, void* stream) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !pyr || !idx) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(pyr) || !aligned16(idx)) return PISA_E_ALIGNMENT;
    s = check_ws(cfg, workspace, workspace_bytes);
    if (s) return s;
    const BmLayout L = blockmajor_layout(bm_shape(cfg));
    uint8_t* ws = (uint8_t*)workspace;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(ws + L.misc, 0, 256, st) != cudaSuccess) return PISA_E_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return cuda_status(launch_bsa_tc(Q, pyr, ws + L.phl, idx, (int*)(ws + L.misc) + 1, select_params_of(cfg),
                                     cfg->Hq / cfg->Hkv, sms, st));
}

int64_t pisa_workspace_bytes(const pisa_cfg* cfg) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return 0;
    return (int64_t)blockmajor_layout(bm_shape(cfg)).total;
}

int pisa_workspace_status(const pisa_cfg* cfg, const void* workspace, void* stream) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!workspace) return PISA_E_INVALID;
    const BmLayout L = blockmajor_layout(bm_shape(cfg));
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, (const uint8_t*)workspace + L.misc + 4, 4, cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return PISA_E_CUDA;
    return word == 0 ? PISA_OK : PISA_E_TIMEOUT;
}

int pisa_select_ws(const pisa_cfg* cfg, const void* Q, const void* K, const float* pyr, int32_t* idx,
                   void* workspace, size_t workspace_bytes, void* stream) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !pyr || !idx) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned32(pyr) || !aligned16(idx)) return PISA_E_ALIGNMENT;
    s = check_ws(cfg, workspace, workspace_bytes);
    if (s) return s;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_select_bm(Q, K, pyr, idx, select_params(cfg, g), bm_shape(cfg), workspace, nullptr,
                                        (cudaStream_t)stream));
}

int pisa_sparse_attn_ws(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, const int32_t* idx,
                        void* O, void* workspace, size_t workspace_bytes, void* stream) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !V || !idx || !O) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(O)) return PISA_E_ALIGNMENT;
    s = check_ws(cfg, workspace, workspace_bytes);
    if (s) return s;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_attn_bm(Q, K, V, idx, O, select_params(cfg, g), bm_shape(cfg), workspace, false,
                                      nullptr, (cudaStream_t)stream));
}

static int backward_ws(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, const int32_t* idx,
                       const void* dO, float* dQ, float* dK, float* dV, void* workspace, size_t workspace_bytes,
                       bool saved, const PhaseEvents* ev, void* stream) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !V || !idx || !dO || !dQ || !dK || !dV) return PISA_E_INVALID;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV))
        return PISA_E_ALIGNMENT;
    if (!workspace) return PISA_E_INVALID;
    if (((uintptr_t)workspace & 255u) != 0) return PISA_E_ALIGNMENT;
    if (workspace_bytes < blockmajor_bwd_bytes(bm_shape(cfg))) return PISA_E_INVALID;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_attn_bwd_bm(Q, K, V, idx, dO, dQ, dK, dV, select_params(cfg, g), bm_shape(cfg),
                                          workspace, saved, ev, (cudaStream_t)stream));
}

int64_t pisa_backward_workspace_bytes(const pisa_cfg* cfg) {
    int s = check_bm(cfg);
    if (s) return s;
    if (cfg->N == 0) return 0;
    return (int64_t)blockmajor_bwd_bytes(bm_shape(cfg));
}

int pisa_sparse_attn_backward_ws(const pisa_cfg* cfg, const void* Q, const void* K, const void* V,
                                 const int32_t* idx, const void* dO, float* dQ, float* dK, float* dV, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return backward_ws(cfg, Q, K, V, idx, dO, dQ, dK, dV, workspace, workspace_bytes, false, nullptr, stream);
}

int pisa_sparse_attn_backward_saved_ws(const pisa_cfg* cfg, const void* Q, const void* K, const void* V,
                                       const int32_t* idx, const void* dO, float* dQ, float* dK, float* dV,
                                       void* workspace, size_t workspace_bytes, void* stream) {
    return backward_ws(cfg, Q, K, V, idx, dO, dQ, dK, dV, workspace, workspace_bytes, true, nullptr, stream);
}

int pisa_sparse_attn_backward_ws_events(const pisa_cfg* cfg, const void* Q, const void* K, const void* V,
                                        const int32_t* idx, const void* dO, float* dQ, float* dK, float* dV,
                                        void* workspace, size_t workspace_bytes, void* const* events, int n_events,
                                        void* stream) {
    PhaseEvents ev{events, n_events};
    return backward_ws(cfg, Q, K, V, idx, dO, dQ, dK, dV, workspace, workspace_bytes, false, &ev, stream);
}

int pisa_forward_ws_events(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, float* pyr,
                           int32_t* idx, void* O, void* workspace, size_t workspace_bytes, void* const* events,
                           int n_events, void* stream) {
    int s = check_forward_ws(cfg, Q, K, V, pyr, idx, O, workspace, workspace_bytes);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (n_events < 0 || (n_events > 0 && !events)) return PISA_E_INVALID;
    const PhaseEvents ev{events, n_events};
    cudaStream_t st = (cudaStream_t)stream;
    if (n_events > 0 && events[0]) cudaEventRecord((cudaEvent_t)events[0], st);
    s = pisa_build_pyramid(cfg, K, pyr, stream);
    if (s) return s;
    if (n_events > 1 && events[1]) cudaEventRecord((cudaEvent_t)events[1], st);
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    const SelectParams sp = select_params(cfg, g);
    const BmShape sh = bm_shape(cfg);
    s = cuda_status(launch_select_bm(Q, K, pyr, idx, sp, sh, workspace, &ev, st));
    if (s) return s;
    return cuda_status(launch_attn_bm(Q, K, V, idx, O, sp, sh, workspace, true, &ev, st));
}

int pisa_forward_host(const pisa_cfg* cfg, const void* Q_host, const void* K_host, const void* V_host,
                      int32_t* idx_host, void* O_host, void* Q, void* K, void* V, float* pyr, int32_t* idx,
                      void* O, void* workspace, size_t workspace_bytes, void* stream) {
    // every check of the device step comes first: a failed call enqueues no copy
    int s = check_forward_ws(cfg, Q, K, V, pyr, idx, O, workspace, workspace_bytes);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q_host || !K_host || !V_host || !idx_host || !O_host) return PISA_E_INVALID;
    const size_t es = cfg->dtype == PISA_DTYPE_BF16 ? 2 : 4;
    const size_t q_bytes = (size_t)cfg->B * cfg->Hq * cfg->N * cfg->d * es;
    const size_t kv_bytes = (size_t)cfg->B * cfg->Hkv * cfg->N * cfg->d * es;
    const size_t idx_bytes = (size_t)cfg->B * cfg->Hkv * cfg->N * cfg->K * sizeof(int32_t);
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(Q, Q_host, q_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(K, K_host, kv_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(V, V_host, kv_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return PISA_E_CUDA;
    s = pisa_forward_ws(cfg, Q, K, V, pyr, idx, O, workspace, workspace_bytes, stream);
    if (s) return s;
    if (cudaMemcpyAsync(idx_host, idx, idx_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(O_host, O, q_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return PISA_E_CUDA;
    return PISA_OK;
}

int pisa_forward_ws(const pisa_cfg* cfg, const void* Q, const void* K, const void* V, float* pyr, int32_t* idx,
                    void* O, void* workspace, size_t workspace_bytes, void* stream) {
    return pisa_forward_ws_events(cfg, Q, K, V, pyr, idx, O, workspace, workspace_bytes, nullptr, 0, stream);
}

int pisa_build_pyramid_prefix(const pisa_cfg* cfg, const void* Kc, const int32_t* len, float* pyr, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Kc || !len || !pyr) return PISA_E_INVALID;
    if (!aligned16(Kc) || !aligned16(pyr)) return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_pool(cfg->dtype, cfg->d, Kc, pyr, pool_params(cfg, g, len), (cudaStream_t)stream));
}

int pisa_pyramid_grow(const pisa_cfg* cfg_old, const float* pyr_old, const pisa_cfg* cfg_new, float* pyr_new,
                      void* stream) {
    int s = check_grow(cfg_old, cfg_new);
    if (s) return s;
    if (cfg_old->N == 0) return PISA_OK;
    s = check_grow_pyramids(pyr_old, pyr_new);
    if (s) return s;
    Geom go, gn;
    make_geom(cfg_old->N, cfg_old->C, &go);
    make_geom(cfg_new->N, cfg_new->C, &gn);
    return cuda_status(launch_pyramid_grow(pyr_old, pyr_new, (int64_t)cfg_new->B * cfg_new->Hkv, cfg_new->d, go, gn,
                                           (cudaStream_t)stream));
}

int64_t pisa_cache_capacity(int64_t n, int C) {
    if (C <= 0 || n < 0) return PISA_E_INVALID;
    int64_t cap = C;
    while (cap < n) {
        if (cap > ((int64_t)1 << 40)) return PISA_E_UNSUPPORTED;
        cap *= 2;
    }
    return cap;
}

int pisa_cache_grow(const pisa_cfg* cfg_old, const void* Kc_old, const void* Vc_old, const float* pyr_old,
                    const pisa_cfg* cfg_new, void* Kc_new, void* Vc_new, float* pyr_new, void* stream) {
    // every check, the pyramids' included, comes before the first launch
    int s = check_grow(cfg_old, cfg_new);
    if (s) return s;
    if (cfg_old->N == 0) return PISA_OK;
    if (!Kc_old || !Vc_old || !Kc_new || !Vc_new || Kc_new == Kc_old || Vc_new == Vc_old || Kc_new == Vc_new)
        return PISA_E_INVALID;
    if (!aligned16(Kc_old) || !aligned16(Vc_old) || !aligned16(Kc_new) || !aligned16(Vc_new))
        return PISA_E_ALIGNMENT;
    s = check_grow_pyramids(pyr_old, pyr_new);
    if (s) return s;
    const int64_t units = (int64_t)cfg_new->B * cfg_new->Hkv;
    const int row_bytes = cfg_new->d * (cfg_new->dtype == PISA_DTYPE_BF16 ? 2 : 4);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = launch_cache_grow(Kc_old, Kc_new, units, cfg_old->N, cfg_new->N, row_bytes, st);
    if (e == cudaSuccess) e = launch_cache_grow(Vc_old, Vc_new, units, cfg_old->N, cfg_new->N, row_bytes, st);
    if (e != cudaSuccess) return PISA_E_CUDA;
    return pisa_pyramid_grow(cfg_old, pyr_old, cfg_new, pyr_new, stream);
}

int pisa_pyramid_append(const pisa_cfg* cfg, void* Kc, void* Vc, float* pyr, const void* k_new, const void* v_new,
                        const int32_t* pos, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Kc || !Vc || !pyr || !k_new || !v_new || !pos) return PISA_E_INVALID;
    if (!aligned16(Kc) || !aligned16(Vc) || !aligned16(pyr) || !aligned16(k_new) || !aligned16(v_new))
        return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_append(cfg->dtype, cfg->d, Kc, Vc, pyr, k_new, v_new, pos, decode_params(cfg, g),
                                     (cudaStream_t)stream));
}

int pisa_decode(const pisa_cfg* cfg, const void* q_new, const void* Kc, const void* Vc, const float* pyr,
                const int32_t* pos, int32_t* idx, void* o, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->causal != 1) return PISA_E_INVALID;  // the new token sees only the past
    if (cfg->N == 0) return PISA_OK;
    if (!q_new || !Kc || !Vc || !pyr || !pos || !idx || !o) return PISA_E_INVALID;
    if (!aligned16(q_new) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(pyr) || !aligned16(o))
        return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_decode(cfg->dtype, cfg->d, q_new, const_cast<void*>(Kc), const_cast<void*>(Vc),
                                     const_cast<float*>(pyr), pos, idx, o, nullptr, nullptr, decode_params(cfg, g),
                                     (cudaStream_t)stream));
}

int pisa_decode_step(const pisa_cfg* cfg, const void* q_new, const void* k_new, const void* v_new, void* Kc,
                     void* Vc, float* pyr, const int32_t* pos, int32_t* idx, void* o, void* stream) {
    int s = check_gpu(cfg);
    if (s) return s;
    if (cfg->causal != 1) return PISA_E_INVALID;
    if (cfg->N == 0) return PISA_OK;
    if (!q_new || !k_new || !v_new || !Kc || !Vc || !pyr || !pos || !idx || !o) return PISA_E_INVALID;
    if (!aligned16(q_new) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(Kc) || !aligned16(Vc) ||
        !aligned16(pyr) || !aligned16(o))
        return PISA_E_ALIGNMENT;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    return cuda_status(launch_decode(cfg->dtype, cfg->d, q_new, Kc, Vc, pyr, pos, idx, o, k_new, v_new,
                                     decode_params(cfg, g), (cudaStream_t)stream));
}

const char* pisa_status_string(int status) {
    switch (status) {
        case PISA_OK: return "ok";
        case PISA_E_INVALID: return "invalid argument";
        case PISA_E_UNSUPPORTED: return "configuration outside the GPU kernels' limits";
        case PISA_E_CUDA: return "CUDA launch or runtime error";
        case PISA_E_ALIGNMENT: return "tensor pointer not 16-byte aligned (the pyramid: 32-byte for the block-major calls)";
        case PISA_E_TIMEOUT: return "a tensor-core tile gave up a bounded wait";
        case PISA_E_SCRATCH_LIMIT: return "problem exceeds the fixed scratch of pisa_select_noalloc";
    }
    return "unknown status";
}

const char* pisa_version(void) { return "pisa-b200 0.1.0 sm_100a"; }

}  // extern "C"
