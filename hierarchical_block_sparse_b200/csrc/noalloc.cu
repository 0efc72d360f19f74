// noalloc.cu -- pisa_select_noalloc: the block-major tensor-core selection
// for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc or any allocating
// routine: code embedded in a host application that owns the GPU memory pool
// and hands plugins no allocator, serving loops that forbid device
// allocations once they have started (fixed memory budgets), or plain C
// callers with no allocator at hand. pisa_select_ws needs a caller-provided
// workspace; this entry point instead uses one fixed scratch array compiled
// into the library, so the caller passes only inputs and outputs.
//
// The scratch is a file-scope __device__ array of kScratchBytes. Every GPU that
// loads the library holds it until the process exits. Host code cannot use the
// array's name as a device address (it names a host-side stand-in), so the
// device address is looked up with cudaGetSymbolAddress, with the device
// current, on the first call made in a CUDA context (the runtime's primary
// context of a device, or a context the caller made current through the
// driver API); make that first call before any stream capture. A lookup that
// fails is not remembered: the next call tries again. All calls in a context
// share the array and it keeps the previous call's contents: the selection
// clears what must start at zero (its counters and error word) on every call,
// and two calls that overlap on the GPU race on the array.
#include <cuda.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "pisa.h"
#include "pisa_internal.h"

namespace pisa {
namespace {

constexpr size_t kScratchBytes = PISA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxContexts = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// successful lookups, keyed by the CUDA context they were made in
std::mutex g_mu;
CUcontext g_ctx[kMaxContexts];
void* g_addr[kMaxContexts];
int g_n = 0;

using CtxGetCurrent = CUresult (*)(CUcontext*);

// the calling thread's current CUDA context (nullptr if it cannot be read)
CUcontext current_context() {
    static CtxGetCurrent fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (CtxGetCurrent) nullptr;
        return (CtxGetCurrent)f;
    }();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// device address of g_scratch in the current context
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);  // also makes the device's primary context current if none is
    if (e != cudaSuccess) return e;
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_mu);
    if (ctx) {
        for (int i = 0; i < g_n; ++i)
            if (g_ctx[i] == ctx) {
                *out = g_addr[i];
                return cudaSuccess;
            }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    if (ctx && g_n < kMaxContexts) {
        g_ctx[g_n] = ctx;
        g_addr[g_n] = p;
        ++g_n;
    }
    *out = p;
    return cudaSuccess;
}

// the selection's regions in the scratch, or an error status
int noalloc_layout(const pisa_cfg* cfg, BmLayout* L) {
    // the limits of the workspace path apply (bf16, d = 128, C = 64, ...)
    const int64_t need = pisa_workspace_bytes(cfg);
    if (need < 0) return (int)need;
    *L = blockmajor_layout(bm_shape_of(cfg));
    // the selection uses every region except the attention accumulator, which is last
    if (L->oacc > kScratchBytes) return PISA_E_SCRATCH_LIMIT;
    return PISA_OK;
}

}  // namespace
}  // namespace pisa

using namespace pisa;

extern "C" int pisa_select_noalloc(const pisa_cfg* cfg, const void* Q, const void* K, const float* pyr, int32_t* idx,
                                   void* stream) {
    BmLayout L;
    const int s = noalloc_layout(cfg, &L);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !pyr || !idx) return PISA_E_INVALID;
    if ((((uintptr_t)Q | (uintptr_t)K | (uintptr_t)idx) & 15u) != 0 || ((uintptr_t)pyr & 31u) != 0)
        return PISA_E_ALIGNMENT;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return PISA_E_CUDA;
    const cudaError_t e = launch_select_bm(Q, K, pyr, idx, select_params_of(cfg), bm_shape_of(cfg), ws, nullptr,
                                           (cudaStream_t)stream);
    return e == cudaSuccess ? PISA_OK : PISA_E_CUDA;
}

extern "C" int pisa_select_noalloc_status(const pisa_cfg* cfg, void* stream) {
    BmLayout L;
    const int s = noalloc_layout(cfg, &L);
    if (s) return s;
    if (cfg->N == 0) return PISA_OK;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return PISA_E_CUDA;
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, (const uint8_t*)ws + L.misc + 4, 4, cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return PISA_E_CUDA;
    return word == 0 ? PISA_OK : PISA_E_TIMEOUT;
}
