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
// device address is looked up with cudaGetSymbolAddress once per device, with
// that device current, on the first call made on it; make that first call
// before any stream capture. All calls on a device share the array and it
// keeps the previous call's contents: the selection clears what must start at
// zero (its counters and error word) on every call, and two calls that
// overlap on the GPU race on the array.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "pisa.h"
#include "pisa_internal.h"

namespace pisa {
namespace {

constexpr size_t kScratchBytes = PISA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::once_flag g_once[kMaxDevices];
void* g_addr[kMaxDevices];
cudaError_t g_err[kMaxDevices];

// device address of g_scratch on the current device (looked up once per device)
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_once[dev], [dev] {
        void* p = nullptr;
        g_err[dev] = cudaGetSymbolAddress(&p, g_scratch);
        g_addr[dev] = g_err[dev] == cudaSuccess ? p : nullptr;
    });
    *out = g_addr[dev];
    return g_err[dev];
}

}  // namespace
}  // namespace pisa

using namespace pisa;

extern "C" int pisa_select_noalloc(const pisa_cfg* cfg, const void* Q, const void* K, const float* pyr, int32_t* idx,
                                   void* stream) {
    // the limits of the workspace path apply (bf16, d = 128, C = 64, ...)
    const int64_t need = pisa_workspace_bytes(cfg);
    if (need < 0) return (int)need;
    if (cfg->N == 0) return PISA_OK;
    if (!Q || !K || !pyr || !idx) return PISA_E_INVALID;
    if ((((uintptr_t)Q | (uintptr_t)K | (uintptr_t)idx) & 15u) != 0 || ((uintptr_t)pyr & 31u) != 0)
        return PISA_E_ALIGNMENT;
    BmShape s;
    s.B = cfg->B; s.Hq = cfg->Hq; s.Hkv = cfg->Hkv; s.N = cfg->N; s.G = cfg->Hq / cfg->Hkv;
    s.M1 = ((int64_t)cfg->N + cfg->C - 1) / cfg->C;
    Geom g;
    make_geom(cfg->N, cfg->C, &g);
    s.rows = g.rows;
    s.variant = cfg->score_variant;
    const BmLayout L = blockmajor_layout(s);
    // the selection uses every region except the attention accumulator, which is last
    if (L.oacc > kScratchBytes) return PISA_E_SCRATCH_LIMIT;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess || !ws) return PISA_E_CUDA;
    SelectParams sp;
    sp.B = cfg->B; sp.Hq = cfg->Hq; sp.Hkv = cfg->Hkv; sp.N = cfg->N; sp.C = cfg->C; sp.K = cfg->K;
    sp.causal = cfg->causal; sp.forced_mask = cfg->forced_mask;
    sp.qscale = (float)(1.4426950408889634 / sqrt((double)cfg->d));
    sp.geom = g;
    sp.variant = cfg->score_variant;
    const cudaError_t e = launch_select_bm(Q, K, pyr, idx, sp, s, ws, nullptr, (cudaStream_t)stream);
    return e == cudaSuccess ? PISA_OK : PISA_E_CUDA;
}
