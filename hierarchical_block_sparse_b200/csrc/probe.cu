// probe.cu -- a CUDA-core fp32 FMA throughput probe, so that the "alu"
// roofline of the walk kernels is taken against a measured peak rather than
// one derived from unit counts and the maximum clock.
//
// Every thread runs 8 independent FMA chains (enough to cover the FMA
// latency with full occupancy) of either scalar fp32 FMAs or packed fp32x2
// FMAs (two lanes per instruction); the chains are summed into `out` so that
// nothing is eliminated. FLOP per launch = threads * iters * 8 * 2 (x2 packed).
#include <cuda_runtime.h>
#include <stdint.h>

#include "pisa.h"

namespace {

template <bool PACKED>
__global__ void __launch_bounds__(256) fma_probe_kernel(float* __restrict__ out, int iters) {
    const float s = 1e-3f * (float)(threadIdx.x & 31);
    if constexpr (PACKED) {
        float2 a[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = make_float2(s + j, s - j);
        const float2 m = make_float2(0.9999f, 1.0001f), c = make_float2(1e-4f, -1e-4f);
        for (int i = 0; i < iters; ++i) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = __ffma2_rn(a[j], m, c);
        }
        float r = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) r += a[j].x + a[j].y;
        out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = r;
    } else {
        float a[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = s + j;
        const float m = 0.9999f, c = 1e-4f;
        for (int i = 0; i < iters; ++i) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = fmaf(a[j], m, c);
        }
        float r = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) r += a[j];
        out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = r;
    }
}

}  // namespace

extern "C" int pisa_fma_probe(float* out, int blocks, int iters, int packed, void* stream) {
    if (!out || blocks < 1 || iters < 1) return PISA_E_INVALID;
    if (packed) fma_probe_kernel<true><<<blocks, 256, 0, (cudaStream_t)stream>>>(out, iters);
    else fma_probe_kernel<false><<<blocks, 256, 0, (cudaStream_t)stream>>>(out, iters);
    return cudaGetLastError() == cudaSuccess ? PISA_OK : PISA_E_CUDA;
}
