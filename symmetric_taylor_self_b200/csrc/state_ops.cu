// Operations on recurrent states.
//
// [CC-TAYLOR] "Feature maps and linear attention": S and Z are sums over the
// tokens seen, so they may be computed by a parallel prefix scan: the state of
// a concatenation of token segments is the sum of the segments' states.  This
// is the exchange step of a prefill split by sequence across GPUs (each rank
// computes its segment's state, then adds the states of the segments before
// it).
#include "sata_internal.h"

namespace sata {
namespace {

// dst[i] += src[i] for n floats; dst and src 16-byte aligned.
__global__ void __launch_bounds__(256) state_add_kernel(float *__restrict__ dst, const float *__restrict__ src,
                                                        int64_t n) {
    const int64_t n4 = n / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    float4 *d4 = reinterpret_cast<float4 *>(dst);
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 a = d4[i];
        const float4 b = s4[i];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
        d4[i] = a;
    }
    for (int64_t i = 4 * n4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride) dst[i] += src[i];
}

cudaError_t add(float *dst, const float *src, int64_t n, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = (n / 4 + 255) / 256;
    const int grid = (int)(blocks < 148 * 16 ? (blocks > 0 ? blocks : 1) : 148 * 16);
    launch_begin(kStateAdd, stream);
    state_add_kernel<<<grid, 256, 0, stream>>>(dst, src, n);
    launch_end(kStateAdd, stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_add(float *S, float *Z, const float *dS, const float *dZ, int64_t nS, int64_t nZ,
                             cudaStream_t stream) {
    cudaError_t e = add(S, dS, nS, stream);
    if (e == cudaSuccess) e = add(Z, dZ, nZ, stream);
    return e;
}

}  // namespace sata
