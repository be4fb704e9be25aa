// sata_decode_step_static: the decode step with no device allocation at all.
//
// Who needs it: code whose device memory is owned by someone else, such as a
// serving runtime that hands out a fixed pre-allocated arena, a plugin running
// inside a host application with its own allocator, or a process held to a
// strict memory budget.  Such callers must not call cudaMalloc, which allocates
// outside their accounting and may also synchronise the device.  The ordinary
// sata_decode_step allocates on first use: its partial-sum workspace and its
// per-(d_K, P) basis tables.  This variant allocates nothing.  Its partial sums
// live in the file-scope static device array below, and it derives each
// feature's index triple and coefficient arithmetically instead of reading a
// table.
//
// Limits and sharing:
//   - The scratch holds kStaticScratchFloats (1 Mi) fp32 values, 4 MiB, present
//     on every GPU that loads the library until the process exits.  A call
//     needing more (B*H * ceil(F/1024) * (d_V+1) values) is rejected with
//     SATA_ENOMEM before anything is launched.
//   - All calls share the one array and it keeps the last call's contents.  The
//     stream kernel writes every partial slot it owns before the finish kernel
//     reads it, so nothing has to start at zero.  Two calls that overlap on the
//     GPU (different streams, no ordering between them) race on the array.
//   - The first call on each device looks up the array's device address with
//     cudaGetSymbolAddress (a host-side symbol name is not a device pointer) and
//     caches it with the device's current context; a call in another context
//     (the one a cudaDeviceReset leaves) looks it up again.  Make the first call
//     in a context before any stream capture.
//   - The kernels are the ordinary decode step's (decode_kernels.cuh) with the
//     basis derived in registers, so the two entry points compute alike.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>

#include "decode_kernels.cuh"

namespace sata {
namespace {

constexpr size_t kStaticScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_decode_scratch[kStaticScratchFloats];

constexpr int kMaxDevices = 64;

// The array's device address per device, with the context it was looked up in:
// a new context on the device (after cudaDeviceReset, say) looks it up again.
struct ScratchAddr {
    CUcontext ctx;
    float *ptr;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch[kMaxDevices] = {};

cudaError_t static_scratch(float **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    e = cudaFree(nullptr);                 // makes the device's primary context current
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    // the driver's cuCtxGetCurrent through the runtime, so the library needs no
    // link-time dependency on the driver library
    static CUresult (*get_ctx)(CUcontext *) = nullptr;
    if (!get_ctx) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorSymbolNotFound;
        get_ctx = reinterpret_cast<CUresult (*)(CUcontext *)>(fn);
    }
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    if (!g_scratch[dev].ptr || g_scratch[dev].ctx != ctx) {
        float *p = nullptr;
        e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch[dev] = {ctx, p};
    }
    *ptr = g_scratch[dev].ptr;
    return cudaSuccess;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace sata

using namespace sata;

extern "C" int sata_decode_step_static(sata_state *st, const void *q, const void *k, const void *v,
                                       float *out) {
    if (!st) return SATA_EINVAL;
    if (st->B < 0 || st->H < 0 || st->d_K < 1 || st->d_V < 1 || st->P < 1) return SATA_EINVAL;
    const int64_t bh64 = (int64_t)st->B * st->H;
    const int d_V = st->d_V;
    if (bh64 > INT32_MAX || st->d_K > kMaxDK || st->P > kMaxPStatic ||
        !(d_V == 4 || d_V == 8 || d_V == 16 || d_V == 32 || d_V == 64 || d_V == 128))
        return SATA_EUNSUPPORTED;
    const int64_t F = num_features(st->d_K, st->P);
    if (st->F != F) return SATA_EINVAL;
    const int BH = (int)bh64;
    if (BH == 0) return SATA_OK;
    if (!q || !k || !v || !out || !st->S || !st->Z) return SATA_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(st->S) ||
        !aligned16(st->Z))
        return SATA_EALIGN;
    const int64_t G = dec::num_groups(F);
    if ((uint64_t)BH * (uint64_t)G * (uint64_t)(d_V + 1) > kStaticScratchFloats) return SATA_ENOMEM;
    float *scratch = nullptr;
    cudaError_t e = static_scratch(&scratch);
    if (e == cudaSuccess) {
        const double c = sqrt((double)st->d_K);
        const dec::DerivedBasis db{st->d_K, {1.f, (float)(1.0 / c), (float)(1.0 / (c * c)), (float)(1.0 / (c * c * c))}};
        e = dec::launch_any(d_V, db, BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch,
                            (cudaStream_t)st->stream, false);
    }
    if (e != cudaSuccess) return record_cuda_error(e);
    st->tokens += 1;
    return SATA_OK;
}
