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
//     caches it; make that first call before any stream capture.
#include <cstdint>
#include <mutex>

#include <cuda_bf16.h>

#include "sata_internal.h"

namespace sata {
namespace {

constexpr size_t kStaticScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_decode_scratch[kStaticScratchFloats];

constexpr int kThreads = 256;
constexpr int kFG = 1024;          // features per CTA
constexpr int kPerThread = kFG / kThreads;
constexpr int kMaxDevices = 64;

std::mutex g_scratch_mu;
float *g_scratch_dev[kMaxDevices] = {};

// Padded index triple (a, b, l) of feature f in basis order (index d stands
// for the constant 1) and its query-side coefficient alpha_p * C_p.
__device__ void unrank_feature(int64_t f, int d, int &a, int &b, int &l, int &p) {
    if (f == 0) { a = b = l = d; p = 0; return; }
    f -= 1;
    if (f < d) { a = b = d; l = (int)f; p = 1; return; }
    f -= d;
    const int64_t m2 = (int64_t)d * (d + 1) / 2;
    if (f < m2) {
        int i = 0;
        while (f >= d - i) { f -= d - i; ++i; }
        a = d; b = i; l = i + (int)f; p = 2;
        return;
    }
    f -= m2;
    int i = 0;
    while (true) {
        const int64_t n = (int64_t)(d - i) * (d - i + 1) / 2;
        if (f < n) break;
        f -= n;
        ++i;
    }
    int j = i;
    while (f >= d - j) { f -= d - j; ++j; }
    a = i; b = j; l = j + (int)f; p = 3;
}

// The feature after (a, b, l) of degree p, in basis order.
__device__ void next_feature(int d, int &a, int &b, int &l, int &p) {
    if (p == 0) { a = b = d; l = 0; p = 1; return; }
    if (p == 1) {
        if (l + 1 < d) { ++l; return; }
        a = d; b = 0; l = 0; p = 2;
        return;
    }
    if (p == 2) {
        if (l + 1 < d) { ++l; return; }
        if (b + 1 < d) { ++b; l = b; return; }
        a = b = l = 0; p = 3;
        return;
    }
    if (l + 1 < d) { ++l; return; }
    if (b + 1 < d) { ++b; l = b; return; }
    ++a; b = l = a;
}

// alpha_p * C_p = C_p / (p! c^p) for the triple, C_p = p! / prod(mult!).
__device__ float feature_coef(int a, int b, int l, int p, float inv_c) {
    if (p == 0) return 1.f;
    if (p == 1) return inv_c;
    if (p == 2) return (b == l ? 0.5f : 1.f) * inv_c * inv_c;
    const float inv_mult = (a == b && b == l) ? (1.f / 6.f) : ((a == b || b == l) ? 0.5f : 1.f);
    return inv_mult * inv_c * inv_c * inv_c;
}

__device__ __forceinline__ float4 fma4(float s, float4 x, float4 y) {
    return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}

// Same streaming scheme as the ordinary decode kernel (update then read each
// S row once, 16-byte accesses), with the basis derived in registers.
template <int DV>
__global__ void __launch_bounds__(kThreads)
decode_static_stream_kernel(float *__restrict__ S, float *__restrict__ Z,
                            const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                            const __nv_bfloat16 *__restrict__ v, int d_K, int64_t F, float inv_c,
                            float *__restrict__ partials) {
    constexpr int TPR = DV / 4;
    constexpr int RPI = kThreads / TPR;
    constexpr int kWarps = kThreads / 32;
    __shared__ float xq[kMaxDK + 1], xk[kMaxDK + 1], xv[DV];
    __shared__ float phik[kFG], aq[kFG];
    __shared__ float red[kWarps][DV + 1];
    const int g = blockIdx.y, G = gridDim.y;
    const int64_t bh = blockIdx.x;
    const int64_t f0 = (int64_t)g * kFG;
    const int nf = (int)(F - f0 < (int64_t)kFG ? F - f0 : (int64_t)kFG);
    const int tid = threadIdx.x;
    for (int i = tid; i <= d_K; i += kThreads) {
        xq[i] = i < d_K ? __bfloat162float(q[bh * d_K + i]) : 1.0f;
        xk[i] = i < d_K ? __bfloat162float(k[bh * d_K + i]) : 1.0f;
    }
    for (int i = tid; i < DV; i += kThreads) xv[i] = __bfloat162float(v[bh * DV + i]);
    __syncthreads();
    {   // this thread's kPerThread consecutive features
        const int fl = tid * kPerThread;
        if (fl < nf) {
            int a, b, l, p;
            unrank_feature(f0 + fl, d_K, a, b, l, p);
            for (int u = 0; u < kPerThread && fl + u < nf; ++u) {
                if (u > 0) next_feature(d_K, a, b, l, p);
                phik[fl + u] = xk[a] * xk[b] * xk[l];
                aq[fl + u] = feature_coef(a, b, l, p, inv_c) * (xq[a] * xq[b] * xq[l]);
            }
        }
    }
    __syncthreads();
    const int col = tid % TPR;
    const int r0 = tid / TPR;
    const float4 vv = make_float4(xv[4 * col], xv[4 * col + 1], xv[4 * col + 2], xv[4 * col + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 *Sb = reinterpret_cast<float4 *>(S + (bh * F + f0) * DV);
    int r = r0;
    for (; r + 3 * RPI < nf; r += 4 * RPI) {
        float4 s[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) s[u] = Sb[(int64_t)(r + u * RPI) * TPR + col];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int rr = r + u * RPI;
            s[u] = fma4(phik[rr], vv, s[u]);
            Sb[(int64_t)rr * TPR + col] = s[u];
            acc = fma4(aq[rr], s[u], acc);
        }
    }
    for (; r < nf; r += RPI) {
        float4 s = Sb[(int64_t)r * TPR + col];
        s = fma4(phik[r], vv, s);
        Sb[(int64_t)r * TPR + col] = s;
        acc = fma4(aq[r], s, acc);
    }
    float dacc = 0.f;
    float *Zb = Z + bh * F + f0;
    for (int f = tid; f < nf; f += kThreads) {
        const float z = Zb[f] + phik[f];
        Zb[f] = z;
        dacc = fmaf(aq[f], z, dacc);
    }
#pragma unroll
    for (int off = TPR; off < 32; off <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dacc += __shfl_xor_sync(0xffffffffu, dacc, off);
    const int warp = tid / 32, lane = tid % 32;
    if (lane < TPR) {
        red[warp][4 * lane + 0] = acc.x;
        red[warp][4 * lane + 1] = acc.y;
        red[warp][4 * lane + 2] = acc.z;
        red[warp][4 * lane + 3] = acc.w;
    }
    if (lane == 0) red[warp][DV] = dacc;
    __syncthreads();
    for (int j = tid; j <= DV; j += kThreads) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][j];
        partials[(bh * G + g) * (DV + 1) + j] = s;
    }
}

template <int DV>
__global__ void decode_static_finish_kernel(const float *__restrict__ partials, int G,
                                            float *__restrict__ out) {
    __shared__ float den;
    const int64_t bh = blockIdx.x;
    const int j = threadIdx.x;
    float s = 0.f;
    if (j <= DV)
        for (int g = 0; g < G; ++g) s += partials[(bh * G + g) * (DV + 1) + j];
    if (j == DV) den = s;
    __syncthreads();
    if (j < DV) out[bh * DV + j] = s / den;
}

template <int DV>
cudaError_t launch_static(int BH, int d_K, int64_t F, float *S, float *Z, const void *q, const void *k,
                          const void *v, float *out, float *scratch, cudaStream_t stream) {
    const int G = (int)((F + kFG - 1) / kFG);
    const float inv_c = 1.0f / sqrtf((float)d_K);
    decode_static_stream_kernel<DV><<<dim3(BH, G), kThreads, 0, stream>>>(
        S, Z, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, d_K, F, inv_c,
        scratch);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_static_finish_kernel<DV><<<BH, ((DV + 1 + 31) / 32) * 32, 0, stream>>>(scratch, G, out);
    return cudaGetLastError();
}

// Device address of the scratch array on the current device, looked up once.
cudaError_t static_scratch(float **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_dev[dev]) {
        float *p = nullptr;
        e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = p;
    }
    *ptr = g_scratch_dev[dev];
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
    const int64_t G = (F + kFG - 1) / kFG;
    if ((uint64_t)BH * (uint64_t)G * (uint64_t)(d_V + 1) > kStaticScratchFloats) return SATA_ENOMEM;
    float *scratch = nullptr;
    cudaError_t e = static_scratch(&scratch);
    if (e == cudaSuccess) {
        cudaStream_t s = (cudaStream_t)st->stream;
        switch (d_V) {
            case 4: e = launch_static<4>(BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch, s); break;
            case 8: e = launch_static<8>(BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch, s); break;
            case 16: e = launch_static<16>(BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch, s); break;
            case 32: e = launch_static<32>(BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch, s); break;
            case 64: e = launch_static<64>(BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch, s); break;
            default: e = launch_static<128>(BH, st->d_K, F, st->S, st->Z, q, k, v, out, scratch, s); break;
        }
    }
    if (e != cudaSuccess) return record_cuda_error(e);
    st->tokens += 1;
    return SATA_OK;
}
