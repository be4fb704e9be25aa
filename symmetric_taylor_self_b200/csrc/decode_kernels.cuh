// Decode-step kernels: one token per head against the fixed-size state.
// Shared by sata_decode_step (decode.cu: basis read from the cached tables) and
// sata_decode_step_static (decode_static.cu: basis derived in registers, no
// tables, partial sums in a static array).  The two differ only in the Basis
// policy that fills phi(k) and alpha*C*phi(q) for a CTA's features.
//
// [CC-TAYLOR] "Self-attention at constant cost per token via symmetry-aware
// Taylor approximation", section "Feature maps and linear attention"
// (特征映射与线性注意力): Z_T = Z_{T-1} + phi(k_T), S_T = S_{T-1} + phi(k_T) v_T^T,
// y_T = sum_p alpha_p phi_p(q_T)^T C_p S_p / sum_p alpha_p <phi_p(q_T), Z_p>_C.
// [CC-HW] "Constant-cost attention: hardware optimization", section "Fixed-size
// hidden state": the per-token cost is set by the state size, not the context.
//
// The step is bound by HBM: every state value is read once and written once
// (8 bytes per value).  Work split: CTA (g, bh) owns features
// [g*kFG, (g+1)*kFG) of head bh; it computes phi(k) and alpha*C*phi(q) for them
// in shared memory, then streams the S rows with 16-byte loads/stores (d_V/4
// threads per row), updating and reading in one pass.  Per-CTA partial
// numerators/denominators go to a small buffer and the finish kernel sums them
// in a fixed order and divides (deterministic).
//
// Everything here has internal linkage (each including file gets its own
// kernels), so the two entry points never share a kernel registration.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

#include "sata_internal.h"

namespace sata {
namespace {
namespace dec {

constexpr int kThreads = 256;
constexpr int kFG = 1024;          // features per CTA

__device__ __forceinline__ float4 fma4(float s, float4 x, float4 y) {
    return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}

// Basis from the cached tables: packed index triple (and, for degrees above 3,
// the leading indices) and the query-side coefficient of every feature.
struct TableBasis {
    const uint32_t *packed, *packed_hi;
    const float *coef;

    __device__ void fill(int64_t f0, int nf, const float *xq, const float *xk, float *phik,
                         float *aq) const {
        for (int f = threadIdx.x; f < nf; f += kThreads) {
            const uint32_t pk = packed[f0 + f];
            const int a = pk & 255, b = (pk >> 8) & 255, l = (pk >> 16) & 255;
            float fk = xk[a] * xk[b] * xk[l], fq = xq[a] * xq[b] * xq[l];
            if (packed_hi) {
                const uint32_t ph = packed_hi[f0 + f];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int i = (ph >> (8 * m)) & 255;
                    fk *= xk[i];
                    fq *= xq[i];
                }
            }
            phik[f] = fk;
            aq[f] = coef[f0 + f] * fq;
        }
    }
};

// Basis derived arithmetically (P <= 4): each thread unranks its first feature
// and steps through kFG / kThreads consecutive ones.  Index d stands for the
// constant 1 (the padding that makes every feature a triple).  ic[p] = c^-p,
// each rounded once from double on the host; a coefficient is 1/prod(mult!) times
// ic[p], so it can differ from the table path's (one rounding of the product) in
// its last bit.
struct DerivedBasis {
    int d;
    float ic[4];

    // Padded triple (a, b, l) of feature f in basis order, and its degree p.
    __device__ static void unrank(int64_t f, int d, int &a, int &b, int &l, int &p) {
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
    __device__ static void next(int d, int &a, int &b, int &l, int &p) {
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
    __device__ static float coef(int a, int b, int l, int p, const float (&ic)[4]) {
        if (p == 0) return 1.f;
        if (p == 1) return ic[1];
        if (p == 2) return (b == l ? 0.5f : 1.f) * ic[2];
        const float inv_mult = (a == b && b == l) ? (1.f / 6.f) : ((a == b || b == l) ? 0.5f : 1.f);
        return inv_mult * ic[3];
    }

    __device__ void fill(int64_t f0, int nf, const float *xq, const float *xk, float *phik,
                         float *aq) const {
        constexpr int kPerThread = kFG / kThreads;
        const int fl = threadIdx.x * kPerThread;
        if (fl >= nf) return;
        int a, b, l, p;
        unrank(f0 + fl, d, a, b, l, p);
        for (int u = 0; u < kPerThread && fl + u < nf; ++u) {
            if (u > 0) next(d, a, b, l, p);
            phik[fl + u] = xk[a] * xk[b] * xk[l];
            aq[fl + u] = coef(a, b, l, p, ic) * (xq[a] * xq[b] * xq[l]);
        }
    }
};

template <int DV, class Basis>
__global__ void __launch_bounds__(kThreads)
stream_kernel(float *__restrict__ S, float *__restrict__ Z, const __nv_bfloat16 *__restrict__ q,
              const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v, Basis basis,
              int d_K, int64_t F, float *__restrict__ partials) {
    constexpr int TPR = DV / 4;              // threads per state row, one float4 each
    constexpr int RPI = kThreads / TPR;      // rows per block iteration
    constexpr int kWarps = kThreads / 32;
    __shared__ float xq[kMaxDK + 1], xk[kMaxDK + 1], xv[DV];
    __shared__ float phik[kFG], aq[kFG];
    __shared__ float red[kWarps][DV + 1];

    const int g = blockIdx.y, G = gridDim.y;
    const int64_t bh = blockIdx.x;
    const int64_t f0 = (int64_t)g * kFG;
    const int nf = (int)(F - f0 < (int64_t)kFG ? F - f0 : (int64_t)kFG);
    const int tid = threadIdx.x;

    // x[d_K] = 1 is the padding index of the basis.
    for (int i = tid; i <= d_K; i += kThreads) {
        xq[i] = i < d_K ? __bfloat162float(q[bh * d_K + i]) : 1.0f;
        xk[i] = i < d_K ? __bfloat162float(k[bh * d_K + i]) : 1.0f;
    }
    for (int i = tid; i < DV; i += kThreads) xv[i] = __bfloat162float(v[bh * DV + i]);
    __syncthreads();
    basis.fill(f0, nf, xq, xk, phik, aq);
    __syncthreads();

    // S rows: update then read (inclusive causal range).
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
    // Z entries: the "+1" column of the state.
    float dacc = 0.f;
    float *Zb = Z + bh * F + f0;
    for (int f = tid; f < nf; f += kThreads) {
        const float z = Zb[f] + phik[f];
        Zb[f] = z;
        dacc = fmaf(aq[f], z, dacc);
    }

    // Reduce: lanes with equal `col` are TPR apart inside a warp.
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
__global__ void finish_kernel(const float *__restrict__ partials, int G, float *__restrict__ out) {
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

inline int num_groups(int64_t F) { return (int)((F + kFG - 1) / kFG); }

// Both kernels of one step on `stream`; `timed` brackets them for the
// per-kernel statistics (the ordinary entry point only).
template <int DV, class Basis>
cudaError_t launch(Basis basis, int BH, int d_K, int64_t F, float *S, float *Z, const void *q, const void *k,
                   const void *v, float *out, float *partials, cudaStream_t stream, bool timed) {
    const int G = num_groups(F);
    if (timed) launch_begin(kDecodeStream, stream);
    stream_kernel<DV, Basis><<<dim3(BH, G), kThreads, 0, stream>>>(
        S, Z, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, basis, d_K, F,
        partials);
    if (timed) launch_end(kDecodeStream, stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (timed) launch_begin(kDecodeFinish, stream);
    finish_kernel<DV><<<BH, ((DV + 1 + 31) / 32) * 32, 0, stream>>>(partials, G, out);
    if (timed) launch_end(kDecodeFinish, stream);
    return cudaGetLastError();
}

template <class Basis>
cudaError_t launch_any(int d_V, Basis basis, int BH, int d_K, int64_t F, float *S, float *Z, const void *q,
                       const void *k, const void *v, float *out, float *partials, cudaStream_t stream,
                       bool timed) {
    switch (d_V) {
        case 4: return launch<4>(basis, BH, d_K, F, S, Z, q, k, v, out, partials, stream, timed);
        case 8: return launch<8>(basis, BH, d_K, F, S, Z, q, k, v, out, partials, stream, timed);
        case 16: return launch<16>(basis, BH, d_K, F, S, Z, q, k, v, out, partials, stream, timed);
        case 32: return launch<32>(basis, BH, d_K, F, S, Z, q, k, v, out, partials, stream, timed);
        case 64: return launch<64>(basis, BH, d_K, F, S, Z, q, k, v, out, partials, stream, timed);
        case 128: return launch<128>(basis, BH, d_K, F, S, Z, q, k, v, out, partials, stream, timed);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dec
}  // namespace
}  // namespace sata
