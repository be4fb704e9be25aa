// Building blocks of the chunked scans that run outside the tensor-core
// prefill (the CUDA-core prefill and the backward): 256 threads, tiles of
// kTF = 128 features, chunks of kL = 32 tokens.  The chunk loader, the
// truncated series, the fixed-order strided sum, and the CUDA-core prefill's
// register-tiled contractions: thread (warp, lane) owns tokens t = warp + 8b
// (b < 4) and features m = lane + 32a (a < 4) or value columns, and reuses every
// shared-memory operand across that tile.  Shared-memory rows of d_V + 1 floats
// have an odd stride for every supported d_V, so the 32 lanes of a warp reading
// 32 different rows hit 32 banks.
#pragma once

#include <cuda_bf16.h>

#include "sata_internal.h"

namespace sata {
namespace simt {

constexpr int kThreads = 256;
constexpr int kTF = 128;   // features per CTA
constexpr int kL = 32;     // chunk length

// T_n(x) = sum_{p<n} x^p / p! (n <= 8) in Horner form, h <- 1 + h x / p; the
// steps are unrolled so each 1/p is a compile-time constant (no division).
__device__ __forceinline__ float taylor_exp(float x, int n) {
    float h = n > 0 ? 1.f : 0.f;
#pragma unroll
    for (int p = 7; p >= 1; --p)
        if (p < n) h = fmaf(h, x * (1.f / p), 1.f);
    return h;
}

// Loads one chunk of kL token rows starting at row0 into shared memory:
// x~q, x~k [kL][d_K + 1] (last column 1) and [v | 1] [kL][d_V + 1]; rows past nt
// are zero.  16-byte loads (8 bf16) when the rows are bf16 and d_K and d_V are
// multiples of 8, else element loads; either way all of a thread's loads are
// issued before its stores, so they are in flight together.
__device__ __forceinline__ float in_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float in_f(float x) { return x; }

template <typename TI>   // bf16 or fp32 token rows
__device__ __forceinline__ void load_qkv_chunk(const TI *q, const TI *k, const TI *v, int64_t row0, int nt, int d_K,
                                               int d_V, float *xq, float *xk, float *xv) {
    const int DK1 = d_K + 1, DV1 = d_V + 1;
    if (sizeof(TI) == 2 && (d_K & 7) == 0 && (d_V & 7) == 0) {
        constexpr int U = (kL * (kMaxDK / 8) + kThreads - 1) / kThreads;
        const int nq = kL * (d_K / 8), nv = kL * (d_V / 8);
        uint4 bq[U], bk[U], bv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = threadIdx.x + u * kThreads;
            bq[u] = bk[u] = bv[u] = make_uint4(0, 0, 0, 0);
            if (e < nq && e / (d_K / 8) < nt) {
                const int64_t off = (row0 + e / (d_K / 8)) * d_K + (e % (d_K / 8)) * 8;
                bq[u] = *reinterpret_cast<const uint4 *>(q + off);
                bk[u] = *reinterpret_cast<const uint4 *>(k + off);
            }
            if (e < nv && e / (d_V / 8) < nt)
                bv[u] = *reinterpret_cast<const uint4 *>(v + (row0 + e / (d_V / 8)) * d_V + (e % (d_V / 8)) * 8);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = threadIdx.x + u * kThreads;
            if (e < nq) {
                const int t = e / (d_K / 8), i = (e % (d_K / 8)) * 8;
                const __nv_bfloat16 *hq = reinterpret_cast<const __nv_bfloat16 *>(&bq[u]);
                const __nv_bfloat16 *hk = reinterpret_cast<const __nv_bfloat16 *>(&bk[u]);
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    xq[t * DK1 + i + w] = __bfloat162float(hq[w]);
                    xk[t * DK1 + i + w] = __bfloat162float(hk[w]);
                }
            }
            if (e < nv) {
                const int t = e / (d_V / 8), j = (e % (d_V / 8)) * 8;
                const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&bv[u]);
#pragma unroll
                for (int w = 0; w < 8; ++w) xv[t * DV1 + j + w] = __bfloat162float(hv[w]);
            }
        }
        for (int t = threadIdx.x; t < kL; t += kThreads) {   // the constant columns
            const float one = t < nt ? 1.f : 0.f;
            xq[t * DK1 + d_K] = one;
            xk[t * DK1 + d_K] = one;
            xv[t * DV1 + d_V] = one;
        }
        return;
    }
    constexpr int U = (kL * (kMaxDK + 1) + kThreads - 1) / kThreads;
    static_assert(kMaxDV <= kMaxDK, "one bound for both loops");
    float a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = threadIdx.x + u * kThreads;
        a[u] = 0.f;
        b[u] = 0.f;
        if (e < kL * DK1) {
            const int t = e / DK1, i = e % DK1;
            if (t < nt) {
                a[u] = i < d_K ? in_f(q[(row0 + t) * d_K + i]) : 1.f;
                b[u] = i < d_K ? in_f(k[(row0 + t) * d_K + i]) : 1.f;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = threadIdx.x + u * kThreads;
        if (e < kL * DK1) {
            xq[e] = a[u];
            xk[e] = b[u];
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = threadIdx.x + u * kThreads;
        a[u] = 0.f;
        if (e < kL * DV1) {
            const int t = e / DV1, j = e % DV1;
            if (t < nt) a[u] = j < d_V ? in_f(v[(row0 + t) * d_V + j]) : 1.f;
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = threadIdx.x + u * kThreads;
        if (e < kL * DV1) xv[e] = a[u];
    }
}

// sum_{g < n} p[g * stride] in a fixed order, eight loads in flight: eight
// running sums over g mod 8, then the tail, then a fixed pairwise combination.
__device__ __forceinline__ float sum_strided(const float *__restrict__ p, int n, int64_t stride) {
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int g = 0;
    for (; g + 8 <= n; g += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = p[(int64_t)(g + u) * stride];
#pragma unroll
        for (int u = 0; u < 8; ++u) s[u] += x[u];
    }
    for (; g < n; ++g) s[0] += p[(int64_t)g * stride];
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

// Register-tiled rank-nt update X[m][j] += sum_t A[t][m] * Y[t][j]: thread
// (warp, lane) owns m = lane + 32a (a < 4) and j = warp + 8n (n < JN).
template <int DV1>
__device__ __forceinline__ void update_rows(float *X, const float *A, const float *Y, int nt) {
    constexpr int JN = (DV1 + 7) / 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float acc[4][JN];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int n = 0; n < JN; ++n) {
            const int j = warp + 8 * n;
            acc[a][n] = j < DV1 ? X[(lane + 32 * a) * DV1 + j] : 0.f;
        }
    for (int t = 0; t < nt; ++t) {
        float x[4], y[JN];
#pragma unroll
        for (int a = 0; a < 4; ++a) x[a] = A[t * kTF + lane + 32 * a];
#pragma unroll
        for (int n = 0; n < JN; ++n) {
            const int j = warp + 8 * n;
            y[n] = j < DV1 ? Y[t * DV1 + j] : 0.f;
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int n = 0; n < JN; ++n) acc[a][n] = fmaf(x[a], y[n], acc[a][n]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int n = 0; n < JN; ++n) {
            const int j = warp + 8 * n;
            if (j < DV1) X[(lane + 32 * a) * DV1 + j] = acc[a][n];
        }
}

// Register-tiled readout acc[b][n] = sum_m A[t][m] * X[m][j] over the kTF
// features, t = warp + 8b (b < 4), j = lane + 32n (n < NJ, j < nj); X rows have
// W floats.
template <int NJ, int W>
__device__ __forceinline__ void readout_cols(const float *A, const float *X, int nj, float (&acc)[4][NJ]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int n = 0; n < NJ; ++n) acc[b][n] = 0.f;
#pragma unroll 4
    for (int m = 0; m < kTF; ++m) {
        float x[NJ], a[4];
#pragma unroll
        for (int n = 0; n < NJ; ++n) {
            const int j = lane + 32 * n;
            x[n] = j < nj ? X[m * W + j] : 0.f;
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) a[b] = A[(warp + 8 * b) * kTF + m];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int n = 0; n < NJ; ++n) acc[b][n] = fmaf(a[b], x[n], acc[b][n]);
    }
}

}  // namespace simt
}  // namespace sata
