// Register-tiled building blocks of the CUDA-core scans (prefill and its
// backward): 256 threads, tiles of kTF = 128 features, chunks of kL = 32 tokens.
// Thread (warp, lane) owns tokens t = warp + 8b (b < 4) and features
// m = lane + 32a (a < 4) or value columns; every operand row is read from shared
// memory once per thread and reused across the thread's register tile.
// Shared-memory rows of d_V + 1 floats have an odd stride for every supported
// d_V, so the 32 lanes of a warp reading 32 different rows hit 32 banks.
#pragma once

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

// Register-tiled contraction out[t][m] = coef[m] * sum_j X[m][j] * Y[t][j] over
// the j < DV1 columns (X: a tile's state rows, Y: the chunk's r or u rows):
// thread (warp, lane) owns t = warp + 8b (b < 4) and m = lane + 32a (a < 4).
template <int DV1>
__device__ __forceinline__ void contract_rows(const float *X, const float *Y, const float *coef, float *out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float acc[4][4] = {};
#pragma unroll 4
    for (int j = 0; j < DV1; ++j) {
        float x[4], y[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) x[a] = X[(lane + 32 * a) * DV1 + j];
#pragma unroll
        for (int b = 0; b < 4; ++b) y[b] = Y[(warp + 8 * b) * DV1 + j];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[b][a] = fmaf(y[b], x[a], acc[b][a]);
    }
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int a = 0; a < 4; ++a)
            out[(warp + 8 * b) * kTF + lane + 32 * a] = coef[lane + 32 * a] * acc[b][a];
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
