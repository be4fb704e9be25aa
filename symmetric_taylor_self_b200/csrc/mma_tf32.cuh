// Warp-level tensor-core contractions for the backward scans: mma.sync
// m16n8k8 with tf32 operands and fp32 accumulation, each fp32 operand split
// into a tf32 high part and a tf32 remainder, and the three products that
// matter summed (a_lo b_hi + a_hi b_lo + a_hi b_hi): about fp32 accuracy with
// fp32 range, so the state needs no scaling.
//
// Fragment layout of m16n8k8 (.tf32), g = lane / 4, c = lane % 4:
//   A (16 x 8, row-major): a0 (g, c), a1 (g + 8, c), a2 (g, c + 4), a3 (g + 8, c + 4)
//   B (8 x 8, k x n):      b0 (k = c, n = g), b1 (k = c + 4, n = g)
//   D (16 x 8):            d0 (g, 2c), d1 (g, 2c + 1), d2 (g + 8, 2c), d3 (g + 8, 2c + 1)
//
// Shared-memory strides are chosen so that a warp's fragment loads hit 32
// distinct banks: an operand whose fragment rows run over g needs a row stride
// of 4 mod 8 floats (4g + c distinct), one whose rows run over c needs 8 mod 16
// (8c + g distinct).
#pragma once

#include <cstdint>

namespace sata {
namespace mma32 {

constexpr int kTF = 128;   // features per CTA (the N or M extent of the feature side)
constexpr int kL = 32;     // tokens per chunk

// Padded widths of a row of d_V + 1 values.
__host__ __device__ constexpr int cols8(int n) { return (n + 7) / 8 * 8; }            // K / N extent
__host__ __device__ constexpr int stride_g(int n) { return cols8(n) + 4; }             // rows over g
__host__ __device__ constexpr int stride_c(int n) { return cols8(n) % 16 == 8 ? cols8(n) : cols8(n) + 8; }
constexpr int kFeatG = kTF + 4;   // [kL][kTF] arrays read with rows over g
constexpr int kFeatC = kTF + 8;   // [kL][kTF] arrays read with rows over c

__device__ __forceinline__ void split(float x, uint32_t &hi, uint32_t &lo) {
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float r = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}

__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += A B with split operands (three tf32 products).
__device__ __forceinline__ void mma3(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], uint32_t bh0,
                                     uint32_t bh1, uint32_t bl0, uint32_t bl1) {
    mma(d, al, bh0, bh1);
    mma(d, ah, bl0, bl1);
    mma(d, ah, bh0, bh1);
}

// A fragment of rows r0 .. r0+15, columns k0 .. k0+7 of a row-major array
// (element (r, k) at p[r * ld + k]).
__device__ __forceinline__ void load_a_rows(const float *p, int ld, int r0, int k0, uint32_t (&h)[4],
                                            uint32_t (&l)[4]) {
    const int g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
    split(p[(r0 + g) * ld + k0 + c], h[0], l[0]);
    split(p[(r0 + g + 8) * ld + k0 + c], h[1], l[1]);
    split(p[(r0 + g) * ld + k0 + c + 4], h[2], l[2]);
    split(p[(r0 + g + 8) * ld + k0 + c + 4], h[3], l[3]);
}

// A fragment whose element (m, k) is stored transposed at p[k * ld + m].
__device__ __forceinline__ void load_a_cols(const float *p, int ld, int m0, int k0, uint32_t (&h)[4],
                                            uint32_t (&l)[4]) {
    const int g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
    split(p[(k0 + c) * ld + m0 + g], h[0], l[0]);
    split(p[(k0 + c) * ld + m0 + g + 8], h[1], l[1]);
    split(p[(k0 + c + 4) * ld + m0 + g], h[2], l[2]);
    split(p[(k0 + c + 4) * ld + m0 + g + 8], h[3], l[3]);
}

// B fragment whose element (k, n) is stored at p[n * ld + k] (rows over g).
__device__ __forceinline__ void load_b_nk(const float *p, int ld, int n0, int k0, uint32_t &h0, uint32_t &h1,
                                          uint32_t &l0, uint32_t &l1) {
    const int g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
    split(p[(n0 + g) * ld + k0 + c], h0, l0);
    split(p[(n0 + g) * ld + k0 + c + 4], h1, l1);
}

// B fragment whose element (k, n) is stored at p[k * ld + n] (rows over c).
__device__ __forceinline__ void load_b_kn(const float *p, int ld, int n0, int k0, uint32_t &h0, uint32_t &h1,
                                          uint32_t &l0, uint32_t &l1) {
    const int g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
    split(p[(k0 + c) * ld + n0 + g], h0, l0);
    split(p[(k0 + c + 4) * ld + n0 + g], h1, l1);
}

// out[t][m] = coef[m] * sum_j X[m][j] Y[t][j] for t < 32, m < 128, j < K
// (K = cols8(d_V + 1); X rows stride ldx (rows over g), Y rows stride ldy (rows
// over g), out rows stride ldo).  Warp w owns token rows 16 (w & 1) .. +15 and
// feature columns 32 (w >> 1) .. +31.
template <int K>
__device__ __forceinline__ void contract_rows(const float *X, int ldx, const float *Y, int ldy, const float *coef,
                                              float *out, int ldo) {
    const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
    const int t0 = 16 * (warp & 1), m0 = 32 * (warp >> 1);
    float d[4][4] = {};
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t ah[4], al[4];
        load_a_rows(Y, ldy, t0, k0, ah, al);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            uint32_t bh0, bh1, bl0, bl1;
            load_b_nk(X, ldx, m0 + 8 * n, k0, bh0, bh1, bl0, bl1);
            mma3(d[n], ah, al, bh0, bh1, bl0, bl1);
        }
    }
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int m = m0 + 8 * n + 2 * c;
        const float c0 = coef[m], c1 = coef[m + 1];
        out[(t0 + g) * ldo + m] = c0 * d[n][0];
        out[(t0 + g) * ldo + m + 1] = c1 * d[n][1];
        out[(t0 + g + 8) * ldo + m] = c0 * d[n][2];
        out[(t0 + g + 8) * ldo + m + 1] = c1 * d[n][3];
    }
}

// X[m][j] += sum_t A[t][m] Y[t][j] for m < 128, j < NJ * 8, t < 32 (X rows
// stride ldx, A [t][m] stride lda (rows over c), Y [t][j] stride ldy (rows over
// c)).  Warp w owns feature rows 16 w .. 16 w + 15 and every column.
template <int NJ>
__device__ __forceinline__ void update_rows(float *X, int ldx, const float *A, int lda, const float *Y, int ldy) {
    const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
    const int m0 = 16 * warp;
    float d[NJ][4];
#pragma unroll
    for (int n = 0; n < NJ; ++n) {
        const int j = 8 * n + 2 * c;
        d[n][0] = X[(m0 + g) * ldx + j];
        d[n][1] = X[(m0 + g) * ldx + j + 1];
        d[n][2] = X[(m0 + g + 8) * ldx + j];
        d[n][3] = X[(m0 + g + 8) * ldx + j + 1];
    }
#pragma unroll
    for (int k0 = 0; k0 < kL; k0 += 8) {
        uint32_t ah[4], al[4];
        load_a_cols(A, lda, m0, k0, ah, al);
#pragma unroll
        for (int n = 0; n < NJ; ++n) {
            uint32_t bh0, bh1, bl0, bl1;
            load_b_kn(Y, ldy, 8 * n, k0, bh0, bh1, bl0, bl1);
            mma3(d[n], ah, al, bh0, bh1, bl0, bl1);
        }
    }
#pragma unroll
    for (int n = 0; n < NJ; ++n) {
        const int j = 8 * n + 2 * c;
        X[(m0 + g) * ldx + j] = d[n][0];
        X[(m0 + g) * ldx + j + 1] = d[n][1];
        X[(m0 + g + 8) * ldx + j] = d[n][2];
        X[(m0 + g + 8) * ldx + j + 1] = d[n][3];
    }
}

// out[t][j] = sum_m A[t][m] G[m][j] for t < 32, j < NT * 8, m < 128 (A [t][m]
// stride lda (rows over g), G rows stride ldg).  The 2 x NT output tiles are
// dealt to the 8 warps round-robin; fn(t, j, value) receives each result.
template <int NT, typename Fn>
__device__ __forceinline__ void readout_cols(const float *A, int lda, const float *G, int ldg, Fn fn) {
    const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2, c = threadIdx.x & 3;
#pragma unroll
    for (int tile = warp; tile < 2 * NT; tile += 8) {
        const int t0 = 16 * (tile & 1), n0 = 8 * (tile >> 1);
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int k0 = 0; k0 < kTF; k0 += 8) {
            uint32_t ah[4], al[4], bh0, bh1, bl0, bl1;
            load_a_rows(A, lda, t0, k0, ah, al);
            load_b_kn(G, ldg, n0, k0, bh0, bh1, bl0, bl1);
            mma3(d, ah, al, bh0, bh1, bl0, bl1);
        }
        fn(t0 + g, n0 + 2 * c, d[0]);
        fn(t0 + g, n0 + 2 * c + 1, d[1]);
        fn(t0 + g + 8, n0 + 2 * c, d[2]);
        fn(t0 + g + 8, n0 + 2 * c + 1, d[3]);
    }
}

}  // namespace mma32
}  // namespace sata
