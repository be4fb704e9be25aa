// Tensor-core prefill, preparation: per-head maxima of q, k, v and the prescaled fp16
// token rows the scan reads (chunk-interleaved), and the bound of an incoming state.
#pragma once

#include "prefill_tc_common.cuh"

namespace sata {
namespace {

// ----------------------------------------------------------------- prep ----

// Per-head maxima of |q|, |k|, |v| over tokens [t0, t1): max of the bf16 bit
// patterns without sign (a NaN input orders above +inf), then one atomic max per
// block on the fp32 bit pattern (non-negative floats order like their bits).  v's
// rows are dvs values apart (dvs >= DV when a call covers a column range of wider
// rows); the maximum is taken over the whole rows, a valid bound for every range.
__device__ __forceinline__ uint32_t absmax_bits(uint4 u, uint32_t m) {
    m = __vmaxu2(m, u.x & 0x7FFF7FFFu);
    m = __vmaxu2(m, u.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, u.z & 0x7FFF7FFFu);
    return __vmaxu2(m, u.w & 0x7FFF7FFFu);
}
__device__ __forceinline__ float bits_max_to_float(uint32_t m) {
    const uint32_t h = (m >> 16) > (m & 0xFFFFu) ? (m >> 16) : (m & 0xFFFFu);
    return __uint_as_float(h << 16);
}
template <int DK, int DV>
__global__ void __launch_bounds__(256)
tc_stats_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const __nv_bfloat16 *__restrict__ v, float *__restrict__ stats, int64_t N, int64_t t0, int64_t t1,
                int bpb, int dvs) {
    const int64_t bh = blockIdx.x / bpb;   // bpb blocks per head
    const int bx = blockIdx.x % bpb;
    uint32_t mq = 0, mk = 0, mv = 0;
    const int64_t nqk = (t1 - t0) * (DK / 8), nv = (t1 - t0) * (dvs / 8);
    const uint4 *q4 = reinterpret_cast<const uint4 *>(q + (bh * N + t0) * DK);
    const uint4 *k4 = reinterpret_cast<const uint4 *>(k + (bh * N + t0) * DK);
    const uint4 *v4 = reinterpret_cast<const uint4 *>(v + (bh * N + t0) * dvs);
    for (int64_t e = (int64_t)bx * 256 + threadIdx.x; e < nqk; e += (int64_t)bpb * 256) {
        mq = absmax_bits(__ldg(q4 + e), mq);
        mk = absmax_bits(__ldg(k4 + e), mk);
    }
    for (int64_t e = (int64_t)bx * 256 + threadIdx.x; e < nv; e += (int64_t)bpb * 256)
        mv = absmax_bits(__ldg(v4 + e), mv);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mq = __vmaxu2(mq, __shfl_xor_sync(0xffffffffu, mq, off));
        mk = __vmaxu2(mk, __shfl_xor_sync(0xffffffffu, mk, off));
        mv = __vmaxu2(mv, __shfl_xor_sync(0xffffffffu, mv, off));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMax(reinterpret_cast<int *>(stats + bh * 4 + 0), __float_as_int(bits_max_to_float(mq)));
        atomicMax(reinterpret_cast<int *>(stats + bh * 4 + 1), __float_as_int(bits_max_to_float(mk)));
        atomicMax(reinterpret_cast<int *>(stats + bh * 4 + 2), __float_as_int(bits_max_to_float(mv)));
    }
}

// Prescaled fp16 token rows of tokens [t0, t1): q16 = q 2^-e_q, k16 = k 2^-e_k,
// v16 = v 2^-e_v (exact scalings by powers of two; every value below 1).  A head
// whose inputs are not finite raises the range flag (its outputs are NaN).  Source
// rows are ld values apart, the D values taken from column off on.
template <int D>
__device__ __forceinline__ void prep_rows(const __nv_bfloat16 *__restrict__ x, __half *__restrict__ x16,
                                          const float *__restrict__ stats, int which, int BH, int64_t N,
                                          int64_t t0, int64_t t1, int nch, int ld, int off) {
    // one thread per token row: its D/8 pieces are one contiguous read, and for each piece
    // consecutive tokens store consecutive 16-byte elements
    const int64_t ntok = t1 - t0;
    const int64_t total = (int64_t)BH * ntok;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bh = e / ntok;
        const int64_t tok = t0 + (e - bh * ntok);
        const HeadExp he = head_exps(stats + bh * 4);
        const int ex = which == 0 ? he.eq : (which == 1 ? he.ek : he.ev);
        const float sc = pow2f(-ex);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (bh * N + tok) * ld + off);
        uint4 *dst = reinterpret_cast<uint4 *>(x16) + (bh * nch + tok / kL) * (D / 8) * kL + tok % kL;
        uint4 u[D / 8];
#pragma unroll
        for (int j = 0; j < D / 8; ++j) u[j] = __ldg(src + j);
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
                const __half2 h = __floats2half2_rn(lo * sc, hi * sc);
                o[i] = *reinterpret_cast<const uint32_t *>(&h);
            }
            dst[j * kL] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}
template <int DK, int DV>
__global__ void __launch_bounds__(256)
tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               const __nv_bfloat16 *__restrict__ v, const float *__restrict__ stats, __half *__restrict__ q16,
               __half *__restrict__ k16, __half *__restrict__ v16, int BH, int64_t N, int64_t t0, int64_t t1,
               int nch, int *flags, int dvs, int voff) {
    if (blockIdx.x == 0)
        for (int bh = threadIdx.x; bh < BH; bh += blockDim.x)
            if (!(stats[bh * 4] <= FLT_MAX && stats[bh * 4 + 1] <= FLT_MAX && stats[bh * 4 + 2] <= FLT_MAX))
                atomicExch(flags + kFlagRange, 1);
    prep_rows<DK>(q, q16, stats, 0, BH, N, t0, t1, nch, DK, 0);
    prep_rows<DK>(k, k16, stats, 1, BH, N, t0, t1, nch, DK, 0);
    prep_rows<DV>(v, v16, stats, 2, BH, N, t0, t1, nch, dvs, voff);
}

// max |S|, |Z| of each head of an incoming state -> stats[bh][3] (S rows of DV values: the
// whole rows when a call covers a column range of them).  The state is read once per
// segment before the scan can start, so it is read as 16-byte elements (S is 16-byte
// aligned, DV a multiple of 4) by a grid that spans the SMs, several loads in flight per
// thread.
__global__ void __launch_bounds__(256)
tc_state_stats_kernel(const float *__restrict__ S, const float *__restrict__ Z, float *__restrict__ stats, int64_t F,
                      int DV) {
    const int64_t bh = blockIdx.x;
    const int64_t i0 = blockIdx.y * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.y * blockDim.x;
    const int64_t n4 = F * DV / 4;
    const float4 *S4 = reinterpret_cast<const float4 *>(S + bh * F * DV);
    float m = 0.f;
#pragma unroll 4
    for (int64_t i = i0; i < n4; i += stride) {
        const float4 x = __ldg(S4 + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
    }
    for (int64_t i = i0; i < F; i += stride) m = fmaxf(m, fabsf(__ldg(Z + bh * F + i)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<int *>(stats + bh * 4 + 3), __float_as_int(m));
}

}  // namespace
}  // namespace sata
