// Tensor-core prefill, the finish: the fixed-order sum of unit partials (fixed-order
// mode) and the intra-chunk block on tensor cores with the division.
#pragma once

#include "prefill_tc_common.cuh"

namespace sata {
namespace {

// Sum the G unit partials of every (head, chunk, column, token):
// part [BH][G][nc][DV+1][128] -> red [BH][nc][DV+1][128].  A pure streaming
// kernel (float4, eight loads in flight per thread, fixed summation order).
template <int DV>
__global__ void __launch_bounds__(256)
tc_reduce_kernel(const float4 *__restrict__ part, float4 *__restrict__ red, int BH, int G, int nc) {
    const int64_t per_head = (int64_t)nc * sum_quads(DV) * kL;
    const int64_t total = (int64_t)BH * per_head;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bh = e / per_head, rem = e % per_head;
        const float4 *src = part + bh * G * per_head + rem;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int gg = 0;
        for (; gg + 8 <= G; gg += 8) {
            float4 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = src[(int64_t)(gg + u) * per_head];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc.x += x[u].x; acc.y += x[u].y; acc.z += x[u].z; acc.w += x[u].w;
            }
        }
        for (; gg < G; ++gg) {
            const float4 x = src[(int64_t)gg * per_head];
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
        red[e] = acc;
    }
}

// Per (head, chunk): the intra-chunk block on tensor cores, plus the division.
//   S = Q' K'^T        prescaled fp16 rows (q 2^-e_q, k 2^-e_k), fp32 accumulate in TMEM
//   W[t][s] = sum_{p<P} (S_ts 2^(e_q+e_k) / c)^p / p!  for s <= t, row t scaled by 2^-e_t into the
//                      fp16 range, split into two fp16 parts W_hi + W_lo (about 22 significant
//                      bits: the polynomial's terms can cancel, so one fp16 rounding of W is not
//                      accurate enough)
//   O = W_hi [V'|1] + W_lo [V'|1]   TMEM,  V' = v 2^-e_v
//   out[t] = (2^(e_t+e_v) O_num + num_t) / (2^e_t O_den + den_t), num/den the summed inter-chunk
//            readouts (true frame)
// One CTA per (head, chunk): 8 warps, two per TMEM lane quarter (thread = token row), the
// two halves of a row's weight columns and output columns split between them.
template <int DK, int DV>
struct FinCfg {
    static constexpr int KB = (DK + 63) / 64;          // 64-wide K atoms of Q and K
    static constexpr int NV = DV + 16;
    static constexpr int STG = DV + 4;                 // output staging row stride (floats)
    static constexpr int OFF_Q = 0;                    // [128 t][64 KB d] K-major SW128
    static constexpr int OFF_K = KB * 16384;           // [128 s][64 KB d] K-major SW128
    static constexpr int OFF_W = 2 * KB * 16384;       // W_hi [128 t][128 s] K-major SW128, two K atoms
    static constexpr int OFF_WLO = 0;                  // W_lo, same layout, over Q and K once S is done
    static constexpr int V0 = OFF_W + 32768 > 128 * STG * 4 ? OFF_W + 32768 : 128 * STG * 4;
    static constexpr int OFF_V = (V0 + 1023) / 1024 * 1024;   // [128 s][NV n] MN-major, no swizzle
    static constexpr int LBO_V = (NV / 8) * 128;
    static constexpr int OFF_BAR = OFF_V + 128 * NV * 2;
    static constexpr int OFF_WM = OFF_BAR + 64;        // [2][128] row maxima of the two column halves
    static constexpr int TCOLS = 128 + NV <= 256 ? 256 : 512;
    // with all 512 TMEM columns, one CTA per SM (a shared-memory request above half the SM)
    static constexpr int SMEM0 = OFF_WM + 1024 + 1024;
    static constexpr int SMEM = TCOLS == 512 && SMEM0 < 120 * 1024 ? 120 * 1024 : SMEM0;
    static_assert(2 * KB * 16384 >= 32768, "W_lo");
    static_assert(SMEM <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(256)
tc_finish_kernel(const __half *__restrict__ q16, const __half *__restrict__ k16, const __half *__restrict__ v16,
                 const float *__restrict__ stats, const float *__restrict__ red, float *__restrict__ out,
                 float *__restrict__ den_out, int c0, int nc, int nch, int64_t N, int P, float inv_c, int *flags,
                 int64_t wait_ns, int dvs, int voff) {
    using F = FinCfg<DK, DV>;
    constexpr int NV = F::NV;
    extern __shared__ uint8_t fraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(fraw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const uint32_t bar = sb + F::OFF_BAR;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sm + F::OFF_BAR + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + F::OFF_BAR + 20);
    const int tid = threadIdx.x, warp = tid / 32;
    const int quarter = warp & 3, half = warp >> 2;   // TMEM lane quarter, column half
    const int64_t bh = blockIdx.x / nc;
    const int cl = blockIdx.x % nc;
    const int64_t t0 = (int64_t)(c0 + cl) * kL;
    const int nt = (int)(N - t0 < kL ? N - t0 : kL);
    const HeadExp he = head_exps(stats + bh * 4);
    if (tid == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)),
                     "r"(F::TCOLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // ---- operands: prescaled fp16 rows (chunk-interleaved, token fastest), swizzled
    const uint4 *qcr = chunk_rows<DK>(q16, bh, nch, c0 + cl), *kcr = chunk_rows<DK>(k16, bh, nch, c0 + cl);
    const uint4 *vcr = chunk_rows<DV>(v16, bh, nch, c0 + cl);
    for (int e = tid; e < kL * (DK / 8); e += 256) {   // Q and K: DK/8 pieces of 8 d per row
        const int r = e % kL, c = e / kL;
        uint4 hq = make_uint4(0, 0, 0, 0), hk = make_uint4(0, 0, 0, 0);
        if (r < nt) {
            hq = __ldg(qcr + c * kL + r);
            hk = __ldg(kcr + c * kL + r);
        }
        const int off = (c / 8) * 16384 + r * 128 + (((c % 8) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(sm + F::OFF_Q + off) = hq;
        *reinterpret_cast<uint4 *>(sm + F::OFF_K + off) = hk;
    }
    for (int e = tid; e < kL * (NV / 8); e += 256) {   // [V'|1]: row s, 8 n per 16-byte core row
        const int r = e % kL, c = e / kL;
        uint4 hv = make_uint4(0, 0, 0, 0);
        if (r < nt) {
            if (c < DV / 8) hv = __ldg(vcr + c * kL + r);
            else if (c == DV / 8) hv.x = 0x3C00u;   // the 1 column
        }
        *reinterpret_cast<uint4 *>(sm + F::OFF_V + (r / 8) * F::LBO_V + c * 128 + (r % 8) * 16) = hv;
    }
    fence_proxy_async();
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter W{abort_flag, flags + kFlagTimeout, wait_ns};
    // ---- S = Q' K'^T  [128 t x 128 s], K = DK
    if (tid == 0) {
        constexpr uint32_t id_s = idesc_f16(128, 128, 0, 0);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks)
            tc_mma(tmem, sdesc(sb + F::OFF_Q + (ks / 4) * 16384 + (ks % 4) * 32, 16, 1024, 2),
                   sdesc(sb + F::OFF_K + (ks / 4) * 16384 + (ks % 4) * 32, 16, 1024, 2), id_s, ks > 0 ? 1u : 0u);
        tc_commit(bar);
    }
    __syncwarp();
    bool ok = W.wait(bar, 0);
    tc_after();
    const int t = quarter * 32 + (tid & 31);         // token row = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // ---- W row t: polynomial, causal mask, power-of-two scale into the fp16 range
    // Horner form of sum_{p<P} x^p / p!, x = S' 2^E / c: h <- 1 + h * S' * (2^E / (c p)), P <= 4
    const float xs = pow2f_sat(he.eq + he.ek) * inv_c;
    const float cp1 = xs, cp2 = xs * 0.5f, cp3 = xs * (1.f / 3.f);
    auto wval = [&](float sv, int s) -> float {
        float h = 1.f;
        if (P > 3) h = fmaf(h, sv * cp3, 1.f);
        if (P > 2) h = fmaf(h, sv * cp2, 1.f);
        if (P > 1) h = fmaf(h, sv * cp1, 1.f);
        return (s <= t && t < nt) ? h : 0.f;
    };
    float wmax = 0.f;
    if (ok) {
#pragma unroll 1
        for (int c16 = 4 * half; c16 < 4 * half + 4; ++c16) {
            uint32_t rr[16];
            tc_ld16(tmem + lane_off + c16 * 16, rr);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) wmax = fmaxf(wmax, fabsf(wval(__uint_as_float(rr[i]), c16 * 16 + i)));
        }
    }
    {   // the row's maximum over both column halves
        float *wm = reinterpret_cast<float *>(sm + F::OFF_WM);
        wm[half * 128 + t] = wmax;
        __syncthreads();
        wmax = fmaxf(wm[t], wm[128 + t]);
    }
    // e_t: 2^-e_t wmax < 2^15
    const int ebits = (int)((__float_as_uint(wmax) >> 23) & 255) - 127;
    const int e_t = ebits > 14 ? ebits - 14 : 0;
    const float down = pow2f_sat(-e_t);
    if (ok) {
#pragma unroll 1
        for (int c16 = 4 * half; c16 < 4 * half + 4; ++c16) {
            uint32_t rr[16];
            tc_ld16(tmem + lane_off + c16 * 16, rr);
            tc_wait_ld();
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                __align__(16) __half2 hw[4], lw[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int s0 = c16 * 16 + h8 * 8 + 2 * i;
                    const float w0 = wval(__uint_as_float(rr[h8 * 8 + 2 * i]), s0) * down;
                    const float w1 = wval(__uint_as_float(rr[h8 * 8 + 2 * i + 1]), s0 + 1) * down;
                    hw[i] = __floats2half2_rn(w0, w1);
                    lw[i] = __floats2half2_rn(w0 - __low2float(hw[i]), w1 - __high2float(hw[i]));
                }
                const int s8 = c16 * 2 + h8;                                // 8-wide s group 0..15
                const int off = (s8 / 8) * 16384 + t * 128 + (((s8 % 8) ^ (t & 7)) << 4);
                *reinterpret_cast<uint4 *>(sm + F::OFF_W + off) = *reinterpret_cast<const uint4 *>(hw);
                *reinterpret_cast<uint4 *>(sm + F::OFF_WLO + off) = *reinterpret_cast<const uint4 *>(lw);
            }
        }
    }
    fence_proxy_async();
    tc_before();
    __syncthreads();
    tc_after();
    // ---- O = (W_hi + W_lo) [V'|1]  [128 t x NV], K = 128
    if (tid == 0 && ok) {
        constexpr uint32_t id_o = idesc_f16(128, NV, 0, 1);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc_mma(tmem + 128,
                       sdesc(sb + (part ? F::OFF_WLO : F::OFF_W) + (ks / 4) * 16384 + (ks % 4) * 32, 16, 1024, 2),
                       sdesc(sb + F::OFF_V + ks * 2 * F::LBO_V, F::LBO_V, 128, 0), id_o, (part | ks) ? 1u : 0u);
        tc_commit(bar);
    }
    __syncwarp();
    ok = ok && W.wait(bar, 1);
    tc_after();
    // ---- epilogue: add the inter-chunk sums, divide, stage the row
    float *stg = reinterpret_cast<float *>(sm);
    if (ok) {
        const float upz = pow2f_sat(e_t), upv = pow2f_sat(e_t + he.ev);
        const float4 *rp = reinterpret_cast<const float4 *>(red) + (bh * nc + cl) * sum_quads(DV) * kL + t;
        float inv;
        bool finite = true;
        {   // denominator: column DV
            uint32_t rr[16];
            tc_ld16(tmem + 128 + lane_off + DV, rr);
            tc_wait_ld();
            const float den = fmaf(__uint_as_float(rr[0]), upz, rp[(DV / 4) * kL].x);
            inv = 1.f / den;
            finite = fabsf(inv) <= FLT_MAX;
            if (den_out && half == 0 && t < nt) den_out[bh * N + t0 + t] = den;   // kept for the backward pass
        }
        constexpr int NG = DV / 16, NG0 = (NG + 1) / 2;   // output column groups: [0, NG0) and [NG0, NG)
#pragma unroll
        for (int c16 = half ? NG0 : 0; c16 < (half ? NG : NG0); ++c16) {
            uint32_t rr[16];
            tc_ld16(tmem + 128 + lane_off + c16 * 16, rr);
            tc_wait_ld();
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                const float4 sv = rp[(c16 * 4 + i4) * kL];
                const float sq[4] = {sv.x, sv.y, sv.z, sv.w};
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o[i] = fmaf(__uint_as_float(rr[4 * i4 + i]), upv, sq[i]) * inv;
                    finite = finite && fabsf(o[i]) <= FLT_MAX;
                }
                *reinterpret_cast<float4 *>(stg + t * F::STG + c16 * 16 + 4 * i4) = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
        // a non-finite output (inputs or sums beyond the fp32 range) is reported, never silent
        if (!finite && t < nt) atomicExch(flags + kFlagRange, 1);
    }
    tc_before();
    __syncthreads();
    if (ok) {
        for (int e = tid; e < nt * (DV / 4); e += 256) {
            const int r = e / (DV / 4), c4 = e % (DV / 4);
            reinterpret_cast<float4 *>(out + (bh * N + t0 + r) * dvs + voff)[c4] =
                *reinterpret_cast<const float4 *>(stg + r * F::STG + 4 * c4);
        }
    }
    if (warp == 0) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(F::TCOLS) : "memory");
    }
}

}  // namespace
}  // namespace sata
