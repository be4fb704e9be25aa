// Tensor-core prefill for sm_100a: the chunked state scan on tcgen05 / TMEM.
//
// [CC-TAYLOR] = "Self-attention at constant cost per token via symmetry-aware
// Taylor approximation" (blog.hotdry.top).  Section "Feature maps and linear
// attention" (特征映射与线性注意力): states Z_p = sum phi_p(k), S_p = sum phi_p(k) v^T,
// computable by a parallel prefix scan; output y = sum_p alpha_p phi_p(q)^T C_p S_p /
// sum_p alpha_p <phi_p(q), Z_p>_C.  Section "Hardware optimization paths"
// (硬件优化实现路径): build features without copies, exploit the shared prefixes of
// the nondecreasing index tuples, evaluate the terms concurrently, keep hot data
// on chip.  [CC-HW] "Constant-cost attention: hardware optimization", section
// "Compute density": phi = x[..., M].prod(-1); section "Future directions": fuse
// the feature map with the prefix accumulation.
//
// Chunked form (chunk c of L = 128 tokens, feature tile j of 128 features):
//   readout  D_O[t, :] += (alpha C phi_j(q_t)) . [S|Z]_j(before c)     (tcgen05, TMEM)
//   update   [S|Z]_j    += phi_j(K_c)^T [V_c | 1]                      (tcgen05, TMEM)
//   intra    sum_{s in c, s <= t} w_ts [v_s | 1], w = sum_p (q.k/c)^p/p!  (finish kernel)
// One CTA owns MT feature tiles of one head; its [S|Z] tiles stay resident in
// TMEM (fp32) for the whole sequence, so the state never travels through HBM.
// Features are generated on the fly from the chunk's k and q columns into
// shared memory, never written to HBM.
//
// Operand precision: fp16 operands, fp32 accumulation (the fp16 rate equals the
// bf16 rate; its 3 extra mantissa bits keep the per-token error well inside
// 2e-3, which bf16 features do not).  The state is rounded to fp16 only as the
// readout operand, after an exact power-of-two scale 2^-sigma_c chosen from a
// rigorous bound |S| <= |S_init| + tokens * max(1,|k|)^(P-1) * max(1,|v|), and the
// readout result is scaled back by 2^sigma_c in fp32: no fp16 overflow is
// possible.  Inputs must satisfy |k| <= 40, |q|/c <= 40, |v| <= 60000 (fp16
// features); otherwise the call reports SATA_ERANGE at sync.
//
// Kernels: tc_prep (chunk images + per-head maxima), tc_state_stats (max |state|
// when continuing), tc_scan (the warp-specialised scan), tc_finish (sum of the
// feature-tile partials, intra-chunk block, division).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kL = 128;               // chunk length (tokens)
constexpr int kNQ = 2;                // ring stages of alpha*C*phi(q) tiles (shared memory)
constexpr int kStageBytes = 128 * kL * 2;
constexpr int kScanThreads = 448;     // 14 warps
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpConv0 = 2, kWarpGen0 = 6;
constexpr int kGenWarps = 8;
constexpr int64_t kDefaultWaitNs = 2000000000LL;   // 2 s per wait
constexpr size_t kPartialBudget = size_t(4) << 30;

template <int DK, int DV>
struct Cfg {
    static constexpr int NV = DV + 16;                           // MMA N: [V | 1 | 0 pad]
    static constexpr int MT_MAX = DV == 64 ? 4 : (DV == 32 ? 8 : 12);
    static constexpr int ROW = kL * 2;                           // one (q/c)^T row: 128 fp16
    static constexpr int KROW = ROW + 16;                        // k^T rows padded so that 32 lanes
                                                                 // reading 32 rows hit distinct banks
    static constexpr int IMG_V = NV * ROW;                       // [V|1]^T, K-major SW128
    static constexpr int OFF_IQ = IMG_V;                         // (q/c)^T, row DK = 1
    static constexpr int OFF_IK = IMG_V + (DK + 1) * ROW;        // k^T, row DK = 1
    static constexpr int IMG = OFF_IK + (DK + 1) * KROW;
    static constexpr int IMG_PAD = (IMG + 1023) / 1024 * 1024;
    static constexpr int OFF_RING = 2 * IMG_PAD;
    static constexpr int OFF_BS = OFF_RING + kNQ * kStageBytes;
    static constexpr int BS_BYTES = 128 * NV * 2;
    static constexpr int OFF_TAB = OFF_BS + 2 * BS_BYTES;
    static constexpr int OFF_MC = OFF_TAB + MT_MAX * 128 * 4;
    static constexpr int OFF_BAR = (OFF_MC + MT_MAX * 128 * 2 + 15) / 16 * 16;
    // barrier indices (pairs are double buffers)
    static constexpr int B_INF = 0, B_INE = 2, B_QF = 4, B_QE = 6, B_KF = 8, B_KE = 10, B_BSF = 12,
                         B_BSE = 14, B_SD = 16, B_OF = B_SD + MT_MAX, B_OE = B_OF + 1, B_FIN = B_OE + 1,
                         N_BAR = B_FIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;            // + base alignment slack
    static constexpr int COL_O = MT_MAX * NV;                    // TMEM: readout accumulator
    static constexpr int COL_A = COL_O + NV;                     // TMEM: two phi(k) stages, 32 columns each
    static constexpr int LBO_BS = (NV / 8) * 128;
    static_assert(COL_A + 64 <= 512, "TMEM columns");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(NV % 16 == 0, "MMA N");
};

struct ScanParams {
    const uint8_t *img;       // [BH][nchunks][IMG]
    const float *stats;       // [BH][4] max|q|, max|k|, max|v|, max|state|
    const uint32_t *packed;   // basis: a | b<<8 | l<<16 | p<<24
    const float *mcoef;       // C/p!
    float *S, *Z;             // state in/out
    float *part;              // [BH][G][nc][DV+1][128]
    int *flags;
    int64_t F, N;
    int BH, G, MT, c0, nc, nchunks, P;
    int load_state, store_state, stall_chunk;
    float inv_c;
    int64_t wait_ns;
};

// ----------------------------------------------------------------- PTX ----

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or the hint (ns) elapses, instead of spinning.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ int64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return (int64_t)t;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// A operand in TMEM (rows on lanes, two fp16 per 32-bit column, even K in the low half).
__device__ __forceinline__ void tc_mma_ta(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (start, leading/stride byte offsets, layout:
// 0 = no swizzle (core matrices), 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)(layout & 7) << 61);
}
// Instruction descriptor for kind::f16: fp16 A and B, fp32 D, M x N, operand majors.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float pow2f(int e) {   // exact 2^e, |e| <= 126
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// Exponent sigma_c such that |state before chunk c| * 2^-sigma_c < 2^15.
__device__ __forceinline__ int state_sigma(int64_t c, float mk, float mv, float ms, int P) {
    const float kk = fmaxf(1.f, mk);
    float mphi = 1.f;
    for (int p = 1; p < P; ++p) mphi *= kk;
    const float bound = ms + (float)c * (float)kL * mphi * fmaxf(1.f, mv) + 1.f;
    const int e = (int)((__float_as_uint(bound) >> 23) & 255) - 126;   // bound < 2^e
    int s = e - 15;
    return s < -100 ? -100 : (s > 100 ? 100 : s);
}

struct Waiter {
    volatile int *abort_flag;
    int *gflag;
    int64_t limit;
    // Bounded wait on an mbarrier phase.  On expiry: raise the CTA abort flag and
    // the device timeout flag, return false.  Also returns false once another
    // role has aborted.
    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
        if (mbar_try(bar, parity)) return true;
        const int64_t t0 = gtimer();
        while (true) {
            if (mbar_try_sleep(bar, parity, 100000u)) return true;
            if (*abort_flag) return false;
            if (gtimer() - t0 > limit) {
                *abort_flag = 1;
                atomicExch(gflag, 1);
                return false;
            }
        }
    }
    // Bounded wait that ignores the abort flag (draining in-flight async work).
    __device__ __forceinline__ bool drain(uint32_t bar, uint32_t parity) const {
        const int64_t t0 = gtimer();
        while (!mbar_try_sleep(bar, parity, 100000u)) {
            if (gtimer() - t0 > limit) {
                atomicExch(gflag, 1);
                return false;
            }
        }
        return true;
    }
};

__device__ __forceinline__ uint4 hmul4(uint4 a, uint4 b) {
    uint4 r;
    __half2 *ra = reinterpret_cast<__half2 *>(&a), *rb = reinterpret_cast<__half2 *>(&b),
            *rr = reinterpret_cast<__half2 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) rr[i] = __hmul2(ra[i], rb[i]);
    return r;
}
__device__ __forceinline__ uint4 hmul4s(uint4 a, __half2 m) {
    uint4 r;
    __half2 *ra = reinterpret_cast<__half2 *>(&a), *rr = reinterpret_cast<__half2 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) rr[i] = __hmul2(ra[i], m);
    return r;
}

// ----------------------------------------------------------------- prep ----

// Per (head, chunk): write the chunk image [ [V|1]^T (K-major, 128-byte swizzle)
// | (q/c)^T | k^T (rows padded to 272 bytes) ], fp16, padded tokens zero
// (including their 1 entries), and raise the per-head maxima of |q|, |k|, |v|.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               const __nv_bfloat16 *__restrict__ v, uint8_t *__restrict__ img,
               float *__restrict__ stats, int BH, int64_t N, int nchunks, float inv_c) {
    using C = Cfg<DK, DV>;
    constexpr int PK = DK + 2, PV = DV + 2;
    extern __shared__ __half psm[];
    __half *sk = psm;                 // [128][PK]
    __half *sq = sk + kL * PK;        // [128][PK]
    __half *sv = sq + kL * PK;        // [128][PV]
    __shared__ float red[3][8];
    const int tid = threadIdx.x;
    const __half one = __float2half(1.f), zero = __float2half(0.f);
    for (int64_t idx = blockIdx.x; idx < (int64_t)BH * nchunks; idx += gridDim.x) {
        const int64_t bh = idx / nchunks;
        const int c = (int)(idx % nchunks);
        const int64_t t0 = (int64_t)c * kL;
        const int nt = (int)(N - t0 < kL ? N - t0 : kL);
        float mq = 0.f, mk = 0.f, mv = 0.f;
        for (int e = tid; e < kL * DK / 8; e += 256) {
            const int t = e / (DK / 8), i8 = (e % (DK / 8)) * 8;
            uint4 rk = make_uint4(0, 0, 0, 0), rq = make_uint4(0, 0, 0, 0);
            if (t < nt) {
                rk = *reinterpret_cast<const uint4 *>(k + (bh * N + t0 + t) * DK + i8);
                rq = *reinterpret_cast<const uint4 *>(q + (bh * N + t0 + t) * DK + i8);
            }
            const __nv_bfloat16 *bk = reinterpret_cast<const __nv_bfloat16 *>(&rk);
            const __nv_bfloat16 *bq = reinterpret_cast<const __nv_bfloat16 *>(&rq);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float fk = __bfloat162float(bk[j]), fq = __bfloat162float(bq[j]);
                mk = fmaxf(mk, fabsf(fk));
                mq = fmaxf(mq, fabsf(fq));
                sk[t * PK + i8 + j] = __float2half_rn(fk);
                sq[t * PK + i8 + j] = __float2half_rn(fq * inv_c);
            }
        }
        for (int e = tid; e < kL * DV / 8; e += 256) {
            const int t = e / (DV / 8), i8 = (e % (DV / 8)) * 8;
            uint4 rv = make_uint4(0, 0, 0, 0);
            if (t < nt) rv = *reinterpret_cast<const uint4 *>(v + (bh * N + t0 + t) * DV + i8);
            const __nv_bfloat16 *bv = reinterpret_cast<const __nv_bfloat16 *>(&rv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float fv = __bfloat162float(bv[j]);
                mv = fmaxf(mv, fabsf(fv));
                sv[t * PV + i8 + j] = __float2half_rn(fv);
            }
        }
        __syncthreads();
        uint8_t *out = img + idx * (int64_t)C::IMG;
        // [V|1]^T: element (n, t) at (t/64)*(NV*128) + n*128 + ((((t%64)/8) ^ (n%8))*16) + (t%8)*2
        for (int e = tid; e < C::NV * 16; e += 256) {
            const int n = e / 16, t8 = e % 16;
            __align__(16) __half h[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = t8 * 8 + j;
                h[j] = n < DV ? sv[t * PV + n] : ((n == DV && t < nt) ? one : zero);
            }
            const int off = (t8 / 8) * (C::NV * 128) + n * 128 + (((t8 % 8) ^ (n % 8)) * 16);
            *reinterpret_cast<uint4 *>(out + off) = *reinterpret_cast<const uint4 *>(h);
        }
        // k^T and (q/c)^T: row i holds tokens 0..127; row DK is 1 (0 for padded tokens)
        for (int e = tid; e < (DK + 1) * 16; e += 256) {
            const int i = e / 16, t8 = e % 16;
            __align__(16) __half hk[8], hq[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = t8 * 8 + j;
                hk[j] = i < DK ? sk[t * PK + i] : (t < nt ? one : zero);
                hq[j] = i < DK ? sq[t * PK + i] : (t < nt ? one : zero);
            }
            *reinterpret_cast<uint4 *>(out + C::OFF_IK + i * C::KROW + t8 * 16) = *reinterpret_cast<const uint4 *>(hk);
            *reinterpret_cast<uint4 *>(out + C::OFF_IQ + i * C::ROW + t8 * 16) = *reinterpret_cast<const uint4 *>(hq);
        }
        // per-head maxima (non-negative floats order like their bit patterns)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, off));
            mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, off));
            mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, off));
        }
        if ((tid & 31) == 0) {
            red[0][tid / 32] = mq;
            red[1][tid / 32] = mk;
            red[2][tid / 32] = mv;
        }
        __syncthreads();
        if (tid < 3) {
            float m = 0.f;
            for (int w = 0; w < 8; ++w) m = fmaxf(m, red[tid][w]);
            atomicMax(reinterpret_cast<int *>(stats + bh * 4 + tid), __float_as_int(m));
        }
        __syncthreads();
    }
}

// max |S|, |Z| of each head of an incoming state -> stats[bh][3]
__global__ void tc_state_stats_kernel(const float *__restrict__ S, const float *__restrict__ Z,
                                      float *__restrict__ stats, int64_t F, int DV) {
    const int64_t bh = blockIdx.x;
    float m = 0.f;
    const int64_t nS = F * DV;
    for (int64_t i = blockIdx.y * (int64_t)blockDim.x + threadIdx.x; i < nS + F;
         i += (int64_t)gridDim.y * blockDim.x) {
        const float x = i < nS ? S[bh * nS + i] : Z[bh * F + (i - nS)];
        m = fmaxf(m, fabsf(x));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<int *>(stats + bh * 4 + 3), __float_as_int(m));
}

// ----------------------------------------------------------------- scan ----

template <int DK, int DV>
__global__ void __launch_bounds__(kScanThreads, 1) tc_scan_kernel(const ScanParams p) {
    using C = Cfg<DK, DV>;
    constexpr int NV = C::NV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto BAR = [bar0](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    uint32_t *tab = reinterpret_cast<uint32_t *>(smem + C::OFF_TAB);
    __half *mc = reinterpret_cast<__half *>(smem + C::OFF_MC);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t bh = blockIdx.x / p.G;
    const int g = blockIdx.x % p.G;
    const int64_t f0 = (int64_t)g * p.MT * 128;
    const float mq = p.stats[bh * 4 + 0], mk = p.stats[bh * 4 + 1], mv = p.stats[bh * 4 + 2],
                ms = p.stats[bh * 4 + 3];
    // fp16 operand range (uniform over the CTA: exit before any barrier or TMEM use)
    if (!(mq * p.inv_c <= 40.f && mk <= 40.f && mv <= 60000.f && ms <= 1e30f)) {
        if (threadIdx.x == 0) atomicExch(p.flags + kFlagRange, 1);
        return;
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::N_BAR; ++i) {
            uint32_t cnt = 1;
            if (i == C::B_INE || i == C::B_INE + 1) cnt = kGenWarps + 1;
            else if ((i >= C::B_QF && i < C::B_QF + 2) || (i >= C::B_KF && i < C::B_KF + 2)) cnt = kGenWarps;
            else if (i == C::B_BSF || i == C::B_BSF + 1 || i == C::B_OE) cnt = 4;
            mbar_init(BAR(i), cnt);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpProducer) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_before();
    }
    if (warp >= kWarpGen0) {   // this CTA's feature descriptors
        const uint32_t pad = (uint32_t)DK | ((uint32_t)DK << 8) | ((uint32_t)DK << 16);
        for (int i = threadIdx.x - kWarpGen0 * 32; i < C::MT_MAX * 128; i += kGenWarps * 32) {
            const int64_t f = f0 + i;
            const bool ok = i < p.MT * 128 && f < p.F;
            tab[i] = ok ? (p.packed[f] & 0xFFFFFFu) : pad;
            mc[i] = __float2half_rn(ok ? p.mcoef[f] : 0.f);
        }
    }
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter W{abort_flag, p.flags + kFlagTimeout, p.wait_ns};

    if (warp == kWarpProducer) {
        // ------------------------------------------------ chunk images in
        if (lane == 0) {
            int last[2] = {-1, -1};
            for (int cl = 0; cl < p.nc; ++cl) {
                const int ib = cl & 1;
                if (!W.wait(BAR(C::B_INE + ib), ((cl >> 1) & 1) ^ 1)) break;
                if (p.c0 + cl == p.stall_chunk) continue;   // test hook: withhold this chunk
                mbar_expect_tx(BAR(C::B_INF + ib), C::IMG);
                bulk_g2s(sb + ib * C::IMG_PAD, p.img + ((int64_t)bh * p.nchunks + p.c0 + cl) * C::IMG, C::IMG,
                         BAR(C::B_INF + ib));
                last[ib] = cl;
            }
            for (int ib = 0; ib < 2; ++ib)   // no copy may still be landing at exit
                if (last[ib] >= 0) W.drain(BAR(C::B_INF + ib), (last[ib] >> 1) & 1);
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
            constexpr uint32_t id_upd = idesc_f16(128, NV, 0, 0);
            constexpr uint32_t id_rd = idesc_f16(128, NV, 1, 1);
            int qa = 0, qk = 0;
            bool ok = true;
            for (int cl = 0; cl < p.nc && ok; ++cl) {
                const int ib = cl & 1;
                if (!(ok = W.wait(BAR(C::B_INF + ib), (cl >> 1) & 1))) break;
                const uint32_t vimg = sb + ib * C::IMG_PAD;
                for (int j = 0; j < p.MT; ++j) {
                    const int qn = cl * p.MT + j, bsb = qn & 1, sa = qa & 1;
                    ok = W.wait(BAR(C::B_BSF + bsb), (qn >> 1) & 1) && W.wait(BAR(C::B_QF + sa), (qa >> 1) & 1);
                    if (ok && j == 0) ok = W.wait(BAR(C::B_OE), (cl & 1) ^ 1);   // epilogue of cl-1 done
                    if (!ok) break;
                    tc_after();
                    // readout: D_O += (alpha C phi(q)) [128 t x 128 f] . [S|Z]_j fp16 [128 f x NV]
                    const uint32_t a_st = sb + C::OFF_RING + sa * kStageBytes;
                    const uint32_t b_s = sb + C::OFF_BS + bsb * C::BS_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc_mma(tmem + C::COL_O, sdesc(a_st + ks * 2048, 16384, 1024, 2),
                               sdesc(b_s + ks * 2 * C::LBO_BS, C::LBO_BS, 128, 0), id_rd,
                               (j > 0 || ks > 0) ? 1u : 0u);
                    tc_commit(BAR(C::B_QE + sa));
                    tc_commit(BAR(C::B_BSE + bsb));
                    if (j == p.MT - 1) tc_commit(BAR(C::B_OF));
                    ++qa;
                    // update: [S|Z]_j += phi(K)^T [128 f x 64 t] (TMEM) . [V|1] [64 t x NV], two halves
                    for (int h = 0; h < 2 && ok; ++h) {
                        const int sk = qk & 1;
                        if (!(ok = W.wait(BAR(C::B_KF + sk), (qk >> 1) & 1))) break;
                        tc_after();
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc_mma_ta(tmem + j * NV, tmem + C::COL_A + sk * 32 + ks * 8,
                                      sdesc(vimg + h * (NV * 128) + ks * 32, 16, 1024, 2), id_upd, 1u);
                        tc_commit(BAR(C::B_KE + sk));
                        ++qk;
                    }
                    if (!ok) break;
                    tc_commit(BAR(C::B_SD + j));
                }
                if (!ok) break;
                tc_commit(BAR(C::B_INE + ib));
            }
            // every issued MMA completes before TMEM is released
            tc_commit(BAR(C::B_FIN));
            W.drain(BAR(C::B_FIN), 0);
        }
    } else if (warp >= kWarpConv0 && warp < kWarpGen0) {
        // ------------------------------------------------ state conversion + epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint32_t r[NV];
        // initial state -> TMEM (zeros for a fresh sequence)
        for (int j = 0; j < p.MT; ++j) {
            const int64_t f = f0 + j * 128 + row;
            const bool have = p.load_state && f < p.F;
#pragma unroll
            for (int col = 0; col < NV; ++col) {
                float x = 0.f;
                if (have && col < DV) x = p.S[(bh * p.F + f) * DV + col];
                else if (have && col == DV) x = p.Z[bh * p.F + f];
                r[col] = __float_as_uint(x);
            }
#pragma unroll
            for (int c16 = 0; c16 < NV / 16; ++c16) tc_st16(tmem + lane_off + j * NV + c16 * 16, r + c16 * 16);
        }
        tc_wait_st();
        int64_t part_base = ((int64_t)bh * p.G + g) * p.nc;
        auto epilogue = [&](int cl) -> bool {
            if (!W.wait(BAR(C::B_OF), cl & 1)) return false;
            tc_after();
#pragma unroll
            for (int c16 = 0; c16 < NV / 16; ++c16) tc_ld16(tmem + lane_off + C::COL_O + c16 * 16, r + c16 * 16);
            tc_wait_ld();
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_OE));
            const float up = pow2f(state_sigma(p.c0 + cl, mk, mv, ms, p.P));
            float *dst = p.part + ((part_base + cl) * (DV + 1)) * kL + row;
#pragma unroll
            for (int col = 0; col <= DV; ++col) dst[col * kL] = __uint_as_float(r[col]) * up;
            return true;
        };
        bool ok = true;
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const float down = pow2f(-state_sigma(p.c0 + cl, mk, mv, ms, p.P));
            for (int j = 0; j < p.MT; ++j) {
                const int qn = cl * p.MT + j, bsb = qn & 1;
                if (cl > 0 && !(ok = W.wait(BAR(C::B_SD + j), (cl - 1) & 1))) break;
                tc_after();
#pragma unroll
                for (int c16 = 0; c16 < NV / 16; ++c16) tc_ld16(tmem + lane_off + j * NV + c16 * 16, r + c16 * 16);
                tc_wait_ld();
                if (!(ok = W.wait(BAR(C::B_BSE + bsb), ((qn >> 1) & 1) ^ 1))) break;
                // B_s: [S|Z]_j * 2^-sigma as fp16, K = feature rows, N-major core matrices
                uint8_t *bs = smem + C::OFF_BS + bsb * C::BS_BYTES + (row / 8) * C::LBO_BS + (row % 8) * 16;
#pragma unroll
                for (int m = 0; m < NV / 8; ++m) {
                    __align__(16) __half2 h[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        h[u] = __floats2half2_rn(__uint_as_float(r[m * 8 + 2 * u]) * down,
                                                 __uint_as_float(r[m * 8 + 2 * u + 1]) * down);
                    *reinterpret_cast<uint4 *>(bs + m * 128) = *reinterpret_cast<const uint4 *>(h);
                }
                fence_proxy_async();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_BSF + bsb));
                if (j == 0 && cl > 0 && !(ok = epilogue(cl - 1))) break;
            }
        }
        if (ok) ok = epilogue(p.nc - 1);
        if (ok && p.store_state) {
            for (int j = 0; j < p.MT && ok; ++j) {
                if (!(ok = W.wait(BAR(C::B_SD + j), (p.nc - 1) & 1))) break;
                tc_after();
#pragma unroll
                for (int c16 = 0; c16 < NV / 16; ++c16) tc_ld16(tmem + lane_off + j * NV + c16 * 16, r + c16 * 16);
                tc_wait_ld();
                const int64_t f = f0 + j * 128 + row;
                if (f < p.F) {
                    float4 *dS = reinterpret_cast<float4 *>(p.S + (bh * p.F + f) * DV);
#pragma unroll
                    for (int c4 = 0; c4 < DV / 4; ++c4)
                        dS[c4] = make_float4(__uint_as_float(r[4 * c4]), __uint_as_float(r[4 * c4 + 1]),
                                             __uint_as_float(r[4 * c4 + 2]), __uint_as_float(r[4 * c4 + 3]));
                    p.Z[bh * p.F + f] = __uint_as_float(r[DV]);
                }
            }
        }
        tc_before();
    } else if (warp >= kWarpGen0) {
        // ------------------------------------------------ feature generation
        const int gt = threadIdx.x - kWarpGen0 * 32;
        // alpha*C*phi(q/c) tiles into shared memory: thread = 8 tokens x 8 features
        const int tg = gt & 15;            // tokens 8*tg .. 8*tg+7
        const int fgrp = gt >> 4;          // features 8*fgrp .. 8*fgrp+7 of the tile
        const int xoff = tg * 16;
        const int hoff = (tg >> 3) * 16384;
        const int cidx = tg & 7;
        // phi(k) tiles into TMEM: lane = feature row of the tile, 32 tokens per warp
        const int kq = warp & 3;                           // TMEM lane quarter of this warp
        const int krow = kq * 32 + lane;
        const int ksub = (warp - kWarpGen0) >> 2;          // which 32 tokens of a 64-token stage
        const uint32_t k_lane_off = (uint32_t)(kq * 32) << 16;
        int qa = 0, qk = 0;
        bool ok = true;
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int ib = cl & 1;
            if (!(ok = W.wait(BAR(C::B_INF + ib), (cl >> 1) & 1))) break;
            const uint8_t *xq = smem + ib * C::IMG_PAD + C::OFF_IQ;
            const uint8_t *xk = smem + ib * C::IMG_PAD + C::OFF_IK;
            for (int j = 0; j < p.MT && ok; ++j) {
                {   // alpha*C*phi(q/c), shared memory, 128-byte swizzled [f][t]
                    const int sa = qa & 1;
                    if (!(ok = W.wait(BAR(C::B_QE + sa), ((qa >> 1) & 1) ^ 1))) break;
                    uint8_t *stage = smem + C::OFF_RING + sa * kStageBytes + hoff;
                    const uint4 *tj4 = reinterpret_cast<const uint4 *>(tab + j * 128 + fgrp * 8);
                    const uint4 t_lo = tj4[0], t_hi = tj4[1];
                    const uint32_t tw[8] = {t_lo.x, t_lo.y, t_lo.z, t_lo.w, t_hi.x, t_hi.y, t_hi.z, t_hi.w};
                    __align__(16) __half mj[8];
                    *reinterpret_cast<uint4 *>(mj) = *reinterpret_cast<const uint4 *>(mc + j * 128 + fgrp * 8);
                    uint32_t prev = 0xFFFFFFFFu;
                    uint4 pre = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t w = tw[i];
                        if ((w & 0xFFFFu) != prev) {   // new prefix pair (a, b)
                            prev = w & 0xFFFFu;
                            const uint4 xa = *reinterpret_cast<const uint4 *>(xq + (w & 255u) * C::ROW + xoff);
                            const uint4 xb = *reinterpret_cast<const uint4 *>(xq + ((w >> 8) & 255u) * C::ROW + xoff);
                            pre = hmul4(xa, xb);
                        }
                        const uint4 xl = *reinterpret_cast<const uint4 *>(xq + ((w >> 16) & 255u) * C::ROW + xoff);
                        const uint4 val = hmul4s(hmul4(pre, xl), __half2half2(mj[i]));
                        const int fr = fgrp * 8 + i;
                        *reinterpret_cast<uint4 *>(stage + fr * 128 + ((cidx ^ i) << 4)) = val;
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(BAR(C::B_QF + sa));
                    ++qa;
                }
                {   // phi(k), TMEM: this lane's feature over 32 tokens, per 64-token stage
                    const uint32_t w = tab[j * 128 + krow];
                    const uint8_t *ra = xk + (w & 255u) * C::KROW;
                    const uint8_t *rb = xk + ((w >> 8) & 255u) * C::KROW;
                    const uint8_t *rl = xk + ((w >> 16) & 255u) * C::KROW;
                    for (int h = 0; h < 2; ++h) {
                        const int sk = qk & 1;
                        if (!(ok = W.wait(BAR(C::B_KE + sk), ((qk >> 1) & 1) ^ 1))) break;
                        const int tb = (64 * h + 32 * ksub) * 2;   // byte offset of this warp's tokens
                        uint32_t rr[16];
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            const uint4 xa = *reinterpret_cast<const uint4 *>(ra + tb + g8 * 16);
                            const uint4 xb = *reinterpret_cast<const uint4 *>(rb + tb + g8 * 16);
                            const uint4 xl = *reinterpret_cast<const uint4 *>(rl + tb + g8 * 16);
                            const uint4 val = hmul4(hmul4(xa, xb), xl);
                            rr[4 * g8 + 0] = val.x;
                            rr[4 * g8 + 1] = val.y;
                            rr[4 * g8 + 2] = val.z;
                            rr[4 * g8 + 3] = val.w;
                        }
                        tc_st16(tmem + k_lane_off + C::COL_A + sk * 32 + 16 * ksub, rr);
                        tc_wait_st();
                        tc_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(C::B_KF + sk));
                        ++qk;
                    }
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_INE + ib));
        }
        tc_before();
    }

    __syncthreads();
    if (warp == kWarpProducer) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

// --------------------------------------------------------------- finish ----

// Sum the G feature-group partials of every (head, chunk, column, token):
// part [BH][G][nc][DV+1][128] -> red [BH][nc][DV+1][128].  A pure streaming
// kernel (float4, eight loads in flight per thread, fixed summation order).
template <int DV>
__global__ void __launch_bounds__(256)
tc_reduce_kernel(const float4 *__restrict__ part, float4 *__restrict__ red, int BH, int G, int nc) {
    const int64_t per_head = (int64_t)nc * (DV + 1) * (kL / 4);
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

// Per (head, chunk): sum the feature tiles' inter-chunk partials, add the
// intra-chunk block sum_{s<=t} w_ts [v_s | 1] (fp32 from the bf16 inputs) and
// divide.  Partial sums stream with float4 loads, several in flight per thread.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
tc_finish_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, const float *__restrict__ part,
                 float *__restrict__ out, int BH, int G, int c0, int nc, int64_t N, int P, float inv_c) {
    constexpr int VP = DV + 1, WP = kL + 1, HW = DV / 2;
    constexpr int ITEMS = VP * (kL / 4);            // float4 items of one chunk's partial
    constexpr int PER = (ITEMS + 255) / 256;
    extern __shared__ float fsm[];
    float *Ps = fsm;                 // [VP][128]  summed partials (col-major by token)
    float *fqT = Ps + VP * kL;       // [DK][128]  q^T  (later: staging [128][DV])
    float *fkT = fqT + DK * kL;      // [DK][128]  k^T  (later: v [128][DV])
    float *Wt = fkT + DK * kL;       // [128][WP]
    const int tid = threadIdx.x;
    const float4 *p4 = reinterpret_cast<const float4 *>(part);
    for (int64_t idx = blockIdx.x; idx < (int64_t)BH * nc; idx += gridDim.x) {
        const int64_t bh = idx / nc;
        const int cl = (int)(idx % nc);
        const int64_t t0 = (int64_t)(c0 + cl) * kL;
        const int nt = (int)(N - t0 < kL ? N - t0 : kL);
        // (1) sum over the G feature-tile groups
        {
            const int64_t gstride = (int64_t)nc * ITEMS;
            const int64_t base = ((int64_t)bh * G * nc + cl) * ITEMS;
            float4 acc[PER];
#pragma unroll
            for (int u = 0; u < PER; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int gg = 0; gg < G; ++gg) {
                const float4 *src = p4 + base + gg * gstride;
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    const int item = tid + u * 256;
                    if (item < ITEMS) {
                        const float4 x = src[item];
                        acc[u].x += x.x; acc[u].y += x.y; acc[u].z += x.z; acc[u].w += x.w;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int item = tid + u * 256;
                if (item < ITEMS) reinterpret_cast<float4 *>(Ps)[item] = acc[u];
            }
        }
        // (2) q^T, k^T in fp32
        for (int e = tid; e < kL * DK; e += 256) {
            const int t = e / DK, i = e % DK;
            float a = 0.f, b = 0.f;
            if (t < nt) {
                a = __bfloat162float(q[(bh * N + t0 + t) * DK + i]);
                b = __bfloat162float(k[(bh * N + t0 + t) * DK + i]);
            }
            fqT[i * kL + t] = a;
            fkT[i * kL + t] = b;
        }
        __syncthreads();
        // (3) W[t][s] = sum_{p<P} (q_t.k_s / c)^p / p! for s <= t, by 8x8 blocks
        {
            const int tb = tid / 16, sbk = tid % 16;
            float acc[8][8];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
            if (sbk <= tb) {
                for (int i = 0; i < DK; ++i) {
                    const float4 qa0 = *reinterpret_cast<const float4 *>(fqT + i * kL + tb * 8);
                    const float4 qa1 = *reinterpret_cast<const float4 *>(fqT + i * kL + tb * 8 + 4);
                    const float4 kb0 = *reinterpret_cast<const float4 *>(fkT + i * kL + sbk * 8);
                    const float4 kb1 = *reinterpret_cast<const float4 *>(fkT + i * kL + sbk * 8 + 4);
                    const float xa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
                    const float xb[8] = {kb0.x, kb0.y, kb0.z, kb0.w, kb1.x, kb1.y, kb1.z, kb1.w};
#pragma unroll
                    for (int a = 0; a < 8; ++a)
#pragma unroll
                        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(xa[a], xb[b], acc[a][b]);
                }
            }
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const int t = tb * 8 + a, s2 = sbk * 8 + b;
                    float w = 0.f;
                    if (s2 <= t && t < nt) {
                        const float x = acc[a][b] * inv_c;
                        float h = 1.f;   // Horner form of sum_{p<P} x^p / p!
                        for (int pp = P - 1; pp >= 1; --pp) h = fmaf(h, x / (float)pp, 1.f);
                        w = h;
                    }
                    Wt[t * WP + s2] = w;
                }
        }
        __syncthreads();
        // (4) v rows (fp32) over k^T's space
        float *fv = fkT;   // [128][DV]
        for (int e = tid; e < kL * DV; e += 256) {
            const int t = e / DV;
            fv[e] = t < nt ? __bfloat162float(v[(bh * N + t0) * DV + e]) : 0.f;
        }
        __syncthreads();
        // (5) out[t][j] = (partial num + sum_s W[t][s] v[s][j]) / (partial den + sum_s W[t][s])
        {
            const int t = tid % kL, h = tid / kL;
            float num[HW];
#pragma unroll
            for (int jj = 0; jj < HW; ++jj) num[jj] = Ps[(h * HW + jj) * kL + t];
            float den = Ps[DV * kL + t];
            for (int s2 = 0; s2 < kL; ++s2) {
                const float w = Wt[t * WP + s2];
                den += w;
                const float *vr = fv + s2 * DV + h * HW;
#pragma unroll
                for (int jj = 0; jj < HW; jj += 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(vr + jj);
                    num[jj] = fmaf(w, x.x, num[jj]);
                    num[jj + 1] = fmaf(w, x.y, num[jj + 1]);
                    num[jj + 2] = fmaf(w, x.z, num[jj + 2]);
                    num[jj + 3] = fmaf(w, x.w, num[jj + 3]);
                }
            }
            float *stage = fqT;   // [128][DV]
#pragma unroll
            for (int jj = 0; jj < HW; ++jj) stage[t * DV + h * HW + jj] = num[jj] / den;
        }
        __syncthreads();
        {
            const float4 *st4 = reinterpret_cast<const float4 *>(fqT);
            float4 *o4 = reinterpret_cast<float4 *>(out + (bh * N + t0) * DV);
            for (int e = tid; e < nt * DV / 4; e += 256) o4[e] = st4[e];
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ host ----

struct Plan {
    int MT = 1, G = 1, nchunks = 0, nc_seg = 0;
    size_t off_stats = 0, off_img = 0, off_part = 0, off_red = 0, off_state = 0, total = 0;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

template <int DK, int DV>
Plan make_plan(int BH, int64_t N, int64_t F, bool need_state) {
    using C = Cfg<DK, DV>;
    Plan pl;
    const int ftiles = (int)((F + 127) / 128);
    // feature tiles per CTA: as many as fit, unless that leaves fewer than two
    // CTAs per SM of work
    int mt = C::MT_MAX;
    while (mt > 1 && (int64_t)BH * ((ftiles + mt - 1) / mt) < 2 * 148) --mt;
    pl.G = (ftiles + mt - 1) / mt;
    pl.MT = (ftiles + pl.G - 1) / pl.G;
    pl.nchunks = (int)((N + kL - 1) / kL);
    const size_t per_chunk = (size_t)BH * pl.G * (DV + 1) * kL * sizeof(float);
    int64_t seg = (int64_t)(kPartialBudget / per_chunk);
    if (seg < 1) seg = 1;
    pl.nc_seg = (int)(seg < pl.nchunks ? seg : pl.nchunks);
    pl.off_stats = 0;
    pl.off_img = align256((size_t)BH * 4 * sizeof(float));
    pl.off_part = pl.off_img + align256((size_t)BH * pl.nchunks * C::IMG);
    pl.off_red = pl.off_part + align256(per_chunk * pl.nc_seg);
    pl.off_state = pl.off_red + align256((size_t)BH * (DV + 1) * kL * sizeof(float) * pl.nc_seg);
    pl.total = pl.off_state + (need_state ? align256((size_t)BH * F * (DV + 1) * sizeof(float)) : 0);
    return pl;
}

template <int DK, int DV>
cudaError_t run(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k, const void *v,
                float *out, float *S, float *Z, bool state_in, void *ws, size_t ws_bytes, int *flags,
                cudaStream_t stream) {
    using C = Cfg<DK, DV>;
    const int64_t F = basis.F;
    const bool own_state = (S == nullptr);
    const Plan pl = make_plan<DK, DV>(BH, N, F, true);
    if (ws_bytes < make_plan<DK, DV>(BH, N, F, own_state).total) return cudaErrorInvalidValue;
    uint8_t *w = (uint8_t *)ws;
    float *stats = (float *)(w + pl.off_stats);
    uint8_t *img = w + pl.off_img;
    float *part = (float *)(w + pl.off_part);
    const int nseg = (pl.nchunks + pl.nc_seg - 1) / pl.nc_seg;
    if (own_state && nseg > 1) {
        S = (float *)(w + pl.off_state);
        Z = S + (size_t)BH * F * DV;
    }
    const float inv_c = 1.0f / sqrtf((float)DK);
    const auto *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k, *vb = (const __nv_bfloat16 *)v;

    cudaError_t e = cudaMemsetAsync(stats, 0, (size_t)BH * 4 * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const size_t prep_smem = sizeof(__half) * kL * (2 * (DK + 2) + (DV + 2));
    e = cudaFuncSetAttribute(tc_prep_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (e != cudaSuccess) return e;
    const int64_t nwork = (int64_t)BH * pl.nchunks;
    const int prep_grid = (int)(nwork < 148 * 8 ? nwork : 148 * 8);
    launch_begin(kTcPrep, stream);
    tc_prep_kernel<DK, DV><<<prep_grid, 256, prep_smem, stream>>>(qb, kb, vb, img, stats, BH, N, pl.nchunks, inv_c);
    launch_end(kTcPrep, stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (state_in) {
        tc_state_stats_kernel<<<dim3(BH, 8), 256, 0, stream>>>(S, Z, stats, F, DV);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(tc_scan_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const size_t fin_smem = sizeof(float) * ((size_t)(DV + 1) * kL + (size_t)2 * DK * kL + (size_t)kL * (kL + 1));
    e = cudaFuncSetAttribute(tc_finish_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fin_smem);
    if (e != cudaSuccess) return e;
    int stall = -1;
    if (g_opt_test_stall) {
        stall = pl.nchunks > 1 ? 1 : 0;
        g_opt_test_stall = 0;
    }
    const int64_t wait_ns = g_opt_wait_limit > 0 ? g_opt_wait_limit : kDefaultWaitNs;
    for (int s = 0; s < nseg; ++s) {
        ScanParams sp;
        sp.img = img;
        sp.stats = stats;
        sp.packed = basis.packed;
        sp.mcoef = basis.mcoef;
        sp.S = S;
        sp.Z = Z;
        sp.part = part;
        sp.flags = flags;
        sp.F = F;
        sp.N = N;
        sp.BH = BH;
        sp.G = pl.G;
        sp.MT = pl.MT;
        sp.c0 = s * pl.nc_seg;
        sp.nc = (pl.nchunks - sp.c0 < pl.nc_seg) ? pl.nchunks - sp.c0 : pl.nc_seg;
        sp.nchunks = pl.nchunks;
        sp.P = basis.P;
        sp.load_state = (s > 0 || state_in) ? 1 : 0;
        sp.store_state = (s + 1 < nseg || !own_state) ? 1 : 0;
        sp.stall_chunk = stall;
        sp.inv_c = inv_c;
        sp.wait_ns = wait_ns;
        launch_begin(kTcScan, stream);
        tc_scan_kernel<DK, DV><<<BH * pl.G, kScanThreads, C::SMEM, stream>>>(sp);
        launch_end(kTcScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        float *red = (float *)(w + pl.off_red);
        const int64_t rwork = (int64_t)BH * sp.nc * (DV + 1) * (kL / 4);
        launch_begin(kTcReduce, stream);
        tc_reduce_kernel<DV><<<(int)((rwork + 255) / 256 < 148 * 32 ? (rwork + 255) / 256 : 148 * 32), 256, 0, stream>>>(
            (const float4 *)part, (float4 *)red, BH, pl.G, sp.nc);
        launch_end(kTcReduce, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t fwork = (int64_t)BH * sp.nc;
        launch_begin(kTcFinish, stream);
        tc_finish_kernel<DK, DV><<<(int)(fwork < 148 * 16 ? fwork : 148 * 16), 256, fin_smem, stream>>>(
            qb, kb, vb, red, out, BH, 1, sp.c0, sp.nc, N, basis.P, inv_c);
        launch_end(kTcFinish, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

bool prefill_tc_supported(int d_K, int d_V, int P) {
    return d_K == d_V && (d_K == 16 || d_K == 32 || d_K == 64) && P >= 1 && P <= 4;
}

size_t prefill_tc_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, bool need_state) {
    switch (d_K * 1000 + d_V) {
        case 16016: return make_plan<16, 16>(BH, N, F, need_state).total;
        case 32032: return make_plan<32, 32>(BH, N, F, need_state).total;
        case 64064: return make_plan<64, 64>(BH, N, F, need_state).total;
        default: return 0;
    }
}

cudaError_t launch_prefill_tc(const DeviceBasis &basis, int BH, int64_t N, int d_V, const void *q,
                              const void *k, const void *v, float *out, float *S, float *Z, bool state_in,
                              void *ws, size_t ws_bytes, int *flags, cudaStream_t stream) {
    switch (basis.d_K * 1000 + d_V) {
        case 16016: return run<16, 16>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream);
        case 32032: return run<32, 32>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream);
        case 64064: return run<64, 64>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace sata
