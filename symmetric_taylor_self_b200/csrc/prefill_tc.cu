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

#include <algorithm>
#include <utility>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kL = 128;               // chunk length (tokens)
constexpr int kScanThreads = 480;     // 15 warps
// warp roles: chunk-image producer, readout MMA issuer, state conversion (4), q side (4),
// k side (4), update MMA issuer
constexpr int kWarpProducer = 0, kWarpMmaRd = 1, kWarpConv0 = 2, kWarpQ0 = 6, kWarpK0 = 10, kWarpMmaUp = 14;
constexpr int kKStages = 3;           // ring of (P2k . x_l) operand stages, 32 tokens each
constexpr int64_t kDefaultWaitNs = 2000000000LL;   // 2 s per wait
constexpr size_t kPartialBudget = size_t(4) << 30;

// Feature organisation.  With x~ = (x, 1) (index D is the constant 1), the P=4
// basis is exactly the nondecreasing triples (a <= b <= l) over 0..D: F =
// binom(D+3, 3).  State rows are grouped by their pair (a, b) and their last
// index l: a CTA ("unit") owns one tile of 128 pairs (pairs sorted by b, then a)
// and up to MT values of l.  With P2(x) = x~_a x~_b per pair:
//   update:  [S|Z]_(pairs, l) += (P2(k) (.) k~_l)^T [V|1]
//   readout: R += (P2(q) (.) q~_l) . (C/p! * [S|Z]_(pairs, l)),   summed over the unit's l
// Both feature operands live in TMEM: the pair products are formed once per chunk
// in registers (one pair row, resp. one token row, per thread) and only scaled by
// the l column before each store, so no feature tile passes through shared memory.
template <int DK, int DV>
struct Cfg {
    static_assert(DK == DV, "square heads");
    static constexpr int D = DK;
    static constexpr int NV = DV + 16;                           // MMA N: [V | 1 | 0 pad]
    // TMEM: MT state tiles (NV columns each), R (NV), q-side operand (64), k-side ring
    static constexpr int MT_MAX = (512 - NV - 64 - 16 * kKStages) / NV;
    static constexpr int ROW = kL * 2;                           // 128 fp16
    static constexpr int KROW = ROW + 16;                        // k^T rows padded so that 32 lanes
                                                                 // reading 32 rows hit distinct banks
    static constexpr int QS = (D + 1 + 7) / 8 * 8;               // token-major q~ row: D+1 fp16, padded
    static constexpr int IMG_V = NV * ROW;                       // [V|1]^T, K-major SW128
    static constexpr int OFF_IQ = IMG_V;                         // q~ = (q/c, 1) token-major [128][QS]
    static constexpr int OFF_IK = IMG_V + kL * QS * 2;           // k~^T = (k, 1)^T [D+1][KROW]
    static constexpr int IMG = OFF_IK + (D + 1) * KROW;
    static constexpr int IMG_PAD = (IMG + 1023) / 1024 * 1024;
    static constexpr int OFF_BS = 2 * IMG_PAD;                   // two fp16 state operands
    static constexpr int BS_BYTES = 128 * NV * 2;
    static constexpr int OFF_PAIR = OFF_BS + 2 * BS_BYTES;       // uint16 [128]
    static constexpr int OFF_COEF = OFF_PAIR + 256;              // float [MT_MAX][128]
    static constexpr int OFF_LV = OFF_COEF + MT_MAX * 128 * 4;   // int [MT_MAX]
    static constexpr int OFF_BAR = OFF_LV + 64;
    // barrier indices
    static constexpr int B_INF = 0, B_INE = 2, B_AQF = 4, B_AQE = 5, B_BSF = 6, B_BSE = 8, B_RE = 10,
                         B_FIN = 11, B_KF = 12, B_KE = B_KF + kKStages, B_SD = B_KE + kKStages,
                         B_SR = B_SD + MT_MAX, N_BAR = B_SR + MT_MAX;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;            // + base alignment slack
    static constexpr int COL_R = MT_MAX * NV;                    // TMEM: readout accumulator
    static constexpr int COL_AQ = COL_R + NV;                    // TMEM: P2(q) (.) q~_l, 64 columns
    static constexpr int COL_AK = COL_AQ + 64;                   // TMEM: (P2(k) (.) k~_l) ring
    static constexpr int LBO_BS = (NV / 8) * 128;
    static_assert(MT_MAX >= 1 && MT_MAX <= 16, "unit l table");
    static_assert(COL_AK + 16 * kKStages <= 512, "TMEM columns");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(NV % 16 == 0, "MMA N");
};

struct ScanParams {
    const uint8_t *img;         // [BH][nchunks][IMG]
    const float *stats;         // [BH][4] max|q|, max|k|, max|v|, max|state|
    const uint16_t *pairs;      // [NPT][128]  a | b << 8
    const int32_t *unit_k;      // [G] pair tile of each unit
    const int32_t *unit_nl;     // [G] number of l values
    const int32_t *unit_l;      // [G][MT_MAX]
    const float *unit_coef;     // [G][MT_MAX][128] C/p! of feature (pair, l), 0 if none
    const int32_t *unit_fidx;   // [G][MT_MAX][128] basis index of feature (pair, l), -1 if none
    float *S, *Z;               // state in/out
    float *part;                // [BH][G][nc][DV+1][128], or with red_atomic the sums [BH][nc][DV+1][128]
    int red_atomic;             // 1: add R into the sums in L2 (fp32 atomics); 0: one partial per unit
    int *flags;
    int64_t F, N;
    int BH, G, c0, nc, nchunks, P;
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

// Packed fp16 products on 32-bit registers (round to nearest).
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// Pair (a, b), a <= b <= D, sorted by b then a: index b (b + 1) / 2 + a; indices
// past the last pair stand for (D, D).  The host plan uses the same order.
template <int D>
struct Pairs {
    static constexpr int N = (D + 1) * (D + 2) / 2;
    static constexpr int NT = (N + 127) / 128;
    __host__ __device__ static constexpr int b(int idx) {
        if (idx >= N) return D;
        int v = 0;
        while ((v + 1) * (v + 2) / 2 <= idx) ++v;
        return v;
    }
    __host__ __device__ static constexpr int a(int idx) { return idx >= N ? D : idx - b(idx) * (b(idx) + 1) / 2; }
};

// Two fp16 values x~_i0, x~_i1 (indices into a token row held as packed half2
// registers) as one half2, i0 in the low half.
template <int I0, int I1, int NX>
__device__ __forceinline__ uint32_t pick2(const uint32_t (&x)[NX]) {
    if constexpr (I0 % 2 == 0 && I1 == I0 + 1) {
        return x[I0 / 2];
    } else {
        constexpr uint32_t s0 = (I0 % 2) * 2, s2 = 4 + (I1 % 2) * 2;
        return __byte_perm(x[I0 / 2], x[I1 / 2], s0 | ((s0 + 1) << 4) | (s2 << 8) | ((s2 + 1) << 12));
    }
}
// P2(q) of one token for pair tile K: pq[m] = (x~_a x~_b) of pairs 2m, 2m+1.
template <int D, int K, int NX, int... M>
__device__ __forceinline__ void p2q_tile(const uint32_t (&x)[NX], uint32_t (&pq)[64], std::integer_sequence<int, M...>) {
    using PT = Pairs<D>;
    ((pq[M] = hmul2u(pick2<PT::a(K * 128 + 2 * M), PT::a(K * 128 + 2 * M + 1)>(x),
                     pick2<PT::b(K * 128 + 2 * M), PT::b(K * 128 + 2 * M + 1)>(x))),
     ...);
}
template <int D, int NX, int... K>
__device__ __forceinline__ void p2q_dispatch(int k, const uint32_t (&x)[NX], uint32_t (&pq)[64],
                                             std::integer_sequence<int, K...>) {
    ((k == K ? (p2q_tile<D, K>(x, pq, std::make_integer_sequence<int, 64>{}), 0) : 0), ...);
}

// ----------------------------------------------------------------- prep ----

// Per (head, chunk): write the chunk image [ [V|1]^T (K-major, 128-byte swizzle)
// | (q/c)^T | k^T (rows padded to 272 bytes) ], fp16, padded tokens zero
// (including their 1 entries), and raise the per-head maxima of |q|, |k|, |v|.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               const __nv_bfloat16 *__restrict__ v, uint8_t *__restrict__ img,
               float *__restrict__ stats, int BH, int64_t N, int nchunks, int cbeg, int ccount, float inv_c) {
    using C = Cfg<DK, DV>;
    constexpr int PK = DK + 2, PV = DV + 2;
    extern __shared__ __half psm[];
    __half *sk = psm;                 // [128][PK]
    __half *sq = sk + kL * PK;        // [128][PK]
    __half *sv = sq + kL * PK;        // [128][PV]
    __shared__ float red[3][8];
    const int tid = threadIdx.x;
    const __half one = __float2half(1.f), zero = __float2half(0.f);
    for (int64_t idx = blockIdx.x; idx < (int64_t)BH * ccount; idx += gridDim.x) {
        const int64_t bh = idx / ccount;
        const int c = cbeg + (int)(idx % ccount);
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
        uint8_t *out = img + (bh * nchunks + c) * (int64_t)C::IMG;
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
        // k~^T: row i holds tokens 0..127; row DK is 1 (0 for padded tokens)
        for (int e = tid; e < (DK + 1) * 16; e += 256) {
            const int i = e / 16, t8 = e % 16;
            __align__(16) __half hk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int t = t8 * 8 + j;
                hk[j] = i < DK ? sk[t * PK + i] : (t < nt ? one : zero);
            }
            *reinterpret_cast<uint4 *>(out + C::OFF_IK + i * C::KROW + t8 * 16) = *reinterpret_cast<const uint4 *>(hk);
        }
        // q~ token-major: row t holds (q_t / c, 1) then zeros (all zero for padded tokens)
        for (int e = tid; e < kL * (C::QS / 8); e += 256) {
            const int t = e / (C::QS / 8), i8 = (e % (C::QS / 8)) * 8;
            __align__(16) __half hq[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i8 + j;
                hq[j] = i < DK ? sq[t * PK + i] : ((i == DK && t < nt) ? one : zero);
            }
            *reinterpret_cast<uint4 *>(out + C::OFF_IQ + (t * C::QS + i8) * 2) = *reinterpret_cast<const uint4 *>(hq);
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
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto BAR = [bar0](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    uint16_t *sp_pair = reinterpret_cast<uint16_t *>(smem + C::OFF_PAIR);
    float *sp_coef = reinterpret_cast<float *>(smem + C::OFF_COEF);
    int *sp_l = reinterpret_cast<int *>(smem + C::OFF_LV);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // unit-major order: every head's largest units are scheduled first
    const int64_t bh = blockIdx.x % p.BH;
    const int u = blockIdx.x / p.BH;
    const int ktile = p.unit_k[u];
    const int nl = p.unit_nl[u];
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
            if (i == C::B_INE || i == C::B_INE + 1) cnt = 1 + 4 + 4;   // MMA commit, q-side, k-side warps
            else if (i == C::B_AQF || i == C::B_RE || i == C::B_BSF || i == C::B_BSF + 1) cnt = 4;
            else if (i >= C::B_KF && i < C::B_KF + kKStages) cnt = 4;
            else if (i >= C::B_SR && i < C::B_SR + C::MT_MAX) cnt = 4;
            else if (i == C::B_FIN) cnt = 2;                             // both MMA issuers
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
    for (int i = threadIdx.x; i < 128; i += blockDim.x) sp_pair[i] = p.pairs[ktile * 128 + i];
    for (int i = threadIdx.x; i < C::MT_MAX * 128; i += blockDim.x)
        sp_coef[i] = p.unit_coef[(int64_t)u * C::MT_MAX * 128 + i];
    for (int i = threadIdx.x; i < C::MT_MAX; i += blockDim.x) sp_l[i] = p.unit_l[u * C::MT_MAX + i];
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
    } else if (warp == kWarpMmaRd) {
        // ------------------------------------------------ readout MMA issue (one thread)
        if (lane == 0) {
            constexpr uint32_t id_rd = idesc_f16(128, NV, 0, 1);    // A TMEM, B MN-major
            int qa = 0;
            bool ok = true;
            for (int cl = 0; cl < p.nc && ok; ++cl) {
                for (int j = 0; j < nl; ++j) {
                    const int bsb = qa & 1;
                    ok = W.wait(BAR(C::B_BSF + bsb), (qa >> 1) & 1) && W.wait(BAR(C::B_AQF), qa & 1);
                    if (ok && j == 0 && cl > 0) ok = W.wait(BAR(C::B_RE), (cl - 1) & 1);   // R of cl-1 read
                    if (!ok) break;
                    tc_after();
                    // R (+)= (P2(q) (.) q~_lj) [128 t x 128 pairs] . (C/p! 2^-s [S|Z])_(pairs, lj) [128 pairs x NV]
                    const uint32_t b_s = sb + C::OFF_BS + bsb * C::BS_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc_mma_ta(tmem + C::COL_R, tmem + C::COL_AQ + ks * 8,
                                  sdesc(b_s + ks * 2 * C::LBO_BS, C::LBO_BS, 128, 0), id_rd,
                                  (j > 0 || ks > 0) ? 1u : 0u);
                    tc_commit(BAR(C::B_BSE + bsb));
                    tc_commit(BAR(C::B_AQE));
                    ++qa;
                }
            }
            // every issued MMA completes before TMEM is released
            tc_commit(BAR(C::B_FIN));
            W.drain(BAR(C::B_FIN), 0);
        }
    } else if (warp == kWarpMmaUp) {
        // ------------------------------------------------ update MMA issue (one thread)
        if (lane == 0) {
            constexpr uint32_t id_upd = idesc_f16(128, NV, 0, 0);   // A TMEM, B K-major
            int st = 0, sph = 0;                                    // k-side ring stage and its phase
            bool ok = true;
            for (int cl = 0; cl < p.nc && ok; ++cl) {
                const int ib = cl & 1;
                if (!(ok = W.wait(BAR(C::B_INF + ib), (cl >> 1) & 1))) break;
                const uint32_t vimg = sb + ib * C::IMG_PAD;
                // [S|Z]_(pairs, lj) += (P2(k) (.) k~_lj) [128 pairs x 32 t] . [V|1] [32 t x NV], by token
                // quarter qq; tile j is final for this chunk after its last quarter
                for (int h = 0; h < 2 && ok; ++h) {
                    for (int j = 0; j < nl && ok; ++j) {
                        // the state conversion has read tile j before it changes
                        if (h == 0 && !(ok = W.wait(BAR(C::B_SR + j), cl & 1))) break;
                        for (int qh = 0; qh < 2; ++qh) {
                            const int qq = 2 * h + qh;
                            if (!(ok = W.wait(BAR(C::B_KF + st), sph))) break;
                            tc_after();
                            tc_mma_ta(tmem + j * NV, tmem + C::COL_AK + st * 16,
                                      sdesc(vimg + h * (NV * 128) + qh * 64, 16, 1024, 2), id_upd, 1u);
                            tc_mma_ta(tmem + j * NV, tmem + C::COL_AK + st * 16 + 8,
                                      sdesc(vimg + h * (NV * 128) + qh * 64 + 32, 16, 1024, 2), id_upd, 1u);
                            tc_commit(BAR(C::B_KE + st));
                            (void)qq;
                            if (++st == kKStages) {
                                st = 0;
                                sph ^= 1;
                            }
                        }
                        if (ok && h == 1) tc_commit(BAR(C::B_SD + j));
                    }
                }
                if (!ok) break;
                tc_commit(BAR(C::B_INE + ib));
            }
            tc_commit(BAR(C::B_FIN));
            W.drain(BAR(C::B_FIN), 0);
        }
    } else if (warp >= kWarpConv0 && warp < kWarpQ0) {
        // ------------------------------------------------ state -> fp16 readout operand
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;            // pair row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint32_t r[NV];
        // initial state -> TMEM (zeros for a fresh sequence)
        for (int j = 0; j < nl; ++j) {
            const int f = p.unit_fidx[((int64_t)u * C::MT_MAX + j) * 128 + row];
            const bool have = p.load_state && f >= 0;
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
        bool ok = true;
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const float down = pow2f(-state_sigma(p.c0 + cl, mk, mv, ms, p.P));
            for (int j = 0; j < nl; ++j) {
                const int qn = cl * nl + j, bsb = qn & 1;
                if (cl > 0 && !(ok = W.wait(BAR(C::B_SD + j), (cl - 1) & 1))) break;
                tc_after();
#pragma unroll
                for (int c16 = 0; c16 < NV / 16; ++c16) tc_ld16(tmem + lane_off + j * NV + c16 * 16, r + c16 * 16);
                tc_wait_ld();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_SR + j));   // tile j read: the update may proceed
                if (!(ok = W.wait(BAR(C::B_BSE + bsb), ((qn >> 1) & 1) ^ 1))) break;
                const float cf = sp_coef[j * 128 + row] * down;
                uint8_t *bs = smem + C::OFF_BS + bsb * C::BS_BYTES + (row / 8) * C::LBO_BS + (row % 8) * 16;
#pragma unroll
                for (int m = 0; m < NV / 8; ++m) {
                    __align__(16) __half2 h[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        h[w] = __floats2half2_rn(__uint_as_float(r[m * 8 + 2 * w]) * cf,
                                                 __uint_as_float(r[m * 8 + 2 * w + 1]) * cf);
                    *reinterpret_cast<uint4 *>(bs + m * 128) = *reinterpret_cast<const uint4 *>(h);
                }
                fence_proxy_async();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_BSF + bsb));
            }
        }
        if (ok && p.store_state) {
            for (int j = 0; j < nl && ok; ++j) {
                if (!(ok = W.wait(BAR(C::B_SD + j), (p.nc - 1) & 1))) break;
                tc_after();
#pragma unroll
                for (int c16 = 0; c16 < NV / 16; ++c16) tc_ld16(tmem + lane_off + j * NV + c16 * 16, r + c16 * 16);
                tc_wait_ld();
                const int f = p.unit_fidx[((int64_t)u * C::MT_MAX + j) * 128 + row];
                if (f >= 0) {
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
    } else if (warp >= kWarpQ0 && warp < kWarpK0) {
        // ------------------------------------------------ q side: operand per l, partial per chunk
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;               // token row of the chunk = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        // one partial row block per (unit, chunk), or the head's shared sums (added in L2)
        const int64_t part_base = p.red_atomic ? (int64_t)bh * p.nc : ((int64_t)bh * p.G + u) * p.nc;
        int qa = 0;
        bool ok = true;
        // R of chunk cl -> partial (x 2^sigma_cl); the caller has seen the completion of the
        // chunk's last readout
        auto drain = [&](int cl) -> bool {
            tc_after();
            const float up = pow2f(state_sigma(p.c0 + cl, mk, mv, ms, p.P));
            float *dst = p.part + ((part_base + cl) * (DV + 1)) * kL + t;
#pragma unroll
            for (int c16 = 0; c16 * 16 <= D; ++c16) {
                uint32_t rr[16];
                tc_ld16(tmem + lane_off + C::COL_R + c16 * 16, rr);
                tc_wait_ld();
                if (p.red_atomic) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c16 * 16 + i <= D) atomicAdd(dst + (c16 * 16 + i) * kL, __uint_as_float(rr[i]) * up);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c16 * 16 + i <= D) dst[(c16 * 16 + i) * kL] = __uint_as_float(rr[i]) * up;
                }
            }
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_RE));
            return true;
        };
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int ib = cl & 1;
            if (!(ok = W.wait(BAR(C::B_INF + ib), (cl >> 1) & 1))) break;
            const __half *xq = reinterpret_cast<const __half *>(smem + ib * C::IMG_PAD + C::OFF_IQ) + t * C::QS;
            // P2(q) of this token for the tile's 128 pairs (even pair in the low half), from
            // the token's q~ row in registers; pair indices are compile-time per tile
            uint32_t pq[64];
            {
                uint32_t x[C::QS / 2];
#pragma unroll
                for (int i = 0; i < C::QS / 8; ++i) {
                    const uint4 v = reinterpret_cast<const uint4 *>(xq)[i];
                    x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
                }
                p2q_dispatch<D>(ktile, x, pq, std::make_integer_sequence<int, Pairs<D>::NT>{});
            }
            for (int j = 0; j < nl; ++j) {
                const __half2 ql2 = __half2half2(xq[sp_l[j]]);   // q~_l of this token
                uint32_t qlb = *reinterpret_cast<const uint32_t *>(&ql2);
                if (!(ok = W.wait(BAR(C::B_AQE), (qa & 1) ^ 1))) break;
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    // keeps each group's products behind the previous group's store
                    asm volatile("" : "+r"(qlb));
                    uint32_t o[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = hmul2u(pq[c16 * 16 + i], qlb);
                    tc_st16(tmem + lane_off + C::COL_AQ + c16 * 16, o);
                }
                tc_wait_st();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_AQF));
                ++qa;
                // R of the previous chunk is complete once this chunk's first operand is out
                if (j == 0 && cl > 0 && !(ok = drain(cl - 1))) break;
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_INE + ib));
        }
        if (ok && p.nc > 0 && W.wait(BAR(C::B_AQE), (qa & 1) ^ 1)) drain(p.nc - 1);
        tc_before();
    } else if (warp >= kWarpK0) {
        // ------------------------------------------------ k side: (P2(k) (.) k~_l) stages
        const int kq = warp & 3;
        const int prow = kq * 32 + lane;                  // pair row of the tile = TMEM lane
        const uint32_t k_lane_off = (uint32_t)(kq * 32) << 16;
        const uint32_t pw = sp_pair[prow];
        const int pa = pw & 255, pb = pw >> 8;
        int qk = 0;
        bool ok = true;
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int ib = cl & 1;
            if (!(ok = W.wait(BAR(C::B_INF + ib), (cl >> 1) & 1))) break;
            const uint8_t *xk = smem + ib * C::IMG_PAD + C::OFF_IK;
            for (int h = 0; h < 2 && ok; ++h) {
                uint32_t pk[32];   // P2(k) of this pair over tokens 64h .. 64h+63
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint4 xa = *reinterpret_cast<const uint4 *>(xk + pa * C::KROW + (8 * h + g) * 16);
                    const uint4 xb = *reinterpret_cast<const uint4 *>(xk + pb * C::KROW + (8 * h + g) * 16);
                    pk[4 * g] = hmul2u(xa.x, xb.x);
                    pk[4 * g + 1] = hmul2u(xa.y, xb.y);
                    pk[4 * g + 2] = hmul2u(xa.z, xb.z);
                    pk[4 * g + 3] = hmul2u(xa.w, xb.w);
                }
                for (int j = 0; j < nl && ok; ++j) {
                    const uint8_t *xl = xk + sp_l[j] * C::KROW + h * 128;
#pragma unroll
                    for (int qh = 0; qh < 2; ++qh) {
                        const int st = qk % kKStages;
                        if (!(ok = W.wait(BAR(C::B_KE + st), ((qk / kKStages) & 1) ^ 1))) break;
                        uint32_t o[16];
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int gg = 4 * qh + g;                     // 8-token group of the half
                            const uint4 x4 = *reinterpret_cast<const uint4 *>(xl + gg * 16);
                            o[4 * g] = hmul2u(pk[4 * gg], x4.x);
                            o[4 * g + 1] = hmul2u(pk[4 * gg + 1], x4.y);
                            o[4 * g + 2] = hmul2u(pk[4 * gg + 2], x4.z);
                            o[4 * g + 3] = hmul2u(pk[4 * gg + 3], x4.w);
                        }
                        tc_st16(tmem + k_lane_off + C::COL_AK + st * 16, o);
                        tc_wait_st();
                        tc_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(C::B_KF + st));
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

// Per (head, chunk): the intra-chunk block on tensor cores, plus the division.
//   S = Q K^T          fp16 operands (the bf16 inputs, exactly), fp32 accumulate in TMEM
//   W[t][s] = sum_{p<P} (S_ts / c)^p / p!  for s <= t, row t scaled by 2^-e_t, split into two
//                      fp16 parts W_hi + W_lo (about 22 significant bits: the polynomial's terms can
//                      cancel, so one fp16 rounding of W is not accurate enough)
//   O = W_hi [V|1] + W_lo [V|1]   TMEM
//   out[t] = (2^e_t O_num + num_t) / (2^e_t O_den + den_t), num/den the summed inter-chunk partials
// One CTA (4 warps, thread = token row) per (head, chunk).
template <int DK, int DV>
struct FinCfg {
    static constexpr int NV = DV + 16;
    static constexpr int OFF_Q = 0;                // [128 t][64 d] K-major SW128 (d >= DK zero)
    static constexpr int OFF_K = 16384;            // [128 s][64 d] K-major SW128
    static constexpr int OFF_W = 32768;            // W_hi [128 t][128 s] K-major SW128, two 64-wide K blocks
    static constexpr int OFF_WLO = 0;              // W_lo, same layout, over Q and K once S is done
    static constexpr int OFF_V = 65536;            // [128 s][NV n] MN-major, no swizzle
    static constexpr int LBO_V = (NV / 8) * 128;
    static constexpr int OFF_BAR = OFF_V + 128 * NV * 2;
    static constexpr int SMEM = OFF_BAR + 64 + 1024;
    static constexpr int STG = DV + 4;             // staging row stride (floats), over Q, K, W
    static_assert(128 * STG * 4 <= OFF_V, "staging");
    static_assert(DK <= 64, "head size");
};

template <int DK, int DV>
__global__ void __launch_bounds__(128)
tc_finish_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, const float *__restrict__ red, float *__restrict__ out,
                 float *__restrict__ den_out, int c0, int nc, int64_t N, int P, float inv_c, int *flags,
                 int64_t wait_ns) {
    using F = FinCfg<DK, DV>;
    constexpr int NV = F::NV;
    extern __shared__ uint8_t fraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(fraw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const uint32_t bar = sb + F::OFF_BAR;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sm + F::OFF_BAR + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + F::OFF_BAR + 20);
    const int tid = threadIdx.x, warp = tid / 32;
    const int64_t bh = blockIdx.x / nc;
    const int cl = blockIdx.x % nc;
    const int64_t t0 = (int64_t)(c0 + cl) * kL;
    const int nt = (int)(N - t0 < kL ? N - t0 : kL);
    if (tid == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)),
                     "r"(256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // ---- operands: bf16 -> fp16 (exact for the accepted input range), swizzled
    const __half one = __float2half(1.f);
    for (int e = tid; e < kL * 8; e += 128) {      // Q and K: 8 chunks of 8 d per row
        const int r = e / 8, c = e % 8;
        uint4 hq = make_uint4(0, 0, 0, 0), hk = make_uint4(0, 0, 0, 0);
        if (r < nt && c < DK / 8) {
            const uint4 bq = *reinterpret_cast<const uint4 *>(q + (bh * N + t0 + r) * DK + c * 8);
            const uint4 bk = *reinterpret_cast<const uint4 *>(k + (bh * N + t0 + r) * DK + c * 8);
            const __nv_bfloat16 *pq = reinterpret_cast<const __nv_bfloat16 *>(&bq);
            const __nv_bfloat16 *pk = reinterpret_cast<const __nv_bfloat16 *>(&bk);
            __half *oq = reinterpret_cast<__half *>(&hq), *ok2 = reinterpret_cast<__half *>(&hk);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                oq[i] = __float2half_rn(__bfloat162float(pq[i]));
                ok2[i] = __float2half_rn(__bfloat162float(pk[i]));
            }
        }
        const int off = r * 128 + ((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(sm + F::OFF_Q + off) = hq;
        *reinterpret_cast<uint4 *>(sm + F::OFF_K + off) = hk;
    }
    for (int e = tid; e < kL * (NV / 8); e += 128) {   // [V|1]: row s, 8 n per 16-byte core row
        const int r = e / (NV / 8), c = e % (NV / 8);
        uint4 hv = make_uint4(0, 0, 0, 0);
        __half *ov = reinterpret_cast<__half *>(&hv);
        if (r < nt) {
            if (c < DV / 8) {
                const uint4 bv = *reinterpret_cast<const uint4 *>(v + (bh * N + t0 + r) * DV + c * 8);
                const __nv_bfloat16 *pv = reinterpret_cast<const __nv_bfloat16 *>(&bv);
#pragma unroll
                for (int i = 0; i < 8; ++i) ov[i] = __float2half_rn(__bfloat162float(pv[i]));
            } else if (c == DV / 8) {
                ov[0] = one;
            }
        }
        *reinterpret_cast<uint4 *>(sm + F::OFF_V + (r / 8) * F::LBO_V + c * 128 + (r % 8) * 16) = hv;
    }
    fence_proxy_async();
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter W{abort_flag, flags + kFlagTimeout, wait_ns};
    // ---- S = Q K^T  [128 t x 128 s], K = 64
    if (tid == 0) {
        constexpr uint32_t id_s = idesc_f16(128, 128, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            tc_mma(tmem, sdesc(sb + F::OFF_Q + ks * 32, 16, 1024, 2), sdesc(sb + F::OFF_K + ks * 32, 16, 1024, 2),
                   id_s, ks > 0 ? 1u : 0u);
        tc_commit(bar);
    }
    __syncwarp();
    bool ok = W.wait(bar, 0);
    tc_after();
    const int t = tid;                               // token row = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // ---- W row t: polynomial, causal mask, power-of-two scale into the fp16 range
    // Horner form of sum_{p<P} x^p / p!, x = sv / c: h <- 1 + h * sv * (1 / (c p)), P <= 4
    const float cp1 = inv_c, cp2 = inv_c * 0.5f, cp3 = inv_c * (1.f / 3.f);
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
        for (int c16 = 0; c16 < 8; ++c16) {
            uint32_t rr[16];
            tc_ld16(tmem + lane_off + c16 * 16, rr);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) wmax = fmaxf(wmax, fabsf(wval(__uint_as_float(rr[i]), c16 * 16 + i)));
        }
    }
    // e_t: 2^-e_t wmax < 2^15
    const int ebits = (int)((__float_as_uint(wmax) >> 23) & 255) - 127;
    const int e_t = ebits > 14 ? ebits - 14 : 0;
    const float down = pow2f(-e_t);
    if (ok) {
#pragma unroll 1
        for (int c16 = 0; c16 < 8; ++c16) {
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
    // ---- O = (W_hi + W_lo) [V|1]  [128 t x NV], K = 128
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
    // ---- epilogue: add the inter-chunk partials, divide, stage the row
    float *stg = reinterpret_cast<float *>(sm);
    if (ok) {
        const float up = pow2f(e_t);
        const float *rp = red + ((bh * nc + cl) * (DV + 1)) * kL + t;
        float inv;
        {   // denominator: column DV
            uint32_t rr[16];
            tc_ld16(tmem + 128 + lane_off + DV, rr);
            tc_wait_ld();
            const float den = fmaf(__uint_as_float(rr[0]), up, rp[DV * kL]);
            inv = 1.f / den;
            if (den_out && t < nt) den_out[bh * N + t0 + t] = den;   // kept for the backward pass
        }
#pragma unroll
        for (int c16 = 0; c16 < DV / 16; ++c16) {
            uint32_t rr[16];
            tc_ld16(tmem + 128 + lane_off + c16 * 16, rr);
            tc_wait_ld();
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = c16 * 16 + 4 * i4 + i;
                    o[i] = fmaf(__uint_as_float(rr[4 * i4 + i]), up, rp[j * kL]) * inv;
                }
                *reinterpret_cast<float4 *>(stg + t * F::STG + c16 * 16 + 4 * i4) = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
    }
    tc_before();
    __syncthreads();
    if (ok) {
        float4 *o4 = reinterpret_cast<float4 *>(out + (bh * N + t0) * DV);
        for (int e = tid; e < nt * (DV / 4); e += 128) {
            const int r = e / (DV / 4), c4 = e % (DV / 4);
            o4[e] = *reinterpret_cast<const float4 *>(stg + r * F::STG + 4 * c4);
        }
    }
    if (warp == 0) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256) : "memory");
    }
}

// ------------------------------------------------------------------ host ----

// Unit plan: which (pair tile, l values) each CTA owns, and per (unit, l slot,
// row) the basis index and C/p! of feature (a, b, l), or -1 / 0 where the row
// is no feature (b > l, degree >= P, or a padding pair).
struct UnitPlan {
    int D = 0, P = 0, MT = 0, MT_MAX = 0, NPT = 0, G = 0;
    std::vector<uint16_t> pairs;       // [NPT*128]
    std::vector<int32_t> unit_k, unit_nl, unit_l;   // [G], [G], [G*MT_MAX]
    std::vector<float> coef;           // [G*MT_MAX*128]
    std::vector<int32_t> fidx;         // [G*MT_MAX*128]
    size_t off_k = 0, off_nl = 0, off_l = 0, off_coef = 0, off_fidx = 0, bytes = 0;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

bool build_unit_plan(int D, int P, int MT, int MT_MAX, UnitPlan &up) {
    HostBasis hb;
    if (!build_basis_host(D, P, hb)) return false;
    // basis index of each sorted tuple of real indices (indices < D), keyed a | b << 8 | l << 16
    std::map<uint32_t, int32_t> index_of;
    for (size_t f = 0; f < hb.tuples.size(); ++f) {
        uint32_t idx[3] = {(uint32_t)D, (uint32_t)D, (uint32_t)D};
        for (size_t m = 0; m < hb.tuples[f].size(); ++m) idx[m] = hb.tuples[f][m];
        index_of[idx[0] | (idx[1] << 8) | (idx[2] << 16)] = (int32_t)f;
    }
    up.D = D;
    up.P = P;
    up.MT = MT;
    up.MT_MAX = MT_MAX;
    const int npair = (D + 1) * (D + 2) / 2;
    up.NPT = (npair + 127) / 128;
    up.pairs.assign((size_t)up.NPT * 128, (uint16_t)(D | (D << 8)));
    std::vector<int> pa(npair), pb(npair);
    {
        int i = 0;
        for (int b = 0; b <= D; ++b)
            for (int a = 0; a <= b; ++a, ++i) {
                pa[i] = a;
                pb[i] = b;
                up.pairs[i] = (uint16_t)(a | (b << 8));
            }
    }
    struct Unit {
        int k, nl;
        int l[16];
    };
    std::vector<Unit> units;
    int64_t covered = 0;
    for (int k = 0; k < up.NPT; ++k) {
        std::vector<int> ls;
        for (int l = 0; l <= D; ++l) {
            bool any = false;
            for (int r = 0; r < 128 && !any; ++r) {
                const int i = k * 128 + r;
                if (i >= npair || pb[i] > l) continue;
                const int p = (pa[i] < D) + (pb[i] < D) + (l < D);
                any = p < P;
            }
            if (any) ls.push_back(l);
        }
        for (size_t s = 0; s < ls.size(); s += MT) {
            Unit u{k, 0, {}};
            for (size_t j = s; j < ls.size() && j < s + MT; ++j) u.l[u.nl++] = ls[j];
            units.push_back(u);
        }
    }
    std::stable_sort(units.begin(), units.end(), [](const Unit &x, const Unit &y) { return x.nl > y.nl; });
    up.G = (int)units.size();
    up.unit_k.resize(up.G);
    up.unit_nl.resize(up.G);
    up.unit_l.assign((size_t)up.G * MT_MAX, D);
    up.coef.assign((size_t)up.G * MT_MAX * 128, 0.f);
    up.fidx.assign((size_t)up.G * MT_MAX * 128, -1);
    for (int g = 0; g < up.G; ++g) {
        const Unit &u = units[g];
        up.unit_k[g] = u.k;
        up.unit_nl[g] = u.nl;
        for (int j = 0; j < u.nl; ++j) {
            const int l = u.l[j];
            up.unit_l[(size_t)g * MT_MAX + j] = l;
            for (int r = 0; r < 128; ++r) {
                const int i = u.k * 128 + r;
                if (i >= npair || pb[i] > l) continue;
                const int p = (pa[i] < D) + (pb[i] < D) + (l < D);
                if (p >= P) continue;
                auto it = index_of.find((uint32_t)pa[i] | ((uint32_t)pb[i] << 8) | ((uint32_t)l << 16));
                if (it == index_of.end()) return false;
                const size_t at = ((size_t)g * MT_MAX + j) * 128 + r;
                up.fidx[at] = it->second;
                // C_p / p! = 1 / prod over runs of equal real indices of (run length)!
                up.coef[at] = (float)((double)hb.mult[it->second] / (p == 3 ? 6.0 : (p == 2 ? 2.0 : 1.0)));
                ++covered;
            }
        }
    }
    if (covered != (int64_t)hb.tuples.size()) return false;   // every feature exactly once
    up.off_k = align256((size_t)up.NPT * 128 * sizeof(uint16_t));
    up.off_nl = up.off_k + align256((size_t)up.G * 4);
    up.off_l = up.off_nl + align256((size_t)up.G * 4);
    up.off_coef = up.off_l + align256((size_t)up.G * MT_MAX * 4);
    up.off_fidx = up.off_coef + align256(up.coef.size() * 4);
    up.bytes = up.off_fidx + align256(up.fidx.size() * 4);
    return true;
}

std::mutex g_plan_mu;
std::map<std::tuple<int, int, int>, UnitPlan> g_plans;

const UnitPlan *unit_plan(int D, int P, int MT, int MT_MAX) {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    const auto key = std::make_tuple(D, P, MT);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) return &it->second;
    UnitPlan up;
    if (!build_unit_plan(D, P, MT, MT_MAX, up)) return nullptr;
    return &g_plans.emplace(key, std::move(up)).first->second;
}

struct Plan {
    const UnitPlan *up = nullptr;
    int G = 1, nchunks = 0, nc_seg = 0;
    size_t off_stats = 0, off_img = 0, off_part = 0, off_red = 0, off_state = 0, total = 0;
};

template <int DK, int DV>
bool make_plan(int BH, int64_t N, int64_t F, int P, bool need_state, int min_segments, Plan &pl) {
    using C = Cfg<DK, DV>;
    // l values per CTA: as many as fit, unless that leaves the SMs without a full wave
    int mt = C::MT_MAX;
    const UnitPlan *up = unit_plan(DK, P, mt, C::MT_MAX);
    while (up && mt > 1 && (int64_t)BH * up->G < 148) up = unit_plan(DK, P, --mt, C::MT_MAX);
    if (!up) return false;
    pl.up = up;
    pl.G = up->G;
    pl.nchunks = (int)((N + kL - 1) / kL);
    const size_t per_chunk = (size_t)BH * pl.G * (DV + 1) * kL * sizeof(float);
    int64_t seg = (int64_t)(kPartialBudget / per_chunk);
    if (seg < 1) seg = 1;
    // segments of equal length: as few as the partial budget allows, at least min_segments
    int64_t nseg = (pl.nchunks + seg - 1) / seg;
    if (nseg < min_segments) nseg = min_segments < pl.nchunks ? min_segments : pl.nchunks;
    if (nseg < 1) nseg = 1;
    pl.nc_seg = (int)((pl.nchunks + nseg - 1) / nseg);
    pl.off_stats = 0;
    pl.off_img = align256((size_t)BH * 4 * sizeof(float));
    pl.off_part = pl.off_img + align256((size_t)BH * pl.nchunks * C::IMG);
    pl.off_red = pl.off_part + align256(per_chunk * pl.nc_seg);
    pl.off_state = pl.off_red + align256((size_t)BH * (DV + 1) * kL * sizeof(float) * pl.nc_seg);
    pl.total = pl.off_state + (need_state ? align256((size_t)BH * F * (DV + 1) * sizeof(float)) : 0);
    (void)F;
    return true;
}

// Enqueue the copy of token rows [t0, t1) of a [BH][N][width] tensor (elem bytes each).
cudaError_t copy_rows(void *dst, const void *src, int BH, int64_t N, int64_t t0, int64_t t1, int width, int elem,
                      cudaMemcpyKind kind, cudaStream_t s) {
    const size_t pitch = (size_t)N * width * elem, off = (size_t)t0 * width * elem;
    return cudaMemcpy2DAsync((uint8_t *)dst + off, pitch, (const uint8_t *)src + off, pitch,
                             (size_t)(t1 - t0) * width * elem, BH, kind, s);
}

template <int DK, int DV>
cudaError_t run(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k, const void *v,
                float *out, float *S, float *Z, bool state_in, void *ws, size_t ws_bytes, int *flags,
                cudaStream_t stream, const HostIO *io, float *den_out) {
    using C = Cfg<DK, DV>;
    const int64_t F = basis.F;
    const bool own_state = (S == nullptr);
    const int min_seg = io ? kHostSegments : 1;
    Plan pl, need;
    if (!make_plan<DK, DV>(BH, N, F, basis.P, true, min_seg, pl) ||
        !make_plan<DK, DV>(BH, N, F, basis.P, own_state, min_seg, need))
        return cudaErrorInvalidValue;
    if (ws_bytes < need.total) return cudaErrorInvalidValue;
    const UnitPlan &up = *pl.up;
    cudaError_t e = cudaSuccess;
    const uint8_t *tab = (const uint8_t *)device_table(
        ((uint64_t)DK << 32) | ((uint64_t)basis.P << 16) | (uint64_t)up.MT, up.bytes,
        [&up](uint8_t *h) {
            std::memcpy(h, up.pairs.data(), up.pairs.size() * sizeof(uint16_t));
            std::memcpy(h + up.off_k, up.unit_k.data(), up.unit_k.size() * 4);
            std::memcpy(h + up.off_nl, up.unit_nl.data(), up.unit_nl.size() * 4);
            std::memcpy(h + up.off_l, up.unit_l.data(), up.unit_l.size() * 4);
            std::memcpy(h + up.off_coef, up.coef.data(), up.coef.size() * 4);
            std::memcpy(h + up.off_fidx, up.fidx.data(), up.fidx.size() * 4);
        },
        &e);
    if (!tab) return e != cudaSuccess ? e : cudaErrorMemoryAllocation;
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

    e = cudaMemsetAsync(stats, 0, (size_t)BH * 4 * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const size_t prep_smem = sizeof(__half) * kL * (2 * (DK + 2) + (DV + 2));
    e = cudaFuncSetAttribute(tc_prep_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_scan_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_finish_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             FinCfg<DK, DV>::SMEM);
    if (e != cudaSuccess) return e;
    int stall = -1;
    if (g_opt_test_stall) {
        stall = pl.nchunks > 1 ? 1 : 0;
        g_opt_test_stall = 0;
    }
    const int64_t wait_ns = g_opt_wait_limit > 0 ? g_opt_wait_limit : kDefaultWaitNs;
    // events of the host-buffer pipeline; released once enqueued (they live until they complete)
    std::vector<cudaEvent_t> events;
    auto new_event = [&events](cudaEvent_t *ev) {
        cudaError_t r = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        if (r == cudaSuccess) events.push_back(*ev);
        return r;
    };
    struct Release {
        std::vector<cudaEvent_t> &ev;
        ~Release() { for (cudaEvent_t x : ev) cudaEventDestroy(x); }
    } release{events};
    for (int s = 0; s < nseg; ++s) {
        const int c0s = s * pl.nc_seg;
        const int ncs = (pl.nchunks - c0s < pl.nc_seg) ? pl.nchunks - c0s : pl.nc_seg;
        const int64_t tok0 = (int64_t)c0s * kL, tok1 = (int64_t)(c0s + ncs) * kL < N ? (int64_t)(c0s + ncs) * kL : N;
        if (io) {   // this segment's inputs: host -> device on the copy stream, compute waits for them
            cudaEvent_t ev;
            if ((e = copy_rows((void *)q, io->q, BH, N, tok0, tok1, DK, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = copy_rows((void *)k, io->k, BH, N, tok0, tok1, DK, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = copy_rows((void *)v, io->v, BH, N, tok0, tok1, DV, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = new_event(&ev)) || (e = cudaEventRecord(ev, io->h2d)) || (e = cudaStreamWaitEvent(stream, ev, 0)))
                return e;
        }
        {   // chunk images and per-head maxima of this segment (maxima accumulate over segments)
            const int64_t nwork = (int64_t)BH * ncs;
            const int prep_grid = (int)(nwork < 148 * 8 ? nwork : 148 * 8);
            launch_begin(kTcPrep, stream);
            tc_prep_kernel<DK, DV><<<prep_grid, 256, prep_smem, stream>>>(qb, kb, vb, img, stats, BH, N, pl.nchunks,
                                                                           c0s, ncs, inv_c);
            launch_end(kTcPrep, stream);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            if (s == 0 && state_in) {
                tc_state_stats_kernel<<<dim3(BH, 8), 256, 0, stream>>>(S, Z, stats, F, DV);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
        }
        ScanParams sp;
        sp.img = img;
        sp.stats = stats;
        sp.pairs = (const uint16_t *)tab;
        sp.unit_k = (const int32_t *)(tab + up.off_k);
        sp.unit_nl = (const int32_t *)(tab + up.off_nl);
        sp.unit_l = (const int32_t *)(tab + up.off_l);
        sp.unit_coef = (const float *)(tab + up.off_coef);
        sp.unit_fidx = (const int32_t *)(tab + up.off_fidx);
        sp.S = S;
        sp.Z = Z;
        float *red = (float *)(w + pl.off_red);
        const int nc_here = (pl.nchunks - s * pl.nc_seg < pl.nc_seg) ? pl.nchunks - s * pl.nc_seg : pl.nc_seg;
        const bool atomic = g_opt_deterministic == 0;
        if (atomic && (e = cudaMemsetAsync(red, 0, (size_t)BH * nc_here * (DV + 1) * kL * sizeof(float), stream)) !=
                          cudaSuccess)
            return e;
        sp.part = atomic ? red : part;
        sp.red_atomic = atomic ? 1 : 0;
        sp.flags = flags;
        sp.F = F;
        sp.N = N;
        sp.BH = BH;
        sp.G = pl.G;
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
        if (!atomic) {   // the units' partials summed in a fixed order
            const int64_t rwork = (int64_t)BH * sp.nc * (DV + 1) * (kL / 4);
            launch_begin(kTcReduce, stream);
            tc_reduce_kernel<DV><<<(int)((rwork + 255) / 256 < 148 * 32 ? (rwork + 255) / 256 : 148 * 32), 256, 0,
                                   stream>>>((const float4 *)part, (float4 *)red, BH, pl.G, sp.nc);
            launch_end(kTcReduce, stream);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        launch_begin(kTcFinish, stream);
        tc_finish_kernel<DK, DV><<<(int)((int64_t)BH * sp.nc), 128, FinCfg<DK, DV>::SMEM, stream>>>(
            qb, kb, vb, red, out, den_out, sp.c0, sp.nc, N, basis.P, inv_c, flags, wait_ns);
        launch_end(kTcFinish, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (io) {   // this segment's output: device -> host on the second copy stream
            cudaEvent_t ev;
            if ((e = new_event(&ev)) || (e = cudaEventRecord(ev, stream)) || (e = cudaStreamWaitEvent(io->d2h, ev, 0)) ||
                (e = copy_rows(io->out, out, BH, N, tok0, tok1, DV, 4, cudaMemcpyDeviceToHost, io->d2h)))
                return e;
        }
    }
    if (io) {   // the caller's stream completes after the last copy back
        cudaEvent_t ev;
        if ((e = new_event(&ev)) || (e = cudaEventRecord(ev, io->d2h)) || (e = cudaStreamWaitEvent(stream, ev, 0)))
            return e;
    }
    return cudaSuccess;
}

}  // namespace

bool prefill_tc_supported(int d_K, int d_V, int P) {
    return d_K == d_V && (d_K == 16 || d_K == 32 || d_K == 64) && P >= 1 && P <= 4;
}

size_t prefill_tc_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P, bool need_state,
                                  bool host_io) {
    Plan pl;
    bool ok = false;
    const int ms = host_io ? kHostSegments : 1;
    switch (d_K * 1000 + d_V) {
        case 16016: ok = make_plan<16, 16>(BH, N, F, P, need_state, ms, pl); break;
        case 32032: ok = make_plan<32, 32>(BH, N, F, P, need_state, ms, pl); break;
        case 64064: ok = make_plan<64, 64>(BH, N, F, P, need_state, ms, pl); break;
        default: break;
    }
    return ok ? pl.total : 0;
}

cudaError_t launch_prefill_tc(const DeviceBasis &basis, int BH, int64_t N, int d_V, const void *q,
                              const void *k, const void *v, float *out, float *S, float *Z, bool state_in,
                              void *ws, size_t ws_bytes, int *flags, cudaStream_t stream, const HostIO *io,
                              float *den_out) {
    switch (basis.d_K * 1000 + d_V) {
        case 16016:
            return run<16, 16>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io, den_out);
        case 32032:
            return run<32, 32>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io, den_out);
        case 64064:
            return run<64, 64>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io, den_out);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace sata
