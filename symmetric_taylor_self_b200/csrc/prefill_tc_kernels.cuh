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
// Feature organisation.  With x~ = (x, 1) (index D = d_K is the constant 1), the
// basis for P <= 4 is exactly the nondecreasing triples a <= b <= l over 0..D
// (a degree-p monomial is its p real indices followed by D's).  A feature is the
// pair product P2(x)_(a,b) = x~_a x~_b times x~_l.  Pairs are sorted by b, then a,
// and cut into tiles of 128.  A unit (one CTA) owns one pair tile and up to NL
// values l_0..l_{nl-1} ("slots") of the last index.  Its state is one TMEM
// accumulator [128 pairs] x [V_l0 | V_l1 | ... | Z_l0 Z_l1 ... | 0 pad], NU columns.
//
// Chunked form, chunk c of L = 128 tokens (every quantity per head):
//   update   [S|Z] += P2(K_c)^T . W_c,        W_c[t] = [k~_l0 v_t | k~_l1 v_t | ... | k~_l0 k~_l1 ...]
//   readout  R_c    = P2(Q_c) . B_c,           B_c = (C/p! [S|Z] before chunk c), per row and slot
//            num_t += sum_s q~_ls[t] R_c[t, V_s],  den_t += sum_s q~_ls[t] R_c[t, Z_s]
//   intra    sum_{s in c, s <= t} w_ts [v_s | 1], w = sum_p (q.k/c)^p/p!   (finish kernel)
// so the slots share one A operand per side: both contractions are single
// M = 128, N = NU <= 208, K = 128 products per chunk (8 tcgen05.mma each), the
// l factor sits in the B operand of the update and in a per-token epilogue of
// the readout.  P2(q), P2(k) and W are generated from the token rows
// (thread = token) with compile-time pair tables; nothing of the features
// reaches HBM.
//
// Precision: fp16 operands, fp32 accumulation.  Every head's q, k and v are
// prescaled by powers of two (2^-e_q, 2^-e_k, 2^-e_v, from the head's maxima) so
// that every fp16 operand lies below 1 in magnitude, whatever the input range; a
// bf16 value times a power of two is exact in fp16, so the token rows carry no
// rounding.  phi_p(x~) scales by 2^(p e) exactly, and the readout operand of a
// degree-p row carries C/p! c^-p 2^(p (e_q + e_k)) in its fp32 coefficient (1/c is
// irrational for most d_K: folding it into q before the fp16 rounding would cost a
// rounding of every q, amplified by the cancellation inside q.k).  The state is rounded to fp16
// only as the readout operand, after a further power-of-two scale 2^-sigma_c from a
// rigorous bound on |S|, undone in fp32 after the contraction.  Everything stored
// in HBM (state, sums, output) is in the true, unscaled frame.
//
// This header holds the kernels and the host driver as templates over (d_K, d_V); the
// prefill_tc_*.cu files instantiate them (prefill_tc_shapes.h lists the shapes) and
// prefill_tc.cu dispatches.
//
// Kernels: tc_stats (per-head maxima), tc_prep (prescaled fp16 token rows),
// tc_state_stats (max |state| when continuing), tc_scan (the warp-specialised
// scan), tc_reduce (fixed-order sum of unit partials, deterministic mode only),
// tc_finish (intra-chunk block on tensor cores, division).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cfloat>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "prefill_tc_shapes.h"
#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kL = 128;                    // chunk length (tokens)
// Readout sums of a (head, chunk): [DQ][128 tokens][4] fp32, DQ = ceil((d_V + 1) / 4) quads of
// columns (V columns, then the Z column, zero padding): a thread adds its token's quad with
// one vector reduction, and 32 consecutive tokens cover 512 contiguous bytes.
__host__ __device__ constexpr int sum_quads(int DV) { return (DV + 1 + 3) / 4; }
constexpr int kNMax = 208;                 // widest unit: TMEM state + readout + P2(q) <= 512 columns
constexpr int kScanWarps = 13;          // at most 4 warps per SM sub-partition: 128 registers each
constexpr int kScanThreads = kScanWarps * 32;
// warp roles: MMA issuer (one thread, both contractions, in chunk order), k side (4, thread =
// token), q side (4, thread = token = TMEM lane), state conversion (4, thread = pair row = TMEM
// lane)
constexpr int kWarpI = 0, kWarpK0 = 1, kWarpQ0 = 5, kWarpC0 = 9;
constexpr int64_t kDefaultWaitNs = 2000000000LL;   // 2 s per wait
constexpr size_t kPartialBudget = size_t(4) << 30;  // fixed-order mode: unit partials per segment

template <int DK, int DV>
struct Cfg {
    static_assert(DK % 16 == 0 && DK <= 128 && DV % 16 == 0 && DV <= 128, "head sizes");
    static constexpr int D = DK;
    static constexpr int NL = kNMax / (DV + 1) < 1 ? 1 : kNMax / (DV + 1);   // slots per unit
    static constexpr int NMAX = (NL * (DV + 1) + 15) / 16 * 16;              // widest unit N
    static constexpr int NG = NMAX / 16;                                      // 16-column groups
    static constexpr int XW = DK / 2 + 1;        // half2 words of a token row x~ = (x, 1)
    static constexpr int NPAIR = (D + 1) * (D + 2) / 2;
    static constexpr int NPT = (NPAIR + 127) / 128;
    // TMEM columns: state, readout accumulator (32-aligned: the drain reads 32 columns at a
    // time), P2(q) operand (two fp16 per column)
    static constexpr int COL_S = 0, COL_R = (NMAX + 31) / 32 * 32, COL_AQ = COL_R + NMAX;
    // shared memory: P2(k) operand x2 (128-byte swizzled MN-major), W and the state operand
    // B x2 (MN-major core matrices, K groups of 8 rows LBO bytes apart)
    static constexpr int AK_BYTES = 128 * 128 * 2;
    static constexpr int W_BYTES = 128 * NMAX * 2;
    static constexpr int LBO = NMAX * 16;
    static constexpr int OFF_AK = 0;
    static constexpr int OFF_W = 2 * AK_BYTES;
    static constexpr int OFF_BS = OFF_W + W_BYTES;
    static constexpr int OFF_L = OFF_BS + 2 * W_BYTES;   // int [NL]: the unit's l values
    static constexpr int OFF_BAR = OFF_L + 64;
    // barriers: P2(k)+W full, P2(k) buffer empty x2, update done, state read, B full x2, B empty x2,
    // P2(q) full, readout accumulator free, readout done, final drain
    static constexpr int B_AKF = 0, B_AKE = 1, B_UD = 3, B_SR = 4, B_BSF = 5, B_BSE = 7, B_AQF = 9, B_RF = 10,
                         B_RD = 11, B_FIN = 12, N_BAR = 13;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;    // + base alignment slack
    static_assert(COL_AQ + 64 <= 512, "TMEM columns");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(NL <= 16 && NL * 4 <= 64, "slot table");
};

struct ScanParams {
    const __half *q16, *k16, *v16;   // prescaled fp16 token rows, chunk-interleaved (chunk_rows)
    const float *stats;              // [BH][4] max|q|, max|k|, max|v| (this segment), max|state in|
    const uint16_t *pairs;           // [NPT][128]  a | b << 8
    const int32_t *unit_k;           // [G] pair tile of each unit
    const int32_t *unit_nl;          // [G] number of slots
    const int32_t *unit_l;           // [G][NL]
    const float *unit_coef;          // [G][NL][128] C/p! of feature (pair, l), 0 if none
    const int32_t *unit_fidx;        // [G][NL][128] basis index of feature (pair, l), -1 if none
    float *S, *Z;                    // state in/out (true frame)
    float *part;                     // sums [BH][nc][DV+1][128] (red_atomic) or [BH][G][nc][DV+1][128]
    int red_atomic;
    int *flags;
    int64_t F, N;
    int BH, G, c0, nc, nch, P;
    int load_state, store_state, stall_chunk;
    float inv_c;
    int lc;                          // floor(log2 c): the readout operand's scale bound
    int64_t wait_ns;
    // gradient scans (JAC kernels) only: Z-column values per token (prescaled fp16, chunk-
    // interleaved [BH][nch][128]; null: the constant 1), whether the Z columns carry the
    // column prescale, the readout's per-token multipliers (fp32, true frame, chunk-
    // interleaved float4 quads: quad j of token t of chunk c of head bh at element
    // ((bh nch + c) mult_quads + j) 128 + t) and the sums [BH][d_K][N] the drain adds into
    const __half *zval16 = nullptr;
    int zscaled = 0;
    const float *mult = nullptr;
    int mult_quads = 0;
    float *sums_jac = nullptr;
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
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
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
// 2^e for any e: 0 below 2^-126 (such terms are below fp16 resolution of every
// operand they meet), saturating at 2^127.
__device__ __forceinline__ float pow2f_sat(int e) {
    if (e < -126) return 0.f;
    if (e > 127) e = 127;
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// Smallest e with m * 2^-e < 1 (clamped to +-126); 0 for m = 0 or NaN.
__device__ __forceinline__ int scale_exp(float m) {
    if (!(m > 0.f)) return 0;
    const int e = (int)((__float_as_uint(m) >> 23) & 255) - 126;
    return e < -126 ? -126 : (e > 126 ? 126 : e);
}
// The head's prescale exponents: q, k, v are multiplied by 2^-e_q, 2^-e_k, 2^-e_v.
struct HeadExp {
    int eq, ek, ev;
};
__device__ __forceinline__ HeadExp head_exps(const float *st) {
    return HeadExp{scale_exp(st[0]), scale_exp(st[1]), scale_exp(st[2])};
}
// Exponent sigma_c of the readout operand's scale before chunk cl of this call:
// |S'| < 2^e_ms + 128 cl + 1 (every prescaled feature and value is at most 1 in
// magnitude, e_ms bounds the prescaled incoming state), and a degree-p row carries
// C/p! c^-p 2^(p E) <= 2^(p (E - lc)) <= 2^max(0, (P-1)(E - lc)) (C/p! <= 1, lc =
// floor(log2 c)), so |B| < 2^15 for every row.  The bound is tight for the rows that
// reach it; a looser one would push the small rows of B into fp16's subnormal range.
__device__ __forceinline__ int state_sigma_rows(int cl, int e_ms, int e_row) {
    const uint32_t tok = (uint32_t)cl * kL + 1u;
    const int e_tok = 32 - __clz(tok);
    const int eb = (e_ms > e_tok ? e_ms : e_tok) + 1;
    const int s = eb + e_row - 15;
    return s < -120 ? -120 : (s > 120 ? 120 : s);
}
__device__ __forceinline__ int state_sigma(int cl, int e_ms, int E, int P, int lc) {
    const int r = (P - 1) * (E - lc);
    return state_sigma_rows(cl, e_ms, r > 0 ? r : 0);
}
// The same for a gradient scan: a pair row of degree p' <= P - 2 carries
// C/p'! c^-(p'+1) 2^(p' E + e_k) <= 2^(p' (E - lc) + e_k - lc) (the slot index is a
// key-side factor only; the derivative's 1/c is in the row).
__device__ __forceinline__ int jac_sigma(int cl, int E, int ek, int P, int lc) {
    const int r = (P - 2) * (E - lc);
    return state_sigma_rows(cl, -1000, (r > 0 ? r : 0) + ek - lc);
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
__device__ __forceinline__ uint4 hmul2x4(uint4 a, uint32_t b) {
    return make_uint4(hmul2u(a.x, b), hmul2u(a.y, b), hmul2u(a.z, b), hmul2u(a.w, b));
}
__device__ __forceinline__ float h_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))); }

// Pair (a, b), a <= b <= D, sorted by b then a: index b (b + 1) / 2 + a; indices
// past the last pair stand for (D, D).  The host plan uses the same order.
template <int D>
struct Pairs {
    static constexpr int N = (D + 1) * (D + 2) / 2;
    __host__ __device__ static constexpr int b(int idx) {
        if (idx >= N) return D;
        int v = 0;
        while ((v + 1) * (v + 2) / 2 <= idx) ++v;
        return v;
    }
    __host__ __device__ static constexpr int a(int idx) { return idx >= N ? D : idx - b(idx) * (b(idx) + 1) / 2; }
};

// Two fp16 values x~_i0, x~_i1 of a token row held as packed half2 registers, as
// one half2 with i0 in the low half.
template <int I0, int I1, int NX>
__device__ __forceinline__ uint32_t pick2(const uint32_t (&x)[NX]) {
    if constexpr (I0 % 2 == 0 && I1 == I0 + 1) {
        return x[I0 / 2];
    } else {
        constexpr uint32_t s0 = (I0 % 2) * 2, s2 = 4 + (I1 % 2) * 2;
        return __byte_perm(x[I0 / 2], x[I1 / 2], s0 | ((s0 + 1) << 4) | (s2 << 8) | ((s2 + 1) << 12));
    }
}
// P2 of one token row for pair tile K, half2 word M = pairs (2M, 2M+1) of the tile.
template <int D, int K, int M, int NX>
__device__ __forceinline__ uint32_t p2_at(const uint32_t (&x)[NX]) {
    using PT = Pairs<D>;
    return hmul2u(pick2<PT::a(K * 128 + 2 * M), PT::a(K * 128 + 2 * M + 1)>(x),
                  pick2<PT::b(K * 128 + 2 * M), PT::b(K * 128 + 2 * M + 1)>(x));
}
// q side: P2 of the token into 64 registers (the TMEM A operand row).
template <int D, int K, int NX, int... M>
__device__ __forceinline__ void p2q_tile(const uint32_t (&x)[NX], uint32_t (&pq)[64], std::integer_sequence<int, M...>) {
    ((pq[M] = p2_at<D, K, M>(x)), ...);
}
// Tile k of NPT (the last tile also serves any k out of range, so every path writes pq).
template <int D, int K, int NPT, int NX>
__device__ __forceinline__ void p2q_dispatch(int k, const uint32_t (&x)[NX], uint32_t (&pq)[64]) {
    if constexpr (K == NPT - 1) {
        p2q_tile<D, K>(x, pq, std::make_integer_sequence<int, 64>{});
    } else {
        if (k == K) p2q_tile<D, K>(x, pq, std::make_integer_sequence<int, 64>{});
        else p2q_dispatch<D, K + 1, NPT>(k, x, pq);
    }
}
// k side: P2 of the token stored as row t (a K row) of the 128-byte-swizzled
// MN-major A operand: 64-pair M blocks 16 KB apart, 16-byte chunk j of the row at
// chunk position j ^ (t mod 8).
template <int D, int K, int NX, int... J>
__device__ __forceinline__ void p2k_tile(const uint32_t (&x)[NX], uint8_t *ak, int t, std::integer_sequence<int, J...>) {
    ((*reinterpret_cast<uint4 *>(ak + (J / 8) * 16384 + t * 128 + (((J % 8) ^ (t & 7)) << 4)) =
          make_uint4(p2_at<D, K, 4 * J>(x), p2_at<D, K, 4 * J + 1>(x), p2_at<D, K, 4 * J + 2>(x),
                     p2_at<D, K, 4 * J + 3>(x))),
     ...);
}
template <int D, int NX, int... K>
__device__ __forceinline__ void p2k_dispatch(int k, const uint32_t (&x)[NX], uint8_t *ak, int t,
                                             std::integer_sequence<int, K...>) {
    ((k == K ? (p2k_tile<D, K>(x, ak, t, std::make_integer_sequence<int, 16>{}), 0) : 0), ...);
}

// Prescaled fp16 token rows are stored chunk-interleaved: piece j (values 8j..8j+7) of
// token t of chunk c of head bh is 16-byte element ((bh * nch + c) * (D / 8) + j) * 128 + t,
// so 32 consecutive tokens reading one piece read 512 contiguous bytes.  chunk_rows gives
// the chunk's first element.
template <int D>
__device__ __forceinline__ const uint4 *chunk_rows(const __half *x16, int64_t bh, int nch, int c) {
    return reinterpret_cast<const uint4 *>(x16) + ((int64_t)bh * nch + c) * (D / 8) * 128;
}
// Token row x~ = (x, 1) of token t of a chunk (zeros past the sequence end).
template <int DK, int NX>
__device__ __forceinline__ void load_row(const uint4 *cr, int t, bool valid, uint32_t (&x)[NX]) {
#pragma unroll
    for (int i = 0; i < DK / 8; ++i) {
        uint4 u = make_uint4(0, 0, 0, 0);
        if (valid) u = __ldg(cr + i * 128 + t);
        x[4 * i] = u.x;
        x[4 * i + 1] = u.y;
        x[4 * i + 2] = u.z;
        x[4 * i + 3] = u.w;
    }
    x[DK / 2] = 0x3C00u;   // x~_D = 1 (low half)
}
// x~_l of token t as a half2 broadcast (x~_D = 1; 0 past the sequence end).  Read back
// from memory (the row was just fetched): a select over the row's registers with a
// runtime l is turned into an indexed local-memory copy of the row.
__device__ __forceinline__ uint32_t row_half2(const uint4 *cr, int t, int l, int D, bool valid) {
    if (!valid) return 0u;
    const uint32_t h =
        l < D ? (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(cr + (l >> 3) * 128 + t) + (l & 7)) : 0x3C00u;
    return h | (h << 16);
}
template <int N>
__device__ __forceinline__ float sel(const float (&a)[N], int i) {
    float r = 0.f;
#pragma unroll
    for (int j = 0; j < N; ++j) r = (j == i) ? a[j] : r;
    return r;
}
template <int N>
__device__ __forceinline__ int seli(const int (&a)[N], int i) {
    int r = 0;
#pragma unroll
    for (int j = 0; j < N; ++j) r = (j == i) ? a[j] : r;
    return r;
}

// ----------------------------------------------------------------- prep ----

// Per-head maxima of |q|, |k|, |v| over tokens [t0, t1): max of the bf16 bit
// patterns without sign (a NaN input orders above +inf), then one atomic max per
// block on the fp32 bit pattern (non-negative floats order like their bits).
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
                int bpb) {
    const int64_t bh = blockIdx.x / bpb;   // bpb blocks per head
    const int bx = blockIdx.x % bpb;
    uint32_t mq = 0, mk = 0, mv = 0;
    const int64_t nqk = (t1 - t0) * (DK / 8), nv = (t1 - t0) * (DV / 8);
    const uint4 *q4 = reinterpret_cast<const uint4 *>(q + (bh * N + t0) * DK);
    const uint4 *k4 = reinterpret_cast<const uint4 *>(k + (bh * N + t0) * DK);
    const uint4 *v4 = reinterpret_cast<const uint4 *>(v + (bh * N + t0) * DV);
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
// whose inputs are not finite raises the range flag (its outputs are NaN).
template <int D>
__device__ __forceinline__ void prep_rows(const __nv_bfloat16 *__restrict__ x, __half *__restrict__ x16,
                                          const float *__restrict__ stats, int which, int BH, int64_t N,
                                          int64_t t0, int64_t t1, int nch) {
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
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (bh * N + tok) * D);
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
               int nch, int *flags) {
    if (blockIdx.x == 0)
        for (int bh = threadIdx.x; bh < BH; bh += blockDim.x)
            if (!(stats[bh * 4] <= FLT_MAX && stats[bh * 4 + 1] <= FLT_MAX && stats[bh * 4 + 2] <= FLT_MAX))
                atomicExch(flags + kFlagRange, 1);
    prep_rows<DK>(q, q16, stats, 0, BH, N, t0, t1, nch);
    prep_rows<DK>(k, k16, stats, 1, BH, N, t0, t1, nch);
    prep_rows<DV>(v, v16, stats, 2, BH, N, t0, t1, nch);
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

// Token row t of chunk cl into registers, with x~_l of each slot (half2 broadcasts).
template <int DK, int NX, int NL>
__device__ __forceinline__ void fetch_row(const __half *x16, const ScanParams &p, int64_t bh, const int *sl, int cl,
                                          int t, uint32_t (&x)[NX], uint32_t (&xl)[NL]) {
    const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
    const uint4 *cr = chunk_rows<DK>(x16, bh, p.nch, p.c0 + cl);
    load_row<DK>(cr, t, valid, x);
#pragma unroll
    for (int s = 0; s < NL; ++s) xl[s] = row_half2(cr, t, sl[s], DK, valid);
}

// q side: readout R of chunk cl (TMEM, this warp's lanes), combined over the slots with
// q~_l, scaled to the true frame and added into the head's sums (or written as this
// unit's partial).  Arrives on rf_bar once every column is read.
template <int DK, int DV>
__device__ __forceinline__ void q_drain(const ScanParams &p, int64_t bh, int64_t part_base, int nl, int e_ms, int E,
                                        int ev, int cl, int t, int lane, uint32_t tm, uint32_t rf_bar,
                                        const float (&qv)[Cfg<DK, DV>::NL]) {
    using C = Cfg<DK, DV>;
    constexpr int NL = C::NL;
    tc_after();
    const int sg = state_sigma(cl, e_ms, E, p.P, p.lc);
    const float upv = pow2f_sat(sg + ev), upz = pow2f_sat(sg);
    const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
    constexpr int DQ = sum_quads(DV);
    float4 *dst = reinterpret_cast<float4 *>(p.part) + (part_base + cl) * DQ * kL + t;
    float den = 0.f;
    {
        uint32_t rz[16];
        tc_ld16(tm + C::COL_R + nl * DV, rz);
        tc_wait_ld();
#pragma unroll
        for (int s = 0; s < NL; ++s)
            if (s < nl) den = fmaf(qv[s], __uint_as_float(rz[s]), den);
    }
    // 32 columns at a time (16 when d_V = 16): one load per slot, combined, then the columns'
    // quads added (or stored)
    constexpr int GW = DV >= 32 ? 32 : 16;
#pragma unroll 1
    for (int g = 0; g < DV / GW; ++g) {
        float acc[GW];
#pragma unroll
        for (int i = 0; i < GW; ++i) acc[i] = 0.f;
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            if (s < nl) {
                uint32_t ra[GW];
                if constexpr (GW == 32) tc_ld32(tm + C::COL_R + s * DV + GW * g, ra);
                else tc_ld16(tm + C::COL_R + s * DV + GW * g, ra);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < GW; ++i) acc[i] = fmaf(qv[s], __uint_as_float(ra[i]), acc[i]);
            }
        }
        if (g == DV / GW - 1) {   // every column read: the next readout may overwrite R
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(rf_bar);
        }
        if (valid) {
#pragma unroll
            for (int i4 = 0; i4 < GW / 4; ++i4) {
                const float4 val = make_float4(acc[4 * i4] * upv, acc[4 * i4 + 1] * upv, acc[4 * i4 + 2] * upv,
                                               acc[4 * i4 + 3] * upv);
                if (p.red_atomic) atomicAdd(dst + (GW / 4 * g + i4) * kL, val);
                else dst[(GW / 4 * g + i4) * kL] = val;
            }
        }
    }
    if (valid) {   // the Z column opens the last quad (its other columns are padding)
        const float4 val = make_float4(den * upz, 0.f, 0.f, 0.f);
        if (p.red_atomic) atomicAdd(dst + (DV / 4) * kL, val);
        else dst[(DV / 4) * kL] = val;
    }
}

// Gradient scan (JAC) drain: R of chunk cl holds, per slot s (index i_s) and column j,
// sum_pairs P2(a_t) B[pair, (s, j)]; the token's output for slot s is its contraction with
// the token's multipliers m_t (fp32, true frame): sum_{j < d_V} m_t[j] R[t, (s, j)] +
// m_t[d_V] R[t, Z_s], added into sums[bh][i_s][token].  Arrives on rf_bar once every column
// is read.
template <int DK, int DV>
__device__ __forceinline__ void q_drain_jac(const ScanParams &p, int64_t bh, int nl, int E, int ek, int ev, int cl,
                                            int t, int lane, uint32_t tm, uint32_t rf_bar, const int *sl) {
    using C = Cfg<DK, DV>;
    constexpr int NL = C::NL;
    tc_after();
    const int sg = jac_sigma(cl, E, ek, p.P, p.lc);
    const float upv = pow2f_sat(sg + ev), upz = pow2f_sat(sg + (p.zscaled ? ev : 0));
    const int64_t tok = (int64_t)(p.c0 + cl) * kL + t;
    const bool valid = tok < p.N;
    // 32 consecutive tokens read 512 contiguous bytes per quad
    const float4 *m4 = reinterpret_cast<const float4 *>(p.mult) + ((int64_t)bh * p.nch + p.c0 + cl) * p.mult_quads * kL + t;
    float acc[NL], accz[NL];
    {
        uint32_t rz[16];
        tc_ld16(tm + C::COL_R + nl * DV, rz);
        tc_wait_ld();
        const float mz = valid ? __ldg(m4 + (DV / 4) * kL).x : 0.f;
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            acc[s] = 0.f;
            accz[s] = mz * __uint_as_float(rz[s]);
        }
    }
    constexpr int GW = DV >= 32 ? 32 : 16;
#pragma unroll 1
    for (int g = 0; g < DV / GW; ++g) {
        float mv[GW];
#pragma unroll
        for (int i4 = 0; i4 < GW / 4; ++i4) {
            const float4 x = valid ? __ldg(m4 + (GW / 4 * g + i4) * kL) : make_float4(0.f, 0.f, 0.f, 0.f);
            mv[4 * i4] = x.x;
            mv[4 * i4 + 1] = x.y;
            mv[4 * i4 + 2] = x.z;
            mv[4 * i4 + 3] = x.w;
        }
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            if (s < nl) {
                uint32_t ra[GW];
                if constexpr (GW == 32) tc_ld32(tm + C::COL_R + s * DV + GW * g, ra);
                else tc_ld16(tm + C::COL_R + s * DV + GW * g, ra);
                tc_wait_ld();
                float a = acc[s];
#pragma unroll
                for (int i = 0; i < GW; ++i) a = fmaf(mv[i], __uint_as_float(ra[i]), a);
                acc[s] = a;
            }
        }
        if (g == DV / GW - 1) {   // every column read: the next readout may overwrite R
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(rf_bar);
        }
    }
    if (valid) {
#pragma unroll
        for (int s = 0; s < NL; ++s)
            if (s < nl) atomicAdd(p.sums_jac + (bh * DK + sl[s]) * p.N + tok, fmaf(acc[s], upv, accz[s] * upz));
    }
}

// conversion: 16 fp32 state columns of one slot's V part -> 8 packed fp16 words, scaled by f.
__device__ __forceinline__ void conv_v(const uint32_t (&rr)[16], float f, uint32_t (&hp)[8]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const __half2 h = __floats2half2_rn(__uint_as_float(rr[2 * w]) * f, __uint_as_float(rr[2 * w + 1]) * f);
        hp[w] = *reinterpret_cast<const uint32_t *>(&h);
    }
}
// conversion: the Z group (column s = Z of slot s, s < nl; padding after) -> 8 packed words.
template <int NL>
__device__ __forceinline__ void conv_z(const uint32_t (&rr)[16], int nl, const float (&sc)[NL], uint32_t (&hp)[8]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const int s0 = 2 * w, s1 = 2 * w + 1;
        const float f0 = s0 < nl ? sel(sc, s0) : 0.f;
        const float f1 = s1 < nl ? sel(sc, s1) : 0.f;
        const __half2 h = __floats2half2_rn(__uint_as_float(rr[2 * w]) * f0, __uint_as_float(rr[2 * w + 1]) * f1);
        hp[w] = *reinterpret_cast<const uint32_t *>(&h);
    }
}

// JAC = false: the prefill scan (features of degree < P, den from the Z columns).
// JAC = true: a gradient scan of the backward pass: pair rows of degree <= P - 2 (the
// derivative T_{P-1} of the Taylor weight), slots index the key-side vector as a value
// dimension, the Z columns take zval16 (or 1), and the drain contracts each slot's
// columns with the token's multipliers (q_drain_jac).  Fresh state only.
template <int DK, int DV, bool JAC = false>
__global__ void __launch_bounds__(kScanThreads, 1) tc_scan_kernel(const ScanParams p) {
    using C = Cfg<DK, DV>;
    constexpr int NL = C::NL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto BAR = [bar0](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *sl = reinterpret_cast<int *>(smem + C::OFF_L);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // head-major order (a head's units, largest first, then the next head's): the CTAs
    // resident at a time share one or two heads' token rows and sums in L2
    const int64_t bh = blockIdx.x / p.G;
    const int u = blockIdx.x % p.G;
    const int ktile = p.unit_k[u];
    const int nl = p.unit_nl[u];
    const int NU = (nl * (DV + 1) + 15) / 16 * 16;   // MMA N of this unit
    const HeadExp he = head_exps(p.stats + bh * 4);
    const int E = he.eq + he.ek;
    const float ms = p.stats[bh * 4 + 3];
    const int e_ms = (p.load_state && ms > 0.f)
                         ? scale_exp(ms) + ((p.P - 1) * -he.ek > 0 ? (p.P - 1) * -he.ek : 0) + (he.ev < 0 ? -he.ev : 0)
                         : -1000;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::N_BAR; ++i) {
            uint32_t cnt = 1;
            if (i == C::B_AKF || i == C::B_SR || i == C::B_BSF || i == C::B_BSF + 1 || i == C::B_AQF ||
                i == C::B_RF)
                cnt = 4;

            mbar_init(BAR(i), cnt);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x < NL) sl[threadIdx.x] = p.unit_l[u * NL + threadIdx.x];
    if (warp == kWarpI) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_before();
    }
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter W{abort_flag, p.flags + kFlagTimeout, p.wait_ns};

    if (warp == kWarpI) {
        // ------------------------------------------------ MMA issue (one thread, both streams in chunk order)
        if (lane == 0) {
            const uint32_t id_u = idesc_f16(128, NU, 1, 1);   // A, B MN-major in shared memory
            const uint32_t id_r = idesc_f16(128, NU, 0, 1);   // A in TMEM, B MN-major
            const uint32_t wb = sb + C::OFF_W;
            bool ok = true;
            for (int cl = 0; cl < p.nc && ok; ++cl) {
                const int b = cl & 1;
                ok = W.wait(BAR(C::B_AKF), cl & 1) && W.wait(BAR(C::B_SR), cl & 1);
                if (!ok) break;
                tc_after();
                // update: [S|Z] (+)= P2(K)^T [128 pairs x 128 t] . W [128 t x NU]
                const uint32_t ak = sb + C::OFF_AK + b * C::AK_BYTES;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(tmem + C::COL_S, sdesc(ak + ks * 2048, 16384, 1024, 2),
                           sdesc(wb + ks * 2 * C::LBO, C::LBO, 128, 0), id_u,
                           (p.load_state || cl > 0 || ks > 0) ? 1u : 0u);
                tc_commit(BAR(C::B_AKE + b));
                tc_commit(BAR(C::B_UD));
                ok = W.wait(BAR(C::B_AQF), cl & 1) && W.wait(BAR(C::B_BSF + b), (cl >> 1) & 1) &&
                     (cl == 0 || W.wait(BAR(C::B_RF), (cl - 1) & 1));
                if (!ok) break;
                tc_after();
                // readout: R = P2(Q) [128 t x 128 pairs] . B [128 pairs x NU]
                const uint32_t bs = sb + C::OFF_BS + b * C::W_BYTES;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma_ta(tmem + C::COL_R, tmem + C::COL_AQ + ks * 8, sdesc(bs + ks * 2 * C::LBO, C::LBO, 128, 0),
                              id_r, ks > 0 ? 1u : 0u);
                tc_commit(BAR(C::B_BSE + b));
                tc_commit(BAR(C::B_RD));
            }
            // every issued MMA completes before TMEM is released
            tc_commit(BAR(C::B_FIN));
            W.drain(BAR(C::B_FIN), 0);
        }
    } else if (warp < kWarpQ0) {
        // ------------------------------------------------ k side: P2(k) and W per chunk
        const int t = (warp - kWarpK0) * 32 + lane;
        // Per chunk: P2(k) from the prefetched k row once its buffer is free, then the v row is
        // requested and lands while the update of the previous chunk completes, then W, then
        // the next chunk's k row is requested.
        uint32_t x[C::XW], kl[NL];   // this chunk's k row and k~_l (half2 broadcasts), prefetched
        if (p.nc > 0) fetch_row<DK>(p.k16, p, bh, sl, 0, t, x, kl);
        bool ok = true;
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int b = cl & 1;
            // P2(k) into its double buffer once the update of chunk cl-2 has read it
            if (cl >= 2 && !(ok = W.wait(BAR(C::B_AKE + b), ((cl >> 1) - 1) & 1))) break;
            p2k_dispatch<DK>(ktile, x, smem + C::OFF_AK + b * C::AK_BYTES, t,
                             std::make_integer_sequence<int, C::NPT>{});
            uint4 vr[DV / 8];
            {
                const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
                const uint4 *vcr = chunk_rows<DV>(p.v16, bh, p.nch, p.c0 + cl);
#pragma unroll
                for (int i = 0; i < DV / 8; ++i) vr[i] = valid ? __ldg(vcr + i * 128 + t) : make_uint4(0, 0, 0, 0);
            }
            // W (single buffer) once the update of chunk cl-1 has completed
            if (cl >= 1 && !(ok = W.wait(BAR(C::B_UD), (cl - 1) & 1))) break;
            // W row t: [k~_l0 v | k~_l1 v | ... | k~_l0 k~_l1 ... 0 ...] as 16-byte chunks of 8 columns
            uint8_t *wrow = smem + C::OFF_W + (t >> 3) * C::LBO + (t & 7) * 16;
#pragma unroll
            for (int s = 0; s < NL; ++s) {
                if (s < nl) {
#pragma unroll
                    for (int i = 0; i < DV / 8; ++i)
                        *reinterpret_cast<uint4 *>(wrow + (s * (DV / 8) + i) * 128) = hmul2x4(vr[i], kl[s]);
                }
            }
            uint32_t zv = 0x3C003C00u;   // the Z columns' factor: 1, or the token's value (JAC)
            if constexpr (JAC) {
                if (p.zval16) {
                    const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
                    const uint32_t h =
                        valid ? (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.zval16) +
                                                ((int64_t)bh * p.nch + p.c0 + cl) * kL + t)
                              : 0u;
                    zv = h | (h << 16);
                }
            }
            for (int z8 = nl * (DV / 8); z8 < NU / 8; ++z8) {
                uint32_t w4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int s0 = z8 * 8 - nl * DV + 2 * j, s1 = s0 + 1;
                    uint32_t lo = 0, hi = 0;
#pragma unroll
                    for (int s = 0; s < NL; ++s) {
                        const uint32_t kz = JAC ? hmul2u(kl[s], zv) : kl[s];
                        lo = (s == s0 && s < nl) ? (kz & 0xFFFFu) : lo;
                        hi = (s == s1 && s < nl) ? (kz & 0xFFFFu) : hi;
                    }
                    w4[j] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4 *>(wrow + z8 * 128) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async();
            __syncwarp();
            // test hook: one producer signal withheld, so the issuer's wait expires
            if (lane == 0 && !(warp == kWarpK0 && p.c0 + cl == p.stall_chunk)) mbar_arrive(BAR(C::B_AKF));
            // the next chunk's k row, requested after the signal: its slot values are used as
            // soon as they land, so the load latency would otherwise sit before the update
            if (cl + 1 < p.nc) fetch_row<DK>(p.k16, p, bh, sl, cl + 1, t, x, kl);
        }
    } else if (warp < kWarpC0) {
        // ------------------------------------------------ q side: P2(q) operand, readout drain
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;               // token row of the chunk = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int64_t part_base = p.red_atomic ? (int64_t)bh * p.nc : ((int64_t)bh * p.G + u) * p.nc;
        uint32_t pq[64], xl[NL];
        float qlp[NL];
        bool ok = true;
        if (p.nc > 0) {
            uint32_t x[C::XW];
            fetch_row<DK>(p.q16, p, bh, sl, 0, t, x, xl);
            p2q_dispatch<DK, 0, C::NPT>(ktile, x, pq);
        }
        for (int cl = 0; cl < p.nc; ++cl) {
            if (cl > 0 && !(ok = W.wait(BAR(C::B_RD), (cl - 1) & 1))) break;
            tc_after();
#pragma unroll
            for (int i = 0; i < 4; ++i) tc_st16(tmem + lane_off + C::COL_AQ + 16 * i, pq + 16 * i);
            tc_wait_st();
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_AQF));
            if (cl > 0) {
                if constexpr (JAC)
                    q_drain_jac<DK, DV>(p, bh, nl, E, he.ek, he.ev, cl - 1, t, lane, tmem + lane_off, BAR(C::B_RF), sl);
                else
                    q_drain<DK, DV>(p, bh, part_base, nl, e_ms, E, he.ev, cl - 1, t, lane, tmem + lane_off,
                                    BAR(C::B_RF), qlp);
            }
#pragma unroll
            for (int s = 0; s < NL; ++s) qlp[s] = h_lo(xl[s]);
            {   // the next chunk's operand (its row is read after the drain, which needs the
                // registers; the load overlaps the readout now running).  Unconditional, so that
                // pq is provably dead during the drain (the last iteration builds an unused one).
                uint32_t x[C::XW];
                fetch_row<DK>(p.q16, p, bh, sl, cl + 1 < p.nc ? cl + 1 : cl, t, x, xl);
                p2q_dispatch<DK, 0, C::NPT>(ktile, x, pq);
            }
        }
        if (ok && p.nc > 0 && W.wait(BAR(C::B_RD), (p.nc - 1) & 1)) {
            if constexpr (JAC)
                q_drain_jac<DK, DV>(p, bh, nl, E, he.ek, he.ev, p.nc - 1, t, lane, tmem + lane_off, BAR(C::B_RF), sl);
            else
                q_drain<DK, DV>(p, bh, part_base, nl, e_ms, E, he.ev, p.nc - 1, t, lane, tmem + lane_off, BAR(C::B_RF),
                                qlp);
        }
        tc_before();
    } else {
        // ------------------------------------------------ state -> fp16 readout operand
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // pair row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t pw = p.pairs[ktile * 128 + r];
        const int ppair = ((int)(pw & 255u) < DK) + ((int)(pw >> 8) < DK);
        float cf[NL];
        int pe[NL], fi[NL], dg[NL];
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            const int64_t at = ((int64_t)u * NL + s) * 128 + r;
            cf[s] = s < nl ? p.unit_coef[at] : 0.f;
            fi[s] = s < nl ? p.unit_fidx[at] : -1;
            dg[s] = ppair + (sl[s] < DK);               // degree of feature (pair r, l_s)
            // prefill: the feature's degree on both sides; gradient scan: the pair's degree on
            // both sides, the slot on the key side only
            pe[s] = JAC ? (dg[s] - 1) * E + he.ek : dg[s] * E;
            for (int i = 0; i < dg[s]; ++i) cf[s] *= p.inv_c;   // alpha_p = 1 / (p! c^p)
        }
        constexpr int NG = C::NG;
        const int ngu = NU / 16;
        const int ngv = nl * DV / 16;   // groups of V columns; group ngv holds the Z columns (and padding)
        bool ok = true;
        if (p.load_state) {   // incoming state -> TMEM (prescaled frame)
            // a V group is 16 contiguous columns of one feature's S row (four 16-byte loads);
            // the Z group gathers one Z value per slot
#pragma unroll 1
            for (int g = 0; g < NG; ++g) {
                if (g < ngu) {
                    uint32_t v16[16];
                    if (16 * g < nl * DV) {
                        const int sv = (16 * g) / DV;
                        const int f = seli(fi, sv);
                        const float sc = pow2f_sat(-(seli(dg, sv) * he.ek + he.ev));
                        const float4 *src = reinterpret_cast<const float4 *>(p.S + (bh * p.F + (f >= 0 ? f : 0)) * DV +
                                                                             (16 * g) % DV);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float4 x = f >= 0 ? src[j] : make_float4(0.f, 0.f, 0.f, 0.f);
                            v16[4 * j] = __float_as_uint(x.x * sc);
                            v16[4 * j + 1] = __float_as_uint(x.y * sc);
                            v16[4 * j + 2] = __float_as_uint(x.z * sc);
                            v16[4 * j + 3] = __float_as_uint(x.w * sc);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int sz = 16 * g + i - nl * DV;
                            float x = 0.f;
                            if (sz < nl) {
                                const int f = seli(fi, sz);
                                if (f >= 0) x = p.Z[bh * p.F + f] * pow2f_sat(-(seli(dg, sz) * he.ek));
                            }
                            v16[i] = __float_as_uint(x);
                        }
                    }
                    tc_st16(tmem + lane_off + C::COL_S + 16 * g, v16);
                }
            }
            tc_wait_st();
        }
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int b = cl & 1;
            if (cl > 0 && !(ok = W.wait(BAR(C::B_UD), (cl - 1) & 1))) break;
            // B double buffer: the readout of chunk cl-2 has read it
            if (cl >= 2 && !(ok = W.wait(BAR(C::B_BSE + b), ((cl >> 1) - 1) & 1))) break;
            tc_after();
            const int sg = JAC ? jac_sigma(cl, E, he.ek, p.P, p.lc) : state_sigma(cl, e_ms, E, p.P, p.lc);
            float sc[NL];
#pragma unroll
            for (int s = 0; s < NL; ++s) sc[s] = cf[s] * pow2f_sat(pe[s] - sg);
            uint8_t *bs = smem + C::OFF_BS + b * C::W_BYTES + (r >> 3) * C::LBO + (r & 7) * 16;
            if (p.load_state || cl > 0) {
                // the V groups two at a time, the loads of the next pair in flight while this
                // pair converts; then the Z group, the last state read
                uint32_t ra[16], rb[16];
                tc_ld16(tmem + lane_off + C::COL_S, ra);
                if (1 < ngv) tc_ld16(tmem + lane_off + C::COL_S + 16, rb);
                tc_wait_ld();
#pragma unroll 1
                for (int g = 0; g < ngv; g += 2) {
                    uint32_t ha[8], hb[8];
                    conv_v(ra, sel(sc, (16 * g) / DV), ha);
                    if (g + 1 < ngv) conv_v(rb, sel(sc, (16 * g + 16) / DV), hb);
                    if (g + 2 < ngv) tc_ld16(tmem + lane_off + C::COL_S + 16 * (g + 2), ra);
                    if (g + 3 < ngv) tc_ld16(tmem + lane_off + C::COL_S + 16 * (g + 3), rb);
                    *reinterpret_cast<uint4 *>(bs + (2 * g) * 128) = make_uint4(ha[0], ha[1], ha[2], ha[3]);
                    *reinterpret_cast<uint4 *>(bs + (2 * g + 1) * 128) = make_uint4(ha[4], ha[5], ha[6], ha[7]);
                    if (g + 1 < ngv) {
                        *reinterpret_cast<uint4 *>(bs + (2 * g + 2) * 128) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
                        *reinterpret_cast<uint4 *>(bs + (2 * g + 3) * 128) = make_uint4(hb[4], hb[5], hb[6], hb[7]);
                    }
                    if (g + 2 < ngv) tc_wait_ld();
                }
                tc_ld16(tmem + lane_off + C::COL_S + 16 * ngv, ra);
                tc_wait_ld();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_SR));   // state read: the update may proceed
                uint32_t hz[8];
                conv_z<NL>(ra, nl, sc, hz);
                *reinterpret_cast<uint4 *>(bs + (2 * ngv) * 128) = make_uint4(hz[0], hz[1], hz[2], hz[3]);
                *reinterpret_cast<uint4 *>(bs + (2 * ngv + 1) * 128) = make_uint4(hz[4], hz[5], hz[6], hz[7]);
            } else {   // fresh state before the first chunk: the operand is zero
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_SR));
#pragma unroll 1
                for (int g = 0; g < ngu; ++g) {
                    *reinterpret_cast<uint4 *>(bs + (2 * g) * 128) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(bs + (2 * g + 1) * 128) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_BSF + b));
        }
        if (ok && p.store_state && p.nc > 0 && W.wait(BAR(C::B_UD), (p.nc - 1) & 1)) {
            tc_after();
#pragma unroll 1
            for (int g = 0; g < NG; ++g) {
                if (g < ngu) {
                    uint32_t rr[16];
                    tc_ld16(tmem + lane_off + C::COL_S + 16 * g, rr);
                    tc_wait_ld();
                    if (16 * g < nl * DV) {   // 16 contiguous columns of one S row
                        const int sv = (16 * g) / DV;
                        const int f = seli(fi, sv);
                        const float sc = pow2f_sat(seli(dg, sv) * he.ek + he.ev);
                        if (f >= 0) {
                            float4 *dst = reinterpret_cast<float4 *>(p.S + (bh * p.F + f) * DV + (16 * g) % DV);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                dst[j] = make_float4(__uint_as_float(rr[4 * j]) * sc, __uint_as_float(rr[4 * j + 1]) * sc,
                                                     __uint_as_float(rr[4 * j + 2]) * sc,
                                                     __uint_as_float(rr[4 * j + 3]) * sc);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int sz = 16 * g + i - nl * DV;
                            if (sz < nl) {
                                const int f = seli(fi, sz);
                                if (f >= 0)
                                    p.Z[bh * p.F + f] = __uint_as_float(rr[i]) * pow2f_sat(seli(dg, sz) * he.ek);
                            }
                        }
                    }
                }
            }
        }
        tc_before();
    }

    __syncthreads();
    if (warp == kWarpI) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

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
// One CTA (4 warps, thread = token row) per (head, chunk).
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
    static constexpr int TCOLS = 128 + NV <= 256 ? 256 : 512;
    // with all 512 TMEM columns, one CTA per SM (a shared-memory request above half the SM)
    static constexpr int SMEM0 = OFF_BAR + 64 + 1024;
    static constexpr int SMEM = TCOLS == 512 && SMEM0 < 120 * 1024 ? 120 * 1024 : SMEM0;
    static_assert(2 * KB * 16384 >= 32768, "W_lo");
    static_assert(SMEM <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(128)
tc_finish_kernel(const __half *__restrict__ q16, const __half *__restrict__ k16, const __half *__restrict__ v16,
                 const float *__restrict__ stats, const float *__restrict__ red, float *__restrict__ out,
                 float *__restrict__ den_out, int c0, int nc, int nch, int64_t N, int P, float inv_c, int *flags,
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
    for (int e = tid; e < kL * (DK / 8); e += 128) {   // Q and K: DK/8 pieces of 8 d per row
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
    for (int e = tid; e < kL * (NV / 8); e += 128) {   // [V'|1]: row s, 8 n per 16-byte core row
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
    const int t = tid;                               // token row = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
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
    const float down = pow2f_sat(-e_t);
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
            if (den_out && t < nt) den_out[bh * N + t0 + t] = den;   // kept for the backward pass
        }
#pragma unroll
        for (int c16 = 0; c16 < DV / 16; ++c16) {
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
        float4 *o4 = reinterpret_cast<float4 *>(out + (bh * N + t0) * DV);
        for (int e = tid; e < nt * (DV / 4); e += 128) {
            const int r = e / (DV / 4), c4 = e % (DV / 4);
            o4[e] = *reinterpret_cast<const float4 *>(stg + r * F::STG + 4 * c4);
        }
    }
    if (warp == 0) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(F::TCOLS) : "memory");
    }
}

// ------------------------------------------------------------------ host ----

// Unit plan: which (pair tile, l values) each CTA owns, and per (unit, slot, row)
// the basis index and C/p! of feature (a, b, l), or -1 / 0 where the row is no
// feature (b > l, degree >= P, or a padding pair).
struct UnitPlan {
    int D = 0, P = 0, NL = 0, NPT = 0, G = 0;
    std::vector<uint16_t> pairs;       // [NPT*128]
    std::vector<int32_t> unit_k, unit_nl, unit_l;   // [G], [G], [G*NL]
    std::vector<float> coef;           // [G*NL*128]
    std::vector<int32_t> fidx;         // [G*NL*128]
    size_t off_k = 0, off_nl = 0, off_l = 0, off_coef = 0, off_fidx = 0, bytes = 0;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// floor(log2 c), c = sqrt(d_K): the largest e with 2^(2e) <= d_K.
int floor_log2_c(int d_K) {
    int e = 0;
    while ((int64_t)1 << (2 * (e + 1)) <= d_K) ++e;
    return e;
}

bool build_unit_plan(int D, int P, int NL, UnitPlan &up) {
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
    up.NL = NL;
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
        for (size_t s = 0; s < ls.size(); s += NL) {
            Unit u{k, 0, {}};
            for (size_t j = s; j < ls.size() && j < s + NL; ++j) u.l[u.nl++] = ls[j];
            units.push_back(u);
        }
    }
    std::stable_sort(units.begin(), units.end(), [](const Unit &x, const Unit &y) { return x.nl > y.nl; });
    up.G = (int)units.size();
    up.unit_k.resize(up.G);
    up.unit_nl.resize(up.G);
    up.unit_l.assign((size_t)up.G * NL, D);
    up.coef.assign((size_t)up.G * NL * 128, 0.f);
    up.fidx.assign((size_t)up.G * NL * 128, -1);
    for (int g = 0; g < up.G; ++g) {
        const Unit &u = units[g];
        up.unit_k[g] = u.k;
        up.unit_nl[g] = u.nl;
        for (int j = 0; j < u.nl; ++j) {
            const int l = u.l[j];
            up.unit_l[(size_t)g * NL + j] = l;
            for (int r = 0; r < 128; ++r) {
                const int i = u.k * 128 + r;
                if (i >= npair || pb[i] > l) continue;
                const int p = (pa[i] < D) + (pb[i] < D) + (l < D);
                if (p >= P) continue;
                auto it = index_of.find((uint32_t)pa[i] | ((uint32_t)pb[i] << 8) | ((uint32_t)l << 16));
                if (it == index_of.end()) return false;
                const size_t at = ((size_t)g * NL + j) * 128 + r;
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
    up.off_coef = up.off_l + align256((size_t)up.G * NL * 4);
    up.off_fidx = up.off_coef + align256(up.coef.size() * 4);
    up.bytes = up.off_fidx + align256(up.fidx.size() * 4);
    return true;
}

std::mutex g_plan_mu;
std::map<std::tuple<int, int, int>, UnitPlan> g_plans;

const UnitPlan *unit_plan(int D, int P, int NL) {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    const auto key = std::make_tuple(D, P, NL);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) return &it->second;
    UnitPlan up;
    if (!build_unit_plan(D, P, NL, up)) return nullptr;
    return &g_plans.emplace(key, std::move(up)).first->second;
}

// Workspace: per-head maxima, the prescaled fp16 rows, the summed readouts of a
// segment (and, in the fixed-order mode only, the per-unit partials), and the
// state between segments when the caller keeps none.  The device-buffer path
// runs as one segment in the default mode; the host-buffer path splits the
// sequence so that copies overlap the kernels; the fixed-order mode splits it
// to bound the partial buffer.
struct Plan {
    const UnitPlan *up = nullptr;
    int G = 1, nchunks = 0, nc_seg = 0, nseg = 0;   // nc_seg: chunks of the longest segment
    // host-buffer path: segment starts (chunks) of a non-uniform split, seg_c0[nseg] = nchunks
    bool profiled = false;
    int seg_c0[kHostSegments + 1] = {};
    size_t off_stats = 0, off_q16 = 0, off_k16 = 0, off_v16 = 0, off_red = 0, off_part = 0, off_state = 0,
           total = 0;
};

template <int DK, int DV>
bool make_plan(int BH, int64_t N, int64_t F, int P, bool need_state, int min_segments, bool deterministic,
               Plan &pl) {
    using C = Cfg<DK, DV>;
    const UnitPlan *up = unit_plan(DK, P, C::NL);
    if (!up) return false;
    pl.up = up;
    pl.G = up->G;
    pl.nchunks = (int)((N + kL - 1) / kL);
    int64_t nseg = min_segments;
    if (deterministic) {
        const size_t per_chunk = (size_t)BH * pl.G * sum_quads(DV) * kL * 16;
        int64_t seg = (int64_t)(kPartialBudget / per_chunk);
        if (seg < 1) seg = 1;
        const int64_t need = (pl.nchunks + seg - 1) / seg;
        if (need > nseg) nseg = need;
    }
    if (nseg > pl.nchunks) nseg = pl.nchunks;
    if (nseg < 1) nseg = 1;
    pl.nc_seg = (int)((pl.nchunks + nseg - 1) / nseg);
    pl.nseg = (pl.nchunks + pl.nc_seg - 1) / pl.nc_seg;
    if (!deterministic && min_segments == kHostSegments && pl.nchunks >= 16 * kHostSegments) {
        // Copies pipelined with the kernels: the first segment's inputs and the last one's
        // output are exposed, so those segments are short.  A segment's inputs copy in about
        // a third of its compute time and its output in about a quarter, so each segment can
        // be a few times its predecessor while its inputs still land in time, and the last a
        // fraction of the one before it.  10 %, 20 %, 55 %, 15 % of the chunks measured best
        // of the splits tried (uniform quarters: 4 % slower end to end at 65536 tokens).
        static_assert(kHostSegments == 4, "split profile");
        const int cum[kHostSegments] = {0, 10, 30, 85};
        for (int i = 0; i < kHostSegments; ++i) pl.seg_c0[i] = (int)((int64_t)pl.nchunks * cum[i] / 100);
        pl.seg_c0[kHostSegments] = pl.nchunks;
        pl.profiled = true;
        pl.nseg = kHostSegments;
        pl.nc_seg = 0;
        for (int i = 0; i < kHostSegments; ++i)
            if (pl.seg_c0[i + 1] - pl.seg_c0[i] > pl.nc_seg) pl.nc_seg = pl.seg_c0[i + 1] - pl.seg_c0[i];
    }
    pl.off_stats = 0;
    pl.off_q16 = align256((size_t)BH * 4 * sizeof(float));
    const size_t rows = (size_t)BH * pl.nchunks * kL;   // whole chunks, chunk-interleaved
    pl.off_k16 = pl.off_q16 + align256(rows * DK * 2);
    pl.off_v16 = pl.off_k16 + align256(rows * DK * 2);
    pl.off_red = pl.off_v16 + align256(rows * DV * 2);
    pl.off_part = pl.off_red + align256((size_t)BH * sum_quads(DV) * kL * 16 * pl.nc_seg);
    pl.off_state = pl.off_part +
                   (deterministic ? align256((size_t)BH * pl.G * sum_quads(DV) * kL * 16 * pl.nc_seg) : 0);
    pl.total = pl.off_state + (need_state && pl.nseg > 1 ? align256((size_t)BH * F * (DV + 1) * sizeof(float)) : 0);
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
    const bool det = g_opt_deterministic != 0;
    Plan pl;
    if (!make_plan<DK, DV>(BH, N, F, basis.P, own_state, min_seg, det, pl)) return cudaErrorInvalidValue;
    if (ws_bytes < pl.total) return cudaErrorInvalidValue;
    const UnitPlan &up = *pl.up;
    cudaError_t e = cudaSuccess;
    const uint8_t *tab = (const uint8_t *)device_table(
        ((uint64_t)DK << 32) | ((uint64_t)basis.P << 16) | (uint64_t)up.NL | (uint64_t(1) << 60), up.bytes,
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
    __half *q16 = (__half *)(w + pl.off_q16), *k16 = (__half *)(w + pl.off_k16), *v16 = (__half *)(w + pl.off_v16);
    float *red = (float *)(w + pl.off_red);
    float *part = (float *)(w + pl.off_part);
    const int nseg = pl.nseg;
    if (own_state && nseg > 1) {
        S = (float *)(w + pl.off_state);
        Z = S + (size_t)BH * F * DV;
    }
    const float inv_c = 1.0f / sqrtf((float)DK);
    const auto *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k, *vb = (const __nv_bfloat16 *)v;

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
        const int c0s = pl.profiled ? pl.seg_c0[s] : s * pl.nc_seg;
        const int ncs = pl.profiled ? pl.seg_c0[s + 1] - c0s
                                    : ((pl.nchunks - c0s < pl.nc_seg) ? pl.nchunks - c0s : pl.nc_seg);
        const int64_t tok0 = (int64_t)c0s * kL, tok1 = (int64_t)(c0s + ncs) * kL < N ? (int64_t)(c0s + ncs) * kL : N;
        if (io) {   // this segment's inputs: host -> device on the copy stream, compute waits for them
            cudaEvent_t ev;
            if ((e = copy_rows((void *)q, io->q, BH, N, tok0, tok1, DK, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = copy_rows((void *)k, io->k, BH, N, tok0, tok1, DK, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = copy_rows((void *)v, io->v, BH, N, tok0, tok1, DV, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = new_event(&ev)) || (e = cudaEventRecord(ev, io->h2d)) || (e = cudaStreamWaitEvent(stream, ev, 0)))
                return e;
        }
        const bool load_state = (s > 0 || state_in);
        {   // this segment's maxima, prescaled rows and incoming-state bound
            if ((e = cudaMemsetAsync(stats, 0, (size_t)BH * 4 * sizeof(float), stream)) != cudaSuccess) return e;
            const int64_t ntok = tok1 - tok0;
            int bx = (int)((ntok * (DK / 8) + 255) / 256);
            const int bmax = (148 * 8 + BH - 1) / BH;
            if (bx > bmax) bx = bmax;
            if (bx < 1) bx = 1;
            launch_begin(kTcPrep, stream);
            tc_stats_kernel<DK, DV><<<(unsigned)((int64_t)bx * BH), 256, 0, stream>>>(qb, kb, vb, stats, N, tok0,
                                                                                    tok1, bx);
            if ((e = cudaGetLastError()) == cudaSuccess) {
                const int64_t nwork = (int64_t)BH * ntok;   // one thread per token row
                const int pgrid = (int)((nwork + 255) / 256 < 148 * 16 ? (nwork + 255) / 256 : 148 * 16);
                tc_prep_kernel<DK, DV><<<pgrid, 256, 0, stream>>>(qb, kb, vb, stats, q16, k16, v16, BH, N, tok0, tok1,
                                                                   pl.nchunks, flags);
            }
            launch_end(kTcPrep, stream);
            if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
            if (load_state) {
                tc_state_stats_kernel<<<dim3(BH, 8), 256, 0, stream>>>(S, Z, stats, F, DV);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
        }
        ScanParams sp;
        sp.q16 = q16;
        sp.k16 = k16;
        sp.v16 = v16;
        sp.stats = stats;
        sp.pairs = (const uint16_t *)tab;
        sp.unit_k = (const int32_t *)(tab + up.off_k);
        sp.unit_nl = (const int32_t *)(tab + up.off_nl);
        sp.unit_l = (const int32_t *)(tab + up.off_l);
        sp.unit_coef = (const float *)(tab + up.off_coef);
        sp.unit_fidx = (const int32_t *)(tab + up.off_fidx);
        sp.S = S;
        sp.Z = Z;
        if (!det && (e = cudaMemsetAsync(red, 0, (size_t)BH * ncs * sum_quads(DV) * kL * 16, stream)) !=
                        cudaSuccess)
            return e;
        sp.part = det ? part : red;
        sp.red_atomic = det ? 0 : 1;
        sp.flags = flags;
        sp.F = F;
        sp.N = N;
        sp.BH = BH;
        sp.G = pl.G;
        sp.c0 = c0s;
        sp.nc = ncs;
        sp.nch = pl.nchunks;
        sp.P = basis.P;
        sp.load_state = load_state ? 1 : 0;
        sp.store_state = (s + 1 < nseg || !own_state) ? 1 : 0;
        sp.stall_chunk = stall;
        sp.inv_c = inv_c;
        sp.lc = floor_log2_c(DK);
        sp.wait_ns = wait_ns;
        launch_begin(kTcScan, stream);
        tc_scan_kernel<DK, DV><<<BH * pl.G, kScanThreads, C::SMEM, stream>>>(sp);
        launch_end(kTcScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (det) {   // the units' partials summed in a fixed order
            const int64_t rwork = (int64_t)BH * ncs * sum_quads(DV) * kL;
            launch_begin(kTcReduce, stream);
            tc_reduce_kernel<DV><<<(int)((rwork + 255) / 256 < 148 * 32 ? (rwork + 255) / 256 : 148 * 32), 256, 0,
                                   stream>>>((const float4 *)part, (float4 *)red, BH, pl.G, ncs);
            launch_end(kTcReduce, stream);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        launch_begin(kTcFinish, stream);
        tc_finish_kernel<DK, DV><<<(int)((int64_t)BH * ncs), 128, FinCfg<DK, DV>::SMEM, stream>>>(
            q16, k16, v16, stats, red, out, den_out, c0s, ncs, pl.nchunks, N, basis.P, inv_c, flags, wait_ns);
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

// Non-template entry points of one (d_K, d_V) instance (declared in prefill_tc_shapes.h).
#define SATA_TC_DEFINE(a, b)                                                                                  \
    size_t tc_workspace_##a##_##b(int BH, int64_t N, int64_t F, int P, bool need_state, int min_seg, bool det) { \
        Plan pl;                                                                                              \
        return make_plan<a, b>(BH, N, F, P, need_state, min_seg, det, pl) ? pl.total : 0;                     \
    }                                                                                                         \
    cudaError_t tc_run_##a##_##b(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k,   \
                                 const void *v, float *out, float *S, float *Z, bool state_in, void *ws,       \
                                 size_t ws_bytes, int *flags, cudaStream_t stream, const HostIO *io,          \
                                 float *den_out) {                                                            \
        return run<a, b>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io, den_out);  \
    }

}  // namespace sata
