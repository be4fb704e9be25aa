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
// Files: prefill_tc_common.cuh (this: constants, parameters, PTX and operand helpers),
// prefill_tc_prep.cuh (maxima, prescaled rows), prefill_tc_scan.cuh (the scan),
// prefill_tc_finish.cuh (fixed-order reduce, intra-chunk block and division),
// prefill_tc_kernels.cuh (unit plans and the host driver), all templates over (d_K, d_V);
// the prefill_tc_*.cu files instantiate them (prefill_tc_shapes.h lists the shapes) and
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
    float *S, *Z;
    int s_ld = 0, s_off = 0;         // S rows s_ld values apart (0: DV), this call's columns from s_off                    // state in/out (true frame)
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
    // per-chunk maxima of the prescaled column values ([BH][nch], this scan's frame), or null:
    // every column value is at most 1.  With them the readout operand's bound sums the
    // maxima of the chunks so far instead of counting their tokens at the largest value (a
    // gradient scan's r can hold one token hundreds of times the others)
    const float *colmax = nullptr;
    float colmax_floor = 0.f;   // the least column maximum (1: Z columns that carry 1)
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
// |S'| < 2^e_ms + 2^e_tok with 2^e_tok > 128 cl + 1 (every prescaled feature and value is
// at most 1 in magnitude; e_ms bounds the prescaled incoming state), or, with per-chunk
// maxima m_c of the column values, 2^e_tok > 128 sum_{c < cl} m_c + 1; and a degree-p row
// carries C/p! c^-p 2^(p E) <= 2^(p (E - lc)) <= 2^max(0, (P-1)(E - lc)) (C/p! <= 1, lc =
// floor(log2 c)), so |B| < 2^15 for every row.  The bound is tight for the rows that
// reach it; a looser one would push the small rows of B into fp16's subnormal range.
__device__ __forceinline__ int tok_exp(int cl) { return 32 - __clz((uint32_t)cl * kL + 1u); }
__device__ __forceinline__ int tok_exp_sum(float cum) {   // 128 cum + 1 < 2^e (a normal float >= 1)
    return (int)((__float_as_uint(fmaf(128.f, cum, 1.f)) >> 23) & 0xFFu) - 126;
}
__device__ __forceinline__ int state_sigma_rows(int e_tok, int e_ms, int e_row) {
    const int eb = (e_ms > e_tok ? e_ms : e_tok) + 1;
    const int s = eb + e_row - 15;
    return s < -120 ? -120 : (s > 120 ? 120 : s);
}
__device__ __forceinline__ int state_sigma(int e_tok, int e_ms, int E, int P, int lc) {
    const int r = (P - 1) * (E - lc);
    return state_sigma_rows(e_tok, e_ms, r > 0 ? r : 0);
}
// The same for a gradient scan: a pair row of degree p' <= P - 2 carries
// C/p'! c^-(p'+1) 2^(p' E + e_k) <= 2^(p' (E - lc) + e_k - lc) (the slot index is a
// key-side factor only; the derivative's 1/c is in the row).
__device__ __forceinline__ int jac_sigma(int e_tok, int E, int ek, int P, int lc) {
    const int r = (P - 2) * (E - lc);
    return state_sigma_rows(e_tok, -1000, (r > 0 ? r : 0) + ek - lc);
}
// The column bound's exponent before chunk cl (cum: the maxima of chunks < cl summed in
// chunk order; every role sums them the same way, so all agree on sigma).
__device__ __forceinline__ int col_exp(const ScanParams &p, int cl, float cum) {
    return p.colmax ? tok_exp_sum(cum) : tok_exp(cl);
}
__device__ __forceinline__ float col_max(const ScanParams &p, int64_t bh, int cl) {
    return fmaxf(p.colmax[bh * p.nch + p.c0 + cl], p.colmax_floor);
}

// Non-blocking test of an mbarrier phase (the issuer polls two chains).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
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

}  // namespace
}  // namespace sata
