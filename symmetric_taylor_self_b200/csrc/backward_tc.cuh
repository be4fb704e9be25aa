// Backward pass of the prefill on tensor cores: the three gradient scans run as
// tcgen05 scans of the prefill's kind (prefill_tc_scan.cuh), the intra-chunk
// pairs in a CUDA-core finish kernel.
//
// The method's pages define no backward pass ([CC-TAYLOR] "Self-attention at
// constant cost per token via symmetry-aware Taylor approximation" expects the
// attention inside ordinary training pipelines: "Comparison with other methods",
// "Future directions").  This is the exact gradient of its forward ("Feature maps
// and linear attention"): y_t = num_t / den_t, [num_t | den_t] = sum_{s<=t} w_ts u_s,
// u_s = [v_s | 1], w_ts = T_P(x_ts), x_ts = q_t . k_s / c, T_P(x) = sum_{p<P} x^p / p!.
// With g_t = dy_t / den_t and r_t = [g_t | -(g_t . y_t)], dL/dw_ts = r_t . u_s, and
// T_P' = T_{P-1}, so
//   dq_t = 1/c sum_{s<=t} (r_t . u_s) T_{P-1}(x_ts) k_s
//   dk_s = 1/c sum_{t>=s} (r_t . u_s) T_{P-1}(x_ts) q_t
//   dv_s =     sum_{t>=s} T_P(x_ts) g_t.
// Each is a causal sum with a Taylor kernel, so each has the prefill's feature form:
//   * T_{P-1}(q.k/c) = sum over the pairs (a, b), a <= b over the padded indices, of
//     degree p' <= P - 2: C/p'! c^-p' P2(q)_(a,b) P2(k)_(a,b).  dq_t[i] is then a scan
//     whose key-side rows are P2(k_s) and whose values are k_s[i] u_s: the slots of
//     the prefill's scan index i (a value dimension here), its columns are [v | 1],
//     and the drain contracts each slot's columns with r_t (q_drain_jac).
//   * dk is the same scan on the time-reversed sequence with q and k exchanged and
//     the columns [g | -(g . y)] (Z columns from a per-token value), contracted with u.
//   * dv is the prefill scan itself on the time-reversed sequence, queries k, keys q,
//     values g; its num sums are dv (no division).
// Reversal turns the anti-causal sums into causal ones: frame token t' = N - 1 - t.
//
// Kernels: bwd_tc_r (r = [dy/den | -(dy.y)/den] and per-head maxima), bwd_tc_prep
// (prescaled fp16 rows in both orders), three tc_scan launches, bwd_tc_finish (the
// pairs inside a chunk, the 1/c scale, the reversal back).  The readouts are added
// into their sums with fp32 atomics, so the gradients are not bitwise repeatable;
// the library runs its CUDA-core gradient scans instead when the fixed-order mode
// is set.
#pragma once

#include "prefill_tc_kernels.cuh"

namespace sata {
namespace {

__host__ __device__ constexpr int bwd_rs(int DV) { return (DV + 1 + 3) / 4 * 4; }   // r, u row stride
constexpr int kRHead = 14;   // r's prescaled maximum: below 2^14 (an fp16 operand holds up to 65504)

// Unit plan of a gradient scan: per pair tile holding a pair of degree <= P - 2,
// the d_K slot indices i in groups of NL; coefficient C/p'! of the pair (0 on
// pairs of higher degree and on padding), no basis index (fresh state only).
bool build_jac_plan(int D, int P, int NL, UnitPlan &up) {
    up.D = D;
    up.P = P;
    up.NL = NL;
    const int npair = (D + 1) * (D + 2) / 2;
    up.NPT = (npair + 127) / 128;
    up.pairs.assign((size_t)up.NPT * 128, (uint16_t)(D | (D << 8)));
    std::vector<float> pc((size_t)up.NPT * 128, 0.f);
    {
        int i = 0;
        for (int b = 0; b <= D; ++b)
            for (int a = 0; a <= b; ++a, ++i) {
                up.pairs[i] = (uint16_t)(a | (b << 8));
                const int p = (a < D) + (b < D);
                if (p <= P - 2) pc[i] = (p == 2 && a == b) ? 0.5f : 1.f;   // C/p'!: 1/2 for a square
            }
    }
    std::vector<int> tiles;
    for (int k = 0; k < up.NPT; ++k) {
        bool any = false;
        for (int r = 0; r < 128; ++r) any = any || pc[(size_t)k * 128 + r] != 0.f;
        if (any) tiles.push_back(k);
    }
    const int ngroups = (D + NL - 1) / NL;
    up.G = (int)tiles.size() * ngroups;
    up.unit_k.resize(up.G);
    up.unit_nl.resize(up.G);
    up.unit_l.assign((size_t)up.G * NL, D);
    up.coef.assign((size_t)up.G * NL * 128, 0.f);
    up.fidx.assign((size_t)up.G * NL * 128, -1);
    // full groups first (the widest units are scheduled first)
    int g = 0;
    for (int pass = 0; pass < 2; ++pass)
        for (int k : tiles)
            for (int grp = 0; grp < ngroups; ++grp) {
                const int l0 = grp * NL, nl = D - l0 < NL ? D - l0 : NL;
                if ((nl == NL) != (pass == 0)) continue;
                up.unit_k[g] = k;
                up.unit_nl[g] = nl;
                for (int j = 0; j < nl; ++j) {
                    up.unit_l[(size_t)g * NL + j] = l0 + j;
                    for (int r = 0; r < 128; ++r) up.coef[((size_t)g * NL + j) * 128 + r] = pc[(size_t)k * 128 + r];
                }
                ++g;
            }
    if (g != up.G) return false;
    up.off_k = align256((size_t)up.NPT * 128 * sizeof(uint16_t));
    up.off_nl = up.off_k + align256((size_t)up.G * 4);
    up.off_l = up.off_nl + align256((size_t)up.G * 4);
    up.off_coef = up.off_l + align256((size_t)up.G * NL * 4);
    up.off_fidx = up.off_coef + align256(up.coef.size() * 4);
    up.bytes = up.off_fidx + align256(up.fidx.size() * 4);
    return true;
}

std::mutex g_jac_mu;
std::map<std::tuple<int, int, int>, UnitPlan> g_jac_plans;

const UnitPlan *jac_plan(int D, int P, int NL) {
    std::lock_guard<std::mutex> lk(g_jac_mu);
    const auto key = std::make_tuple(D, P, NL);
    auto it = g_jac_plans.find(key);
    if (it != g_jac_plans.end()) return &it->second;
    UnitPlan up;
    if (!build_jac_plan(D, P, NL, up)) return nullptr;
    return &g_jac_plans.emplace(key, std::move(up)).first->second;
}

// Device copy of a unit plan (cached per device and key).
const uint8_t *plan_table(const UnitPlan &up, uint64_t key, cudaError_t *e) {
    return (const uint8_t *)device_table(
        key, up.bytes,
        [&up](uint8_t *h) {
            std::memcpy(h, up.pairs.data(), up.pairs.size() * sizeof(uint16_t));
            std::memcpy(h + up.off_k, up.unit_k.data(), up.unit_k.size() * 4);
            std::memcpy(h + up.off_nl, up.unit_nl.data(), up.unit_nl.size() * 4);
            std::memcpy(h + up.off_l, up.unit_l.data(), up.unit_l.size() * 4);
            std::memcpy(h + up.off_coef, up.coef.data(), up.coef.size() * 4);
            std::memcpy(h + up.off_fidx, up.fidx.data(), up.fidx.size() * 4);
        },
        e);
}

// Largest |x| of each head, as fp32 bit patterns (non-negative floats order like
// their bits): mx[bh][0..3] = max |q|, |k|, |v|, |r|.
__device__ __forceinline__ void warp_max_to(unsigned int *dst, float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    if ((threadIdx.x & 31) == 0 && x > 0.f) atomicMax(dst, __float_as_uint(x));
}

// One thread per token row: r_t = [dy_t / den_t | -(dy_t . y_t) / den_t] (stride bwd_rs),
// and the per-head maxima of |q|, |k|, |v|, |r|.  Blocks never straddle heads.
template <int DK, int DV>
__global__ void __launch_bounds__(128)
bwd_tc_r_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const __nv_bfloat16 *__restrict__ v, const float *__restrict__ dy, const float *__restrict__ y,
                const float *__restrict__ den, float *__restrict__ r, unsigned int *__restrict__ mx, int64_t N) {
    const int64_t bh = blockIdx.y;
    const int64_t t = (int64_t)blockIdx.x * 128 + threadIdx.x;
    const bool valid = t < N;
    const int64_t row = bh * N + (valid ? t : 0);
    float mq = 0.f, mk = 0.f, mv = 0.f, mr = 0.f;
    if (valid) {
#pragma unroll 4
        for (int i = 0; i < DK / 8; ++i) {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(q + row * DK) + i);
            const uint4 b = __ldg(reinterpret_cast<const uint4 *>(k + row * DK) + i);
            const __nv_bfloat16 *ha = reinterpret_cast<const __nv_bfloat16 *>(&a);
            const __nv_bfloat16 *hb = reinterpret_cast<const __nv_bfloat16 *>(&b);
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                mq = fmaxf(mq, fabsf(__bfloat162float(ha[w])));
                mk = fmaxf(mk, fabsf(__bfloat162float(hb[w])));
            }
        }
        const float inv = 1.0f / den[row];
        float dot = 0.f;
        float *rr = r + row * bwd_rs(DV);
#pragma unroll 2
        for (int i = 0; i < DV / 8; ++i) {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(v + row * DV) + i);
            const __nv_bfloat16 *ha = reinterpret_cast<const __nv_bfloat16 *>(&a);
            const float4 d0 = __ldg(reinterpret_cast<const float4 *>(dy + row * DV) + 2 * i);
            const float4 d1 = __ldg(reinterpret_cast<const float4 *>(dy + row * DV) + 2 * i + 1);
            const float4 y0 = __ldg(reinterpret_cast<const float4 *>(y + row * DV) + 2 * i);
            const float4 y1 = __ldg(reinterpret_cast<const float4 *>(y + row * DV) + 2 * i + 1);
            const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
            const float yy[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
            float gg[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                mv = fmaxf(mv, fabsf(__bfloat162float(ha[w])));
                gg[w] = dd[w] * inv;
                dot = fmaf(gg[w], yy[w], dot);
                mr = fmaxf(mr, fabsf(gg[w]));
            }
            reinterpret_cast<float4 *>(rr)[2 * i] = make_float4(gg[0], gg[1], gg[2], gg[3]);
            reinterpret_cast<float4 *>(rr)[2 * i + 1] = make_float4(gg[4], gg[5], gg[6], gg[7]);
        }
        rr[DV] = -dot;
        mr = fmaxf(mr, fabsf(dot));
#pragma unroll
        for (int j = DV + 1; j < bwd_rs(DV); ++j) rr[j] = 0.f;
    }
    warp_max_to(mx + bh * 4 + 0, mq);
    warp_max_to(mx + bh * 4 + 1, mk);
    warp_max_to(mx + bh * 4 + 2, mv);
    warp_max_to(mx + bh * 4 + 3, mr);
}

// Buffers of the gradient scans' operands (prescaled fp16, chunk-interleaved as the
// prefill's rows: chunk_rows).  Normal order: q, k, v.  Reversed order (frame token
// t' = N - 1 - t): q, k, g = r[:d_V] and rho = r[d_V] ([BH][nch][128]).  The readouts'
// multipliers in fp32, chunk-interleaved float4 quads (bwd_rs / 4 per token): r in time
// order (dq) and u = [v | 1] reversed (dk).
struct BwdImages {
    __half *q, *k, *v, *qr, *kr, *gr, *rho;
    float *rq, *uq;
};

// Quad j of a multiplier row of frame token f into its chunk-interleaved place.
__device__ __forceinline__ void put_quad(float *img, int64_t bh, int nch, int mq, int64_t f, int j, float4 x) {
    reinterpret_cast<float4 *>(img)[((bh * nch + f / kL) * mq + j) * kL + f % kL] = x;
}

// Piece j (8 values) of a row into a chunk-interleaved image at frame token f.
template <int D>
__device__ __forceinline__ void put_piece(__half *img, int64_t bh, int nch, int64_t f, int j, uint4 u) {
    reinterpret_cast<uint4 *>(img)[((bh * nch + f / kL) * (D / 8) + j) * kL + f % kL] = u;
}
__device__ __forceinline__ uint4 bf16x8_to_half_scaled(uint4 w, float sc) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(x[i] << 16), hi = __uint_as_float(x[i] & 0xFFFF0000u);
        const __half2 h = __floats2half2_rn(lo * sc, hi * sc);
        o[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ uint4 f32x8_to_half_scaled(float4 a, float4 b, float sc) {
    const __half2 h0 = __floats2half2_rn(a.x * sc, a.y * sc), h1 = __floats2half2_rn(a.z * sc, a.w * sc);
    const __half2 h2 = __floats2half2_rn(b.x * sc, b.y * sc), h3 = __floats2half2_rn(b.z * sc, b.w * sc);
    return make_uint4(*reinterpret_cast<const uint32_t *>(&h0), *reinterpret_cast<const uint32_t *>(&h1),
                      *reinterpret_cast<const uint32_t *>(&h2), *reinterpret_cast<const uint32_t *>(&h3));
}

// One thread per token row: the operand images of the three scans, (block 0 of each
// head) their per-head maxima rows: st_n = (|q|, |k|, |v|, 0) for dq, st_r = (|k|, |q|,
// |r|, 0) for dk and dv, and the per-chunk maxima of the prescaled r (g and -(g.y)) in
// the reversed frame, cm[head][chunk] (zeroed before; fp32 bit patterns).
template <int DK, int DV>
__global__ void __launch_bounds__(128)
bwd_tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ v, const float *__restrict__ r,
                   const unsigned int *__restrict__ mx, float *__restrict__ st_n, float *__restrict__ st_r,
                   unsigned int *__restrict__ cm, BwdImages im, int64_t N, int nch, int *flags) {
    const int64_t bh = blockIdx.y;
    const float fq = __uint_as_float(mx[bh * 4 + 0]), fk = __uint_as_float(mx[bh * 4 + 1]),
                fv = __uint_as_float(mx[bh * 4 + 2]), fr = __uint_as_float(mx[bh * 4 + 3]);
    // r is prescaled so that its largest value lies in [2^(kRHead-1), 2^kRHead) rather than
    // below 1: one token with a tiny denominator can make |r| span many octaves, and below 1
    // the rest would fall into fp16's subnormal range.  The dk and dv scans bound their
    // readout operand by the per-chunk maxima cm instead of by this largest value.
    const float fr_s = fr * pow2f(-kRHead);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        st_n[bh * 4 + 0] = fq; st_n[bh * 4 + 1] = fk; st_n[bh * 4 + 2] = fv; st_n[bh * 4 + 3] = 0.f;
        st_r[bh * 4 + 0] = fk; st_r[bh * 4 + 1] = fq; st_r[bh * 4 + 2] = fr_s; st_r[bh * 4 + 3] = 0.f;
        if (!(fq <= FLT_MAX && fk <= FLT_MAX && fv <= FLT_MAX && fr <= FLT_MAX)) atomicExch(flags + kFlagRange, 1);
    }
    const int64_t t = (int64_t)blockIdx.x * 128 + threadIdx.x;
    if (t >= N) return;
    const int64_t row = bh * N + t, tr = N - 1 - t;
    const float sq = pow2f(-scale_exp(fq)), sk = pow2f(-scale_exp(fk)), sv = pow2f(-scale_exp(fv)),
                sr = pow2f(-scale_exp(fr_s));
#pragma unroll 2
    for (int j = 0; j < DK / 8; ++j) {
        const uint4 a = bf16x8_to_half_scaled(__ldg(reinterpret_cast<const uint4 *>(q + row * DK) + j), sq);
        const uint4 b = bf16x8_to_half_scaled(__ldg(reinterpret_cast<const uint4 *>(k + row * DK) + j), sk);
        put_piece<DK>(im.q, bh, nch, t, j, a);
        put_piece<DK>(im.k, bh, nch, t, j, b);
        put_piece<DK>(im.qr, bh, nch, tr, j, a);
        put_piece<DK>(im.kr, bh, nch, tr, j, b);
    }
    const float *rr = r + row * bwd_rs(DV);
    constexpr int MQ = bwd_rs(DV) / 4;
    float rmax = 0.f;
#pragma unroll 2
    for (int j = 0; j < DV / 8; ++j) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(v + row * DV) + j);
        put_piece<DV>(im.v, bh, nch, t, j, bf16x8_to_half_scaled(w, sv));
        const float4 g0 = __ldg(reinterpret_cast<const float4 *>(rr) + 2 * j);
        const float4 g1 = __ldg(reinterpret_cast<const float4 *>(rr) + 2 * j + 1);
        put_piece<DV>(im.gr, bh, nch, tr, j, f32x8_to_half_scaled(g0, g1, sr));
        rmax = fmaxf(rmax, fmaxf(fmaxf(fmaxf(fabsf(g0.x), fabsf(g0.y)), fmaxf(fabsf(g0.z), fabsf(g0.w))),
                                 fmaxf(fmaxf(fabsf(g1.x), fabsf(g1.y)), fmaxf(fabsf(g1.z), fabsf(g1.w)))));
        put_quad(im.rq, bh, nch, MQ, t, 2 * j, g0);
        put_quad(im.rq, bh, nch, MQ, t, 2 * j + 1, g1);
        const uint32_t x[4] = {w.x, w.y, w.z, w.w};
        put_quad(im.uq, bh, nch, MQ, tr, 2 * j,
                 make_float4(__uint_as_float(x[0] << 16), __uint_as_float(x[0] & 0xFFFF0000u),
                             __uint_as_float(x[1] << 16), __uint_as_float(x[1] & 0xFFFF0000u)));
        put_quad(im.uq, bh, nch, MQ, tr, 2 * j + 1,
                 make_float4(__uint_as_float(x[2] << 16), __uint_as_float(x[2] & 0xFFFF0000u),
                             __uint_as_float(x[3] << 16), __uint_as_float(x[3] & 0xFFFF0000u)));
    }
#pragma unroll
    for (int j = DV / 4; j < MQ; ++j) {   // the last quads: r[d_V] (and zero padding); u's 1
        put_quad(im.rq, bh, nch, MQ, t, j, __ldg(reinterpret_cast<const float4 *>(rr) + j));
        put_quad(im.uq, bh, nch, MQ, tr, j, make_float4(j == DV / 4 ? 1.f : 0.f, 0.f, 0.f, 0.f));
    }
    const float rho = __ldg(rr + DV);
    im.rho[(bh * nch + tr / kL) * kL + tr % kL] = __float2half_rn(rho * sr);
    rmax = fmaxf(rmax, fabsf(rho)) * sr;
    if (!(rmax <= FLT_MAX)) rmax = FLT_MAX;   // a non-finite r has raised the range flag
    atomicMax(cm + bh * nch + tr / kL, __float_as_uint(rmax));
}

// T_n(x) = sum_{p<n} x^p / p! (0 for n = 0), Horner from the top term.
__device__ __forceinline__ float taylor_n(float x, int n) {
    if (n <= 0) return 0.f;
    float h = 1.f;
    for (int p = n - 1; p >= 1; --p) h = fmaf(h, x / (float)p, 1.f);
    return h;
}

// The pairs inside a chunk, per (head, frame chunk, 32 query rows of it).  KIND 0: dq
// (frame = time; queries q, keys k, weights (r_t . u_s) T_{P-1}(x) / c, values k_s);
// KIND 1: dk (frame reversed; queries k, keys q, weights (u_t . r_s) T_{P-1}(x) / c,
// values q_s); KIND 2: dv (frame reversed; queries k, keys q, weights T_P(x), values
// g_s).  The scan's inter-chunk sums are added and the result is stored at the
// token's place in time.
template <int DK, int DV, int KIND>
struct FinBwd {
    static constexpr int AW = DK + 1;                  // row strides (odd: conflict-free columns)
    static constexpr int MW = DV + 1;
    static constexpr int SW = DV + 1;
    static constexpr int RQ = 32;                      // query rows per CTA
    static constexpr int WW = 129;
    static constexpr int SMEM = 4 * (RQ * AW + RQ * MW + kL * AW + kL * SW + RQ * WW);
    static_assert(SMEM <= 232448, "finish shared memory");
};

// Loads rows [0, n) of a frame chunk into shared memory as fp32, row stride `ld`:
// bf16 rows of D values (16-byte loads) or fp32 rows of the r buffer (D + 1 values of
// stride bwd_rs, 16-byte loads); u = [v | 1] rows are bf16 rows plus the constant.
template <int D, bool REV>
__device__ __forceinline__ void fin_rows_bf16(float *dst, int ld, const __nv_bfloat16 *src, int64_t bh, int64_t N,
                                              int64_t f0, int n) {
    for (int e = threadIdx.x; e < n * (D / 8); e += 256) {
        const int i = e / (D / 8), j = e % (D / 8);
        const int64_t f = f0 + i;
        const int64_t o = REV ? N - 1 - f : f;
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(src + (bh * N + o) * D) + j);
        const uint32_t x[4] = {w.x, w.y, w.z, w.w};
        float *d = dst + i * ld + 8 * j;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            d[2 * h] = __uint_as_float(x[h] << 16);
            d[2 * h + 1] = __uint_as_float(x[h] & 0xFFFF0000u);
        }
    }
}
template <int DV, bool REV>
__device__ __forceinline__ void fin_rows_r(float *dst, int ld, int ncols, const float *r, int64_t bh, int64_t N,
                                           int64_t f0, int n) {
    constexpr int Q = bwd_rs(DV) / 4;
    for (int e = threadIdx.x; e < n * Q; e += 256) {
        const int i = e / Q, j = e % Q;
        const int64_t f = f0 + i;
        const int64_t o = REV ? N - 1 - f : f;
        const float4 w = __ldg(reinterpret_cast<const float4 *>(r + (bh * N + o) * bwd_rs(DV)) + j);
        const float x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h)
            if (4 * j + h < ncols) dst[i * ld + 4 * j + h] = x[h];
    }
}

template <int DK, int DV, int KIND>
__global__ void __launch_bounds__(256)
bwd_tc_finish_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                     const __nv_bfloat16 *__restrict__ v, const float *__restrict__ r,
                     const float *__restrict__ sums, float *__restrict__ out, int64_t N, int nch, int P,
                     float inv_c) {
    using FC = FinBwd<DK, DV, KIND>;
    extern __shared__ float fsm[];
    float *A = fsm;                            // [RQ][AW]  query rows
    float *M = A + FC::RQ * FC::AW;            // [RQ][MW]  query multipliers (KIND 0, 1)
    float *B = M + FC::RQ * FC::MW;            // [kL][AW]  key rows
    float *S = B + kL * FC::AW;                // [kL][SW]  key-side u or r (KIND 0, 1), g (KIND 2)
    float *Wt = S + kL * FC::SW;               // [RQ][WW]  weights
    const int64_t bh = blockIdx.x;
    const int c = blockIdx.y, r0 = blockIdx.z * FC::RQ;
    const int64_t f0 = (int64_t)c * kL;
    const int nt = (int)(N - f0 < kL ? N - f0 : kL);
    if (r0 >= nt) return;
    const int nr = nt - r0 < FC::RQ ? nt - r0 : FC::RQ;
    const int ns = r0 + nr;                    // keys 0 .. ns-1 of the chunk
    constexpr bool REV = KIND != 0;
    const __nv_bfloat16 *qa = KIND == 0 ? q : k, *kb = KIND == 0 ? k : q;
    const int tid = threadIdx.x;
    fin_rows_bf16<DK, REV>(A, FC::AW, qa, bh, N, f0 + r0, nr);
    fin_rows_bf16<DK, REV>(B, FC::AW, kb, bh, N, f0, ns);
    if constexpr (KIND != 2) {
        // r rows on the query side for dq, on the key side for dk; u = [v | 1] on the other
        float *mr = KIND == 0 ? M : S, *mu = KIND == 0 ? S : M;
        const int ldr = KIND == 0 ? FC::MW : FC::SW, ldu = KIND == 0 ? FC::SW : FC::MW;
        fin_rows_r<DV, REV>(mr, ldr, DV + 1, r, bh, N, KIND == 0 ? f0 + r0 : f0, KIND == 0 ? nr : ns);
        const int nu = KIND == 0 ? ns : nr;
        fin_rows_bf16<DV, REV>(mu, ldu, v, bh, N, KIND == 0 ? f0 : f0 + r0, nu);
        for (int i = tid; i < nu; i += 256) mu[i * ldu + DV] = 1.f;
    } else {
        fin_rows_r<DV, REV>(S, FC::SW, DV, r, bh, N, f0, ns);
    }
    // rows past the chunk's end: zero, so that whole tiles can be computed
    for (int e = tid; e < (FC::RQ - nr) * FC::AW; e += 256) A[nr * FC::AW + e] = 0.f;
    for (int e = tid; e < (kL - ns) * FC::AW; e += 256) B[ns * FC::AW + e] = 0.f;
    if constexpr (KIND != 2)
        for (int e = tid; e < (FC::RQ - nr) * FC::MW; e += 256) M[nr * FC::MW + e] = 0.f;
    for (int e = tid; e < (kL - ns) * FC::SW; e += 256) S[ns * FC::SW + e] = 0.f;
    __syncthreads();
    // weights: each thread a 4 x 4 tile (query rows 4 wi .. 4 wi + 3, keys ks + 32 j); a
    // warp shares its query rows (broadcast) and spans 32 consecutive keys (odd strides:
    // no bank conflicts)
    {
        const int wi = tid / 32, ks = tid % 32;
        const int i0 = 4 * wi;
        if (i0 < nr) {
            float x[4][4], d[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) x[a][b] = d[a][b] = 0.f;
            const int smax = r0 + i0 + 3;   // the tile's last query row sees keys up to it
#pragma unroll 4
            for (int e = 0; e < DK; ++e) {
                float av[4], bv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) av[a] = A[(i0 + a) * FC::AW + e];
#pragma unroll
                for (int b = 0; b < 4; ++b) bv[b] = B[(ks + 32 * b) * FC::AW + e];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) x[a][b] = fmaf(av[a], bv[b], x[a][b]);
            }
            if constexpr (KIND != 2) {
#pragma unroll 4
                for (int e = 0; e <= DV; ++e) {
                    float mv[4], sv[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) mv[a] = M[(i0 + a) * FC::MW + e];
#pragma unroll
                    for (int b = 0; b < 4; ++b) sv[b] = S[(ks + 32 * b) * FC::SW + e];
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int b = 0; b < 4; ++b) d[a][b] = fmaf(mv[a], sv[b], d[a][b]);
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int s = ks + 32 * b, i = i0 + a;
                    float w = 0.f;
                    if (s <= r0 + i && s <= smax) {
                        const float xx = x[a][b] * inv_c;
                        w = KIND == 2 ? taylor_n(xx, P) : d[a][b] * taylor_n(xx, P - 1) * inv_c;
                    }
                    Wt[i * FC::WW + s] = w;
                }
        }
    }
    __syncthreads();
    // outputs: a warp takes 4 query rows (broadcast weights), a lane NCOL / 32 columns
    constexpr int NCOL = KIND == 2 ? DV : DK;
    constexpr int CPL = (NCOL + 31) / 32;
    {
        const int wi = tid / 32, lane = tid % 32;
        const int i0 = 4 * wi;
        if (i0 < nr) {
            float acc[4][CPL];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) acc[a][cc] = 0.f;
            const int smax = r0 + i0 + 3 < ns - 1 ? r0 + i0 + 3 : ns - 1;
            for (int s = 0; s <= smax; ++s) {
                float wv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) wv[a] = Wt[(i0 + a) * FC::WW + s];
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    const int col = lane + 32 * cc;
                    if (col < NCOL) {
                        const float val = KIND == 2 ? S[s * FC::SW + col] : B[s * FC::AW + col];
#pragma unroll
                        for (int a = 0; a < 4; ++a) acc[a][cc] = fmaf(wv[a], val, acc[a][cc]);
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int t = r0 + i0 + a;   // token of the chunk (frame)
                if (i0 + a >= nr) break;
                const int64_t f = f0 + t;
                const int64_t o = REV ? N - 1 - f : f;
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    const int col = lane + 32 * cc;
                    if (col >= NCOL) continue;
                    float inter;
                    if constexpr (KIND == 2)   // the prefill scan's sums: quads [BH][nch][DQ][128]
                        inter = sums[(((bh * nch + c) * sum_quads(DV) + col / 4) * kL + t) * 4 + col % 4];
                    else                       // the gradient scan's sums [BH][d_K][N]
                        inter = sums[(bh * DK + col) * N + f];
                    out[(bh * N + o) * NCOL + col] = inter + acc[a][cc];
                }
            }
        }
    }
}

// Workspace of the tensor-core backward.  The front region first serves the
// recomputed forward, then the operand images and sums; y, den and r follow it.
struct BwdTcLayout {
    size_t fwd = 0, front = 0, off_mx = 0, off_stn = 0, off_str = 0, off_cm = 0, off_img = 0, off_sq = 0, off_sk = 0,
           off_sv = 0, off_ur = 0, off_rq = 0, off_y = 0, off_den = 0, off_r = 0, total = 0;
    size_t img_q = 0, img_v = 0, img_rho = 0;
};

template <int DK, int DV>
bool bwd_tc_layout(int BH, int64_t N, int64_t F, int P, BwdTcLayout &L) {
    Plan pl;
    if (!make_plan<DK, DV>(BH, N, F, P, true, 1, false, pl)) return false;
    L.fwd = pl.total;
    const int nch = (int)((N + kL - 1) / kL);
    const size_t rows = (size_t)BH * nch * kL;
    L.img_q = align256(rows * DK * 2);
    L.img_v = align256(rows * DV * 2);
    L.img_rho = align256(rows * 2);
    L.off_mx = 0;
    L.off_stn = align256((size_t)BH * 16);
    L.off_str = L.off_stn + align256((size_t)BH * 16);
    L.off_cm = L.off_str + align256((size_t)BH * 16);
    L.off_img = L.off_cm + align256((size_t)BH * nch * 4);
    L.off_sq = L.off_img + 4 * L.img_q + 2 * L.img_v + L.img_rho;
    L.off_sk = L.off_sq + align256((size_t)BH * DK * N * 4);
    L.off_sv = L.off_sk + align256((size_t)BH * DK * N * 4);
    L.off_ur = L.off_sv + align256((size_t)BH * nch * sum_quads(DV) * kL * 16);
    L.off_rq = L.off_ur + align256(rows * bwd_rs(DV) * 4);
    const size_t mine = L.off_rq + align256(rows * bwd_rs(DV) * 4);
    L.front = L.fwd > mine ? L.fwd : mine;
    L.off_y = align256(L.front);
    L.off_den = L.off_y + align256((size_t)BH * N * DV * 4);
    L.off_r = L.off_den + align256((size_t)BH * N * 4);
    L.total = L.off_r + align256((size_t)BH * N * bwd_rs(DV) * 4);
    return true;
}

template <int DK, int DV>
cudaError_t bwd_tc_run(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k, const void *v,
                       const float *dy, float *dq, float *dk, float *dv, void *ws, size_t ws_bytes, int *flags,
                       cudaStream_t stream) {
    using C = Cfg<DK, DV>;
    const int P = basis.P;
    const int64_t F = basis.F;
    BwdTcLayout L;
    if (!bwd_tc_layout<DK, DV>(BH, N, F, P, L) || ws_bytes < L.total) return cudaErrorInvalidValue;
    if (N == 0 || BH == 0) return cudaSuccess;
    uint8_t *w = (uint8_t *)ws;
    float *y = (float *)(w + L.off_y), *den = (float *)(w + L.off_den), *r = (float *)(w + L.off_r);
    const auto *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k, *vb = (const __nv_bfloat16 *)v;
    const int nch = (int)((N + kL - 1) / kL);
    const float inv_c = 1.0f / sqrtf((float)DK);
    const int64_t wait_ns = g_opt_wait_limit > 0 ? g_opt_wait_limit : kDefaultWaitNs;
    cudaError_t e;

    // the forward on tensor cores: y and den
    if ((e = run<DK, DV>(basis, BH, N, q, k, v, y, nullptr, nullptr, false, ws, L.fwd, flags, stream, nullptr, den)) !=
        cudaSuccess)
        return e;

    unsigned int *mx = (unsigned int *)(w + L.off_mx);
    float *st_n = (float *)(w + L.off_stn), *st_r = (float *)(w + L.off_str);
    unsigned int *cm = (unsigned int *)(w + L.off_cm);
    BwdImages im;
    im.q = (__half *)(w + L.off_img);
    im.k = (__half *)(w + L.off_img + L.img_q);
    im.qr = (__half *)(w + L.off_img + 2 * L.img_q);
    im.kr = (__half *)(w + L.off_img + 3 * L.img_q);
    im.v = (__half *)(w + L.off_img + 4 * L.img_q);
    im.gr = (__half *)(w + L.off_img + 4 * L.img_q + L.img_v);
    im.rho = (__half *)(w + L.off_img + 4 * L.img_q + 2 * L.img_v);
    im.uq = (float *)(w + L.off_ur);
    im.rq = (float *)(w + L.off_rq);
    float *sq = (float *)(w + L.off_sq), *sk = (float *)(w + L.off_sk), *sv = (float *)(w + L.off_sv);

    const dim3 rgrid((unsigned)((N + 127) / 128), (unsigned)BH);
    e = cudaMemsetAsync(mx, 0, (size_t)BH * 16, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(cm, 0, (size_t)BH * nch * 4, stream);
    if (e == cudaSuccess) {
        launch_begin(kBwdTcR, stream);
        bwd_tc_r_kernel<DK, DV><<<rgrid, 128, 0, stream>>>(qb, kb, vb, dy, y, den, r, mx, N);
        launch_end(kBwdTcR, stream);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        launch_begin(kBwdTcPrep, stream);
        bwd_tc_prep_kernel<DK, DV><<<rgrid, 128, 0, stream>>>(qb, kb, vb, r, mx, st_n, st_r, cm, im, N, nch, flags);
        launch_end(kBwdTcPrep, stream);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(sq, 0, L.off_ur - L.off_sq, stream)) != cudaSuccess) return e;   // the three sums

    ScanParams base;
    base.stats = nullptr;
    base.S = base.Z = nullptr;
    base.part = nullptr;
    base.red_atomic = 1;
    base.flags = flags;
    base.F = F;
    base.N = N;
    base.BH = BH;
    base.c0 = 0;
    base.nc = nch;
    base.nch = nch;
    base.P = P;
    base.load_state = 0;
    base.store_state = 0;
    base.stall_chunk = -1;
    base.inv_c = inv_c;
    base.lc = floor_log2_c(DK);
    base.wait_ns = wait_ns;
    auto set_plan = [](ScanParams &sp, const UnitPlan &up, const uint8_t *tab) {
        sp.pairs = (const uint16_t *)tab;
        sp.unit_k = (const int32_t *)(tab + up.off_k);
        sp.unit_nl = (const int32_t *)(tab + up.off_nl);
        sp.unit_l = (const int32_t *)(tab + up.off_l);
        sp.unit_coef = (const float *)(tab + up.off_coef);
        sp.unit_fidx = (const int32_t *)(tab + up.off_fidx);
        sp.G = up.G;
    };
    if (P >= 2) {   // dq and dk scans (T_{P-1} = 0 at P = 1: the sums stay zero)
        const UnitPlan *jp = jac_plan(DK, P, C::NL);
        if (!jp) return cudaErrorInvalidValue;
        e = cudaSuccess;
        const uint8_t *jt = plan_table(*jp, ((uint64_t)DK << 32) | ((uint64_t)P << 16) | (uint64_t)C::NL |
                                                (uint64_t(1) << 61), &e);
        if (!jt) return e != cudaSuccess ? e : cudaErrorMemoryAllocation;
        if ((e = cudaFuncSetAttribute(tc_scan_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      C::SMEM)) != cudaSuccess)
            return e;
        ScanParams sp = base;
        set_plan(sp, *jp, jt);
        // dq: frame = time; A = q, B = k, columns [v | 1], multipliers r
        sp.q16 = im.q;
        sp.k16 = im.k;
        sp.v16 = im.v;
        sp.stats = st_n;
        sp.zval16 = nullptr;
        sp.zscaled = 0;
        sp.mult = im.rq;
        sp.mult_quads = bwd_rs(DV) / 4;
        sp.sums_jac = sq;
        launch_begin(kBwdTcScan, stream);
        tc_scan_kernel<DK, DV, true><<<BH * sp.G, kScanThreads, C::SMEM, stream>>>(sp);
        launch_end(kBwdTcScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // dk: frame reversed; A = k, B = q, columns [g | rho], multipliers u
        sp.q16 = im.kr;
        sp.k16 = im.qr;
        sp.v16 = im.gr;
        sp.stats = st_r;
        sp.zval16 = im.rho;
        sp.zscaled = 1;
        sp.mult = im.uq;
        sp.colmax = (const float *)cm;   // columns g and -(g.y)
        sp.sums_jac = sk;
        launch_begin(kBwdTcScan, stream);
        tc_scan_kernel<DK, DV, true><<<BH * sp.G, kScanThreads, C::SMEM, stream>>>(sp);
        launch_end(kBwdTcScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {   // dv: the prefill scan on the reversed sequence, queries k, keys q, values g
        const UnitPlan *up = unit_plan(DK, P, C::NL);
        if (!up) return cudaErrorInvalidValue;
        e = cudaSuccess;
        const uint8_t *tab = plan_table(*up, ((uint64_t)DK << 32) | ((uint64_t)P << 16) | (uint64_t)up->NL |
                                                 (uint64_t(1) << 60), &e);
        if (!tab) return e != cudaSuccess ? e : cudaErrorMemoryAllocation;
        ScanParams sp = base;
        set_plan(sp, *up, tab);
        sp.q16 = im.kr;
        sp.k16 = im.qr;
        sp.v16 = im.gr;
        sp.stats = st_r;
        sp.part = sv;
        sp.colmax = (const float *)cm;   // columns g, and the Z columns' 1
        sp.colmax_floor = 1.f;
        launch_begin(kBwdTcScan, stream);
        tc_scan_kernel<DK, DV><<<BH * sp.G, kScanThreads, C::SMEM, stream>>>(sp);
        launch_end(kBwdTcScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {   // the pairs inside each chunk, the scale, the reversal back
        const dim3 fgrid((unsigned)BH, (unsigned)nch, kL / 32);
        if ((e = cudaFuncSetAttribute(bwd_tc_finish_kernel<DK, DV, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      FinBwd<DK, DV, 0>::SMEM)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwd_tc_finish_kernel<DK, DV, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      FinBwd<DK, DV, 1>::SMEM)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwd_tc_finish_kernel<DK, DV, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      FinBwd<DK, DV, 2>::SMEM)) != cudaSuccess)
            return e;
        launch_begin(kBwdTcFinish, stream);
        bwd_tc_finish_kernel<DK, DV, 0><<<fgrid, 256, FinBwd<DK, DV, 0>::SMEM, stream>>>(qb, kb, vb, r, sq, dq, N,
                                                                                          nch, P, inv_c);
        if ((e = cudaGetLastError()) == cudaSuccess) {
            bwd_tc_finish_kernel<DK, DV, 1><<<fgrid, 256, FinBwd<DK, DV, 1>::SMEM, stream>>>(qb, kb, vb, r, sk, dk,
                                                                                              N, nch, P, inv_c);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) {
            bwd_tc_finish_kernel<DK, DV, 2><<<fgrid, 256, FinBwd<DK, DV, 2>::SMEM, stream>>>(qb, kb, vb, r, sv, dv,
                                                                                              N, nch, P, inv_c);
            e = cudaGetLastError();
        }
        launch_end(kBwdTcFinish, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

// Non-template entry points of one (d_K, d_V) instance of the tensor-core backward.
#define SATA_TC_BWD_DEFINE(a, b)                                                                            \
    size_t tc_bwd_workspace_##a##_##b(int BH, int64_t N, int64_t F, int P) {                                \
        BwdTcLayout L;                                                                                      \
        return bwd_tc_layout<a, b>(BH, N, F, P, L) ? L.total : 0;                                           \
    }                                                                                                       \
    cudaError_t tc_bwd_run_##a##_##b(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k, \
                                     const void *v, const float *dy, float *dq, float *dk, float *dv, void *ws, \
                                     size_t ws_bytes, int *flags, cudaStream_t stream) {                    \
        return bwd_tc_run<a, b>(basis, BH, N, q, k, v, dy, dq, dk, dv, ws, ws_bytes, flags, stream);        \
    }

}  // namespace sata
