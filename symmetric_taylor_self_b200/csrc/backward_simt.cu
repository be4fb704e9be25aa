// Backward pass of the causal prefill (fp32-accurate): the gradients of a loss
// L with respect to q, k and v, given dL/dy for every output.
//
// The method's pages define no backward pass; they expect the attention to be
// trained inside ordinary Transformer pipelines ([CC-TAYLOR] "Comparison with
// other methods"; end-to-end training is listed under "Future directions").
// This is the exact gradient of the forward as defined ([CC-TAYLOR] "Feature
// maps and linear attention"), written in the same feature form so that it
// costs a fixed amount per token:
//   y_t = num_t / den_t,  [num_t | den_t] = sum_{s<=t} w_ts u_s,  u_s = [v_s | 1],
//   w_ts = sum_f a_f phi_f(q_t) phi_f(k_s),  a_f = alpha_p C_p  (coef[] below).
// With g_t = dy_t / den_t and r_t = [g_t | -(g_t . y_t)], the gradient of w_ts
// is dw_ts = r_t . u_s, and
//   dq_t = J_phi(q_t)^T (a (.) S_t r_t),          S_t = sum_{s<=t} phi(k_s) u_s^T
//   dk_s = J_phi(k_s)^T (a (.) G_s u_s),          G_s = sum_{t>=s} phi(q_t) r_t^T
//   dv_s = (a (.) phi(k_s))^T G_s[:, :d_V],
// where J_phi is the Jacobian of the monomial features: d phi_f / d x_i =
// mult_i(f) * (the product of f's other indices).  Chunked like the forward
// (chunks of kL tokens): the state before / after a chunk gives the inter-chunk
// part; pairs inside a chunk are summed directly, with
//   dx_ts = dw_ts * T_{P-1}(x_ts)   (T_P' = T_{P-1}),  x_ts = q_t . k_s / c,
//   dq_t += dx_ts k_s / c,  dk_s += dx_ts q_t / c,  dv_s += w_ts g_t.
//
// Kernels, in stream order:
//   forward on the prefill's own path (tensor-core or CUDA-core) -> y and den;  bwd_r -> r;
//   bwd_q_scan: per feature tile, forward over the chunks with S: dq partials;
//   bwd_finish<dq>: sum the tiles' partials, add the intra-chunk part;
//   bwd_kv_scan: per feature tile, backward over the chunks with G: dk, dv partials;
//   bwd_finish<dk, dv>.
// Partials are summed in a fixed order: the result is deterministic.
#include <cuda_bf16.h>

#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "sata_internal.h"
#include "mma_tf32.cuh"
#include "simt_tiles.cuh"

namespace sata {
namespace {

using simt::kThreads;
using simt::kTF;
using simt::kL;
constexpr int kMaxComp = kMaxP - 2;
// Row stride (floats) of r = [dy / den | -(dy . y) / den]: d_V + 1 rounded up
// to a multiple of 4, so every row starts on a 16-byte boundary.
__host__ __device__ constexpr int r_stride(int d_V) { return (d_V + 1 + 3) / 4 * 4; }   // indices left of a top-degree feature after removing one
constexpr size_t kPartialBudget = size_t(2) << 30;  // bytes of partials per segment

// Features are dealt to the kTF-feature tiles round-robin: tile tau holds the
// features f = tau + m * ntiles, m = 0, 1, ...  The set of monomials of a
// degree is symmetric under relabelling the indices, so a strided sample of it
// contains every index about equally often: the Jacobian lists below have
// nearly equal lengths (a lexicographic block of 128 features would put one
// leading index in every feature and leave the other lists nearly empty).
//
// Jacobian table of one (d_K, P): for every tile and every input index i, the
// tile's features that contain i.  Entry (uint64):
//   bits 0..7 the feature's position m in its tile, 8..15 the multiplicity of
//   i, 16..63 the feature's other indices (one copy of i removed), 8 bits each,
//   padded with d_K (the constant 1).
// Layout: uint32 offsets[ntiles][d_K + 1] (into the entry array), then the
// entries, 8-byte aligned.
struct JacTable {
    std::vector<uint8_t> image;
    size_t off_entries = 0;
    int max_entries = 0;   // longest per-tile entry list
};

bool build_jac_table(int d_K, int P, JacTable &jt) {
    HostBasis hb;
    if (!build_basis_host(d_K, P, hb)) return false;
    const int64_t F = hb.offsets[P];
    const int64_t ntiles = (F + kTF - 1) / kTF;
    std::vector<std::vector<uint64_t>> lists((size_t)ntiles * d_K);
    for (int64_t f = 0; f < F; ++f) {
        const auto &t = hb.tuples[f];
        const int p = (int)t.size();
        const int64_t tile = f % ntiles, m = f / ntiles;
        size_t s = 0;
        while (s < t.size()) {   // runs of equal indices: one entry per distinct index
            size_t e = s;
            while (e < t.size() && t[e] == t[s]) ++e;
            uint64_t ent = (uint64_t)m | ((uint64_t)(e - s) << 8);
            int c = 0;
            for (int x = 0; x < p; ++x) {
                if (x == (int)s) continue;   // drop one copy of the index
                ent |= (uint64_t)t[x] << (16 + 8 * c);
                ++c;
            }
            for (; c < kMaxComp; ++c) ent |= (uint64_t)d_K << (16 + 8 * c);
            lists[(size_t)tile * d_K + t[s]].push_back(ent);
            s = e;
        }
    }
    const size_t noff = (size_t)ntiles * (d_K + 1);
    size_t total = 0;
    for (auto &l : lists) total += l.size();
    jt.off_entries = (noff * sizeof(uint32_t) + 7) / 8 * 8;
    jt.image.assign(jt.off_entries + (total ? total : 1) * sizeof(uint64_t), 0);
    uint32_t *off = (uint32_t *)jt.image.data();
    uint64_t *ent = (uint64_t *)(jt.image.data() + jt.off_entries);
    size_t pos = 0;
    jt.max_entries = 0;
    for (int64_t tile = 0; tile < ntiles; ++tile) {
        const size_t start = pos;
        for (int i = 0; i < d_K; ++i) {
            off[tile * (d_K + 1) + i] = (uint32_t)pos;
            for (uint64_t e : lists[(size_t)tile * d_K + i]) ent[pos++] = e;
        }
        off[tile * (d_K + 1) + d_K] = (uint32_t)pos;
        if ((int)(pos - start) > jt.max_entries) jt.max_entries = (int)(pos - start);
    }
    return true;
}

// Device copy of the table, cached per (device, d_K, P).
const uint8_t *jac_table(int d_K, int P, size_t *off_entries, int *max_entries, cudaError_t *err) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, JacTable> cache;
    const JacTable *jt = nullptr;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto key = std::make_pair(d_K, P);
        auto it = cache.find(key);
        if (it == cache.end()) {
            JacTable t;
            if (!build_jac_table(d_K, P, t)) {
                *err = cudaErrorInvalidValue;
                return nullptr;
            }
            it = cache.emplace(key, std::move(t)).first;
        }
        jt = &it->second;
    }
    *off_entries = jt->off_entries;
    *max_entries = jt->max_entries;
    const uint64_t key = (uint64_t(0xB1) << 56) | ((uint64_t)d_K << 16) | (uint64_t)P;
    return (const uint8_t *)device_table(
        key, jt->image.size(), [jt](uint8_t *h) { std::memcpy(h, jt->image.data(), jt->image.size()); },
        err);
}

// phi_f(x~) for a feature's packed words: x~ is a row of d_K + 1 values whose
// last one is the constant 1; hi = the leading indices (degrees above 3), or
// all d_K when there are none.
__device__ __forceinline__ float feature(const float *x, uint32_t w, uint32_t hi) {
    float v = x[w & 255] * x[(w >> 8) & 255] * x[(w >> 16) & 255];
#pragma unroll
    for (int m = 0; m < 4; ++m) v *= x[(hi >> (8 * m)) & 255];
    return v;
}

// J_phi(x~)^T applied to the tile values of kJT consecutive tokens: for index
// i, acc[j] = sum over the tile's features f containing i of
// val[j][f] * d phi_f / d x_i at token j (x~ rows of DK1 values, val rows of
// kTF).  Each list entry is decoded once and applied to all kJT tokens, whose
// loads are independent of each other.
constexpr int kJT = 8;
__device__ __forceinline__ void jac_t(const uint32_t *off, const uint64_t *ent, int i, const float *x, int DK1,
                                      const float *val, int ldv, int ncomp, float (&acc)[kJT]) {
#pragma unroll
    for (int j = 0; j < kJT; ++j) acc[j] = 0.f;
    const uint32_t b = off[i], e = off[i + 1];
    for (uint32_t n = b; n < e; ++n) {
        const uint64_t u = ent[n];
        const int m = (int)(u & 255);
        const float mult = (float)((u >> 8) & 255);
        int ci[kMaxComp];
#pragma unroll
        for (int c = 0; c < kMaxComp; ++c) ci[c] = (int)((u >> (16 + 8 * c)) & 255);
#pragma unroll
        for (int j = 0; j < kJT; ++j) {
            float d = mult;
#pragma unroll
            for (int c = 0; c < kMaxComp; ++c)
                if (c < ncomp) d *= x[j * DK1 + ci[c]];
            acc[j] = fmaf(val[j * ldv + m], d, acc[j]);
        }
    }
}

// The Jacobian products of one chunk: items (index i, group of kJT tokens),
// kL / kJT groups per index; the results go to out[t * ld + i] for t < nt.
__device__ __forceinline__ void jac_chunk(const uint32_t *off, const uint64_t *ent, const float *x, int DK1,
                                          const float *val, int ldv, int ncomp, int d_K, int nt, float *out,
                                          int64_t ld) {
    constexpr int G = kL / kJT;
    for (int item = threadIdx.x; item < d_K * G; item += kThreads) {
        const int i = item / G, tb = (item % G) * kJT;
        if (tb >= nt) continue;
        float acc[kJT];
        jac_t(off, ent, i, x + tb * DK1, DK1, val + tb * ldv, ldv, ncomp, acc);
#pragma unroll
        for (int j = 0; j < kJT; ++j)
            if (tb + j < nt) __stcs(out + (int64_t)(tb + j) * ld + i, acc[j]);
    }
}

// Zeroes columns n .. w-1 of the kL rows of stride w.
__device__ __forceinline__ void zero_pad(float *x, int w, int n) {
    for (int e = threadIdx.x; e < kL * (w - n); e += kThreads) x[(e / (w - n)) * w + n + e % (w - n)] = 0.f;
}

// Loads one chunk: x~q, x~k [kL][d_K+1] (last column 1), u = [v | 1] and r
// (d_V + 1 values per row, row strides wu and wr, zero padded); rows past the
// end are zero.
__device__ __forceinline__ void load_chunk(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                           const __nv_bfloat16 *v, const float *r, int64_t row0,
                                           int nt, int d_K, int d_V, float *xq, float *xk, float *xu, int wu,
                                           float *xr, int wr) {
    const int DK1 = d_K + 1, DV1 = d_V + 1, RW = r_stride(d_V);
    if ((d_K & 7) == 0 && (d_V & 7) == 0) {
        // 16-byte loads: 8 bf16 of q, k or v, or 4 floats of r, per load; all of a
        // thread's loads are issued before its stores
        constexpr int U = (kL * (kMaxDK / 8) + kThreads - 1) / kThreads;             // q, k, v pieces
        constexpr int UR = (kL * (r_stride(kMaxDV) / 4) + kThreads - 1) / kThreads;  // r pieces
        static_assert(kMaxDV <= kMaxDK, "one bound for q, k and v");
        const int nq = kL * (d_K / 8), nv = kL * (d_V / 8), nr = kL * (RW / 4);
        uint4 bq[U], bk[U], bv[U];
        float4 br[UR];
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
        for (int u = 0; u < UR; ++u) {
            const int e = threadIdx.x + u * kThreads;
            br[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e < nr && e / (RW / 4) < nt)
                br[u] = *reinterpret_cast<const float4 *>(r + (row0 + e / (RW / 4)) * RW + (e % (RW / 4)) * 4);
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
                for (int w = 0; w < 8; ++w) xu[t * wu + j + w] = __bfloat162float(hv[w]);
            }
        }
#pragma unroll
        for (int u = 0; u < UR; ++u) {
            const int e = threadIdx.x + u * kThreads;
            if (e < nr) {
                const int t = e / (RW / 4), j = (e % (RW / 4)) * 4;
                const float x4[4] = {br[u].x, br[u].y, br[u].z, br[u].w};
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    if (j + w < DV1) xr[t * wr + j + w] = x4[w];
            }
        }
        for (int t = threadIdx.x; t < kL; t += kThreads) {   // the constant columns
            const float one = t < nt ? 1.f : 0.f;
            xq[t * DK1 + d_K] = one;
            xk[t * DK1 + d_K] = one;
            xu[t * wu + d_V] = one;
        }
        zero_pad(xu, wu, DV1);
        zero_pad(xr, wr, DV1);
        return;
    }
    // other head sizes: element loads, every element a thread owns loaded
    // before any is stored, so the global loads are in flight together
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
                a[u] = i < d_K ? __bfloat162float(q[(row0 + t) * d_K + i]) : 1.f;
                b[u] = i < d_K ? __bfloat162float(k[(row0 + t) * d_K + i]) : 1.f;
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
        b[u] = 0.f;
        if (e < kL * DV1) {
            const int t = e / DV1, j = e % DV1;
            if (t < nt) {
                a[u] = j < d_V ? __bfloat162float(v[(row0 + t) * d_V + j]) : 1.f;
                b[u] = r[(row0 + t) * RW + j];
            }
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = threadIdx.x + u * kThreads;
        if (e < kL * DV1) {
            xu[(e / DV1) * wu + e % DV1] = a[u];
            xr[(e / DV1) * wr + e % DV1] = b[u];
        }
    }
    zero_pad(xu, wu, DV1);
    zero_pad(xr, wr, DV1);
}

// Shared-memory image of one tile: its features' packed words and weights, its
// Jacobian lists (offsets rebased to 0), and its state rows.
struct TileSmem {
    uint64_t *ent;     // [max_entries]
    uint32_t *off;     // [d_K + 1]
    uint32_t *pk;      // [kTF] packed word (padding rows: the constant feature)
    uint32_t *hi;      // [kTF] leading indices (all d_K when P <= 4)
    float *coef;       // [kTF] a_f (0 on padding rows)
};

__device__ __forceinline__ void load_tile(TileSmem ts, const uint32_t *packed, const uint32_t *packed_hi,
                                          const float *coef, const uint32_t *jac_off, const uint64_t *jac_ent,
                                          int tile, int ntiles, int nf, int d_K) {
    const uint32_t pad = (uint32_t)d_K | ((uint32_t)d_K << 8) | ((uint32_t)d_K << 16);
    const uint32_t pad_hi = pad | ((uint32_t)d_K << 24);
    for (int m = threadIdx.x; m < kTF; m += kThreads) {
        const int64_t fg = (int64_t)tile + (int64_t)m * ntiles;
        const bool ok = m < nf;
        ts.pk[m] = ok ? packed[fg] : pad;
        ts.hi[m] = (ok && packed_hi) ? packed_hi[fg] : pad_hi;
        ts.coef[m] = ok ? coef[fg] : 0.f;
    }
    const uint32_t *toff = jac_off + (size_t)tile * (d_K + 1);
    const uint32_t base = toff[0];
    for (int i = threadIdx.x; i <= d_K; i += kThreads) ts.off[i] = toff[i] - base;
    const uint32_t n = toff[d_K] - base;
    for (uint32_t e = threadIdx.x; e < n; e += kThreads) ts.ent[e] = jac_ent[base + e];
}

// r_t = [dy_t / den_t | -(dy_t . y_t) / den_t], one warp per token.
__global__ void __launch_bounds__(kThreads)
bwd_r_kernel(const float *__restrict__ dy, const float *__restrict__ y, const float *__restrict__ den,
             float *__restrict__ r, int d_V, int64_t rows) {
    const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float inv = 1.0f / den[row];
    float s = 0.f;
    for (int j = lane; j < d_V; j += 32) {
        const float g = dy[row * d_V + j] * inv;
        r[row * r_stride(d_V) + j] = g;
        s = fmaf(g, y[row * d_V + j], s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) r[row * r_stride(d_V) + d_V] = -s;
}

// Shared-memory layout of the two scan kernels (floats after the tables).
// The three contractions run on tensor cores (mma_tf32.cuh); row strides
// follow its bank rules: the state [kTF][WS] and the contraction's token rows
// [kL][WA] are read with rows over g, the update's token rows [kL][WB] and
// feature columns [kL][kFeatC] with rows over c, the dv readout's feature rows
// [kL][kFeatG] with rows over g.
struct ScanSmem {
    static size_t tables(int d_K, int max_entries) {
        size_t b = (size_t)(max_entries > 0 ? max_entries : 1) * sizeof(uint64_t);
        b += ((size_t)(d_K + 1) + 2 * kTF) * sizeof(uint32_t) + kTF * sizeof(float);
        return (b + 15) / 16 * 16;
    }
    static size_t bytes(int d_K, int d_V, bool kv, int max_entries) {
        const size_t WS = mma32::stride_g(d_V + 1), WA = mma32::stride_g(d_V + 1), WB = mma32::stride_c(d_V + 1);
        const size_t feat = kv ? (size_t)kL * (mma32::kFeatG + mma32::kFeatC) : (size_t)2 * kL * mma32::kFeatC;
        return tables(d_K, max_entries) +
               sizeof(float) * ((size_t)kTF * WS + 2 * kL * (d_K + 1) + kL * (WA + WB) + feat);
    }
};

__device__ __forceinline__ TileSmem carve_tables(uint8_t *base, int d_K, int max_entries, float **rest) {
    TileSmem ts;
    ts.ent = (uint64_t *)base;
    uint8_t *p = base + (size_t)(max_entries > 0 ? max_entries : 1) * sizeof(uint64_t);
    ts.off = (uint32_t *)p;
    p += (d_K + 1) * sizeof(uint32_t);
    ts.pk = (uint32_t *)p;
    p += kTF * sizeof(uint32_t);
    ts.hi = (uint32_t *)p;
    p += kTF * sizeof(uint32_t);
    ts.coef = (float *)p;
    p += kTF * sizeof(float);
    const size_t used = (size_t)(p - base);
    *rest = (float *)(base + (used + 15) / 16 * 16);
    return ts;
}

// dq partials of one feature tile of one head over the tokens [t0, t0 + T):
// forward over the chunks with the tile's rows of S = sum phi(k) u^T.
template <int DV>
__global__ void __launch_bounds__(kThreads, DV <= 64 ? 2 : 1)   // two CTAs per SM where shared memory allows
bwd_q_scan_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                  const __nv_bfloat16 *__restrict__ v, const float *__restrict__ r,
                  float *__restrict__ state, const uint32_t *__restrict__ packed,
                  const uint32_t *__restrict__ packed_hi, const float *__restrict__ coef,
                  const uint32_t *__restrict__ jac_off, const uint64_t *__restrict__ jac_ent, int d_K,
                  int max_entries, int ncomp, int64_t F, int64_t N, int64_t t0, int T, int Tseg,
                  int load_state, float *__restrict__ partials) {
    constexpr int DV1 = DV + 1, KC = mma32::cols8(DV1);
    constexpr int WS = mma32::stride_g(DV1), WA = mma32::stride_g(DV1), WB = mma32::stride_c(DV1);
    constexpr int FC = mma32::kFeatC;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int DK1 = d_K + 1;
    float *fs;
    const TileSmem ts = carve_tables(smem_raw, d_K, max_entries, &fs);
    float *Sx = fs;                    // [kTF][WS]  state rows, zero padded
    float *xq = Sx + kTF * WS;         // [kL][DK1]
    float *xk = xq + kL * DK1;
    float *xr = xk + kL * DK1;         // [kL][WA]   r rows (contraction operand)
    float *xu = xr + kL * WA;          // [kL][WB]   u rows (update operand)
    float *phik = xu + kL * WB;        // [kL][FC]
    float *val = phik + kL * FC;       // [kL][FC]

    const int64_t bh = blockIdx.x;
    const int BH = gridDim.x;
    const int tile = blockIdx.y, ntiles = gridDim.y;
    const int nf = (int)((F - tile + ntiles - 1) / ntiles);
    const int tid = threadIdx.x;
    load_tile(ts, packed, packed_hi, coef, jac_off, jac_ent, tile, ntiles, nf, d_K);
    for (int e = tid; e < kTF * WS; e += kThreads) {
        const int m = e / WS, j = e % WS;
        Sx[e] = (load_state && m < nf && j < DV1) ? state[(bh * F + tile + (int64_t)m * ntiles) * DV1 + j] : 0.f;
    }
    for (int c0 = 0; c0 < T; c0 += kL) {
        const int nt = min(kL, T - c0);
        __syncthreads();
        load_chunk(q, k, v, r, bh * N + t0 + c0, nt, d_K, DV, xq, xk, xu, WB, xr, WA);
        __syncthreads();
        for (int e = tid; e < kL * kTF; e += kThreads) {
            const int t = e / kTF, m = e % kTF;
            phik[t * FC + m] = (t < nt && m < nf) ? feature(xk + t * DK1, ts.pk[m], ts.hi[m]) : 0.f;
        }
        mma32::contract_rows<KC>(Sx, WS, xr, WA, ts.coef, val, FC);   // a (.) S r_t (zero rows past nt)
        __syncthreads();
        jac_chunk(ts.off, ts.ent, xq, DK1, val, FC, ncomp, d_K, nt,
                  partials + (((int64_t)tile * BH + bh) * Tseg + c0) * d_K, d_K);
        mma32::update_rows<KC / 8>(Sx, WS, phik, FC, xu, WB);        // S += phi(K)^T U
    }
    __syncthreads();
    for (int e = tid; e < nf * DV1; e += kThreads) {
        const int m = e / DV1, j = e % DV1;
        state[(bh * F + tile + (int64_t)m * ntiles) * DV1 + j] = Sx[m * WS + j];
    }
}

// dk and dv partials of one feature tile of one head over the tokens
// [t0, t0 + T): backward over the chunks with the tile's rows of
// G = sum phi(q) r^T over the tokens after the chunk.
template <int DV>
__global__ void __launch_bounds__(kThreads, DV <= 64 ? 2 : 1)
bwd_kv_scan_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ v, const float *__restrict__ r,
                   float *__restrict__ state, const uint32_t *__restrict__ packed,
                   const uint32_t *__restrict__ packed_hi, const float *__restrict__ coef,
                   const uint32_t *__restrict__ jac_off, const uint64_t *__restrict__ jac_ent, int d_K,
                   int max_entries, int ncomp, int64_t F, int64_t N, int64_t t0, int T, int Tseg,
                   int load_state, float *__restrict__ partials) {
    constexpr int DV1 = DV + 1, KC = mma32::cols8(DV1);
    constexpr int WS = mma32::stride_g(DV1), WA = mma32::stride_g(DV1), WB = mma32::stride_c(DV1);
    constexpr int FC = mma32::kFeatC, FG = mma32::kFeatG;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int DK1 = d_K + 1, DKV = d_K + DV;
    float *fs;
    const TileSmem ts = carve_tables(smem_raw, d_K, max_entries, &fs);
    float *Gx = fs;                    // [kTF][WS]  G rows, zero padded
    float *xq = Gx + kTF * WS;         // [kL][DK1]
    float *xk = xq + kL * DK1;
    float *xu = xk + kL * DK1;         // [kL][WA]   u rows (contraction operand)
    float *xr = xu + kL * WA;          // [kL][WB]   r rows (update operand)
    float *pka = xr + kL * WB;         // [kL][FG]   a (.) phi(k)
    float *val = pka + kL * FG;        // [kL][FC]   a (.) G u, then phi(q)

    const int64_t bh = blockIdx.x;
    const int BH = gridDim.x;
    const int tile = blockIdx.y, ntiles = gridDim.y;
    const int nf = (int)((F - tile + ntiles - 1) / ntiles);
    const int tid = threadIdx.x;
    load_tile(ts, packed, packed_hi, coef, jac_off, jac_ent, tile, ntiles, nf, d_K);
    for (int e = tid; e < kTF * WS; e += kThreads) {
        const int m = e / WS, j = e % WS;
        Gx[e] = (load_state && m < nf && j < DV1) ? state[(bh * F + tile + (int64_t)m * ntiles) * DV1 + j] : 0.f;
    }
    const int nchunks = (T + kL - 1) / kL;
    for (int ci = nchunks - 1; ci >= 0; --ci) {
        const int c0 = ci * kL;
        const int nt = min(kL, T - c0);
        __syncthreads();
        load_chunk(q, k, v, r, bh * N + t0 + c0, nt, d_K, DV, xq, xk, xu, WA, xr, WB);
        __syncthreads();
        for (int e = tid; e < kL * kTF; e += kThreads) {
            const int t = e / kTF, m = e % kTF;
            pka[t * FG + m] = (t < nt && m < nf) ? ts.coef[m] * feature(xk + t * DK1, ts.pk[m], ts.hi[m]) : 0.f;
        }
        mma32::contract_rows<KC>(Gx, WS, xu, WA, ts.coef, val, FC);   // a (.) G u_s
        __syncthreads();
        jac_chunk(ts.off, ts.ent, xk, DK1, val, FC, ncomp, d_K, nt,
                  partials + (((int64_t)tile * BH + bh) * Tseg + c0) * DKV, DKV);
        // dv partial: (a (.) phi(k_s))^T G[:, :d_V]
        float *dvp = partials + (((int64_t)tile * BH + bh) * Tseg + c0) * DKV + d_K;
        mma32::readout_cols<mma32::cols8(DV) / 8>(pka, FG, Gx, WS, [&](int t, int j, float x) {
            if (t < nt && j < DV) __stcs(dvp + (int64_t)t * DKV + j, x);
        });
        __syncthreads();
        for (int e = tid; e < kL * kTF; e += kThreads) {   // phi(q) over the consumed values
            const int t = e / kTF, m = e % kTF;
            val[t * FC + m] = (t < nt && m < nf) ? feature(xq + t * DK1, ts.pk[m], ts.hi[m]) : 0.f;
        }
        __syncthreads();
        mma32::update_rows<KC / 8>(Gx, WS, val, FC, xr, WB);         // G += phi(Q)^T R
    }
    __syncthreads();
    for (int e = tid; e < nf * DV1; e += kThreads) {
        const int m = e / DV1, j = e % DV1;
        state[(bh * F + tile + (int64_t)m * ntiles) * DV1 + j] = Gx[m * WS + j];
    }
}

// Per chunk: sum the tiles' partials in tile order and add the pairs inside the
// chunk.  KV = false: dq (partials [tile][BH][Tseg][d_K]); KV = true: dk and dv
// (partials [tile][BH][Tseg][d_K + d_V]).
template <bool KV>
__global__ void __launch_bounds__(kThreads)
bwd_finish_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                  const __nv_bfloat16 *__restrict__ v, const float *__restrict__ r,
                  const float *__restrict__ partials, int ntiles, int d_K, int d_V, int P, float inv_c,
                  int64_t N, int64_t t0, int T, int Tseg, float *__restrict__ dqk,
                  float *__restrict__ dv) {
    extern __shared__ float smem[];
    const int DV1 = d_V + 1;
    const int PW = KV ? d_K + d_V : d_K;   // partial row width
    float *xq = smem;                  // [kL][d_K]
    float *xk = xq + kL * d_K;
    float *xu = xk + kL * d_K;         // [kL][DV1]
    float *xr = xu + kL * DV1;
    float *Wd = xr + kL * DV1;         // [kL][kL]  dx_ts / c
    float *Ww = Wd + kL * kL;          // [kL][kL]  w_ts

    const int64_t bh = blockIdx.x;
    const int BH = gridDim.x;
    const int c0 = blockIdx.y * kL;
    const int nt = min(kL, T - c0);
    const int64_t row0 = bh * N + t0 + c0;
    const int tid = threadIdx.x;
    for (int e = tid; e < kL * d_K; e += kThreads) {
        const int t = e / d_K, i = e % d_K;
        float a = 0.f, b = 0.f;
        if (t < nt) {
            a = __bfloat162float(q[(row0 + t) * d_K + i]);
            b = __bfloat162float(k[(row0 + t) * d_K + i]);
        }
        xq[e] = a;
        xk[e] = b;
    }
    for (int e = tid; e < kL * DV1; e += kThreads) {
        const int t = e / DV1, j = e % DV1;
        float a = 0.f, b = 0.f;
        if (t < nt) {
            a = j < d_V ? __bfloat162float(v[(row0 + t) * d_V + j]) : 1.f;
            b = r[(row0 + t) * r_stride(d_V) + j];
        }
        xu[e] = a;
        xr[e] = b;
    }
    __syncthreads();
    for (int e = tid; e < kL * kL; e += kThreads) {
        const int t = e / kL, s = e % kL;
        float wd = 0.f, w = 0.f;
        if (t < nt && s <= t) {
            float x = 0.f;
            for (int i = 0; i < d_K; ++i) x = fmaf(xq[t * d_K + i], xk[s * d_K + i], x);
            x *= inv_c;
            // T_P(x) = sum_{p<P} x^p / p! and its derivative T_{P-1}(x) (T_0 = 0)
            const float h = simt::taylor_exp(x, P);
            const float hd = simt::taylor_exp(x, P - 1);
            float dw = 0.f;
            for (int j = 0; j < DV1; ++j) dw = fmaf(xr[t * DV1 + j], xu[s * DV1 + j], dw);
            wd = dw * hd * inv_c;
            w = h;
        }
        Wd[e] = wd;
        Ww[e] = w;
    }
    __syncthreads();
    for (int e = tid; e < nt * d_K; e += kThreads) {
        const int t = e / d_K, i = e % d_K;
        const float a = simt::sum_strided(partials + ((int64_t)bh * Tseg + c0 + t) * PW + i, ntiles,
                                          (int64_t)BH * Tseg * PW);
        float b = 0.f;
        if (!KV) {
            for (int s = 0; s <= t; ++s) b = fmaf(Wd[t * kL + s], xk[s * d_K + i], b);
        } else {   // row t is the key token s here
            for (int u = t; u < nt; ++u) b = fmaf(Wd[u * kL + t], xq[u * d_K + i], b);
        }
        dqk[(row0 + t) * d_K + i] = a + b;
    }
    if (KV) {
        for (int e = tid; e < nt * d_V; e += kThreads) {
            const int s = e / d_V, j = e % d_V;
            const float a = simt::sum_strided(partials + ((int64_t)bh * Tseg + c0 + s) * PW + d_K + j, ntiles,
                                              (int64_t)BH * Tseg * PW);
            float b = 0.f;
            for (int u = s; u < nt; ++u) b = fmaf(Ww[u * kL + s], xr[u * DV1 + j], b);
            dv[(row0 + s) * d_V + j] = a + b;
        }
    }
}

int64_t segment_tokens(int BH, int64_t N, int64_t F, int d_K, int d_V) {
    const int64_t ntiles = (F + kTF - 1) / kTF;
    const int64_t per_token = ntiles * BH * (d_K + d_V) * (int64_t)sizeof(float);
    int64_t T = (int64_t)(kPartialBudget / (size_t)per_token) / kL * kL;
    if (T < kL) T = kL;
    if (T > (int64_t)65535 * kL) T = (int64_t)65535 * kL;   // finish kernels' grid.y
    const int64_t Nr = (N + kL - 1) / kL * kL;
    return T < Nr ? T : Nr;
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

struct BwdLayout {
    int64_t Tseg = 0;
    size_t fwd = 0, part = 0, off_state = 0, off_y = 0, off_den = 0, off_r = 0, total = 0;
};

BwdLayout bwd_layout(int BH, int64_t N, int64_t F, int d_K, int d_V, int P, bool use_tc) {
    BwdLayout L;
    const int64_t ntiles = (F + kTF - 1) / kTF;
    L.Tseg = segment_tokens(BH, N, F, d_K, d_V);
    L.fwd = use_tc ? prefill_tc_workspace_bytes(BH, N, F, d_K, d_V, P, true, false)
                   : prefill_simt_workspace_bytes(BH, N, F, d_V, true);
    L.part = round256((size_t)ntiles * BH * L.Tseg * (d_K + d_V) * sizeof(float));
    const size_t front = L.fwd > L.part ? L.fwd : L.part;   // the forward's workspace, then the partials
    L.off_state = round256(front);
    L.off_y = L.off_state + round256((size_t)BH * F * (d_V + 1) * sizeof(float));
    L.off_den = L.off_y + round256((size_t)BH * N * d_V * sizeof(float));
    L.off_r = L.off_den + round256((size_t)BH * N * sizeof(float));
    L.total = L.off_r + round256((size_t)BH * N * r_stride(d_V) * sizeof(float));
    return L;
}

using ScanFn = void (*)(const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *, const float *,
                       float *, const uint32_t *, const uint32_t *, const float *, const uint32_t *,
                       const uint64_t *, int, int, int, int64_t, int64_t, int64_t, int, int, int, float *);

// The scan kernels are compiled per d_V (register tiles sized at compile time).
bool scan_kernels(int d_V, ScanFn *fq, ScanFn *fkv) {
    switch (d_V) {
        case 4: *fq = bwd_q_scan_kernel<4>; *fkv = bwd_kv_scan_kernel<4>; return true;
        case 8: *fq = bwd_q_scan_kernel<8>; *fkv = bwd_kv_scan_kernel<8>; return true;
        case 16: *fq = bwd_q_scan_kernel<16>; *fkv = bwd_kv_scan_kernel<16>; return true;
        case 32: *fq = bwd_q_scan_kernel<32>; *fkv = bwd_kv_scan_kernel<32>; return true;
        case 64: *fq = bwd_q_scan_kernel<64>; *fkv = bwd_kv_scan_kernel<64>; return true;
        case 128: *fq = bwd_q_scan_kernel<128>; *fkv = bwd_kv_scan_kernel<128>; return true;
        default: return false;
    }
}

}  // namespace

// The gradient scans run on tensor cores (backward_tc.cuh) where the forward does,
// unless the fixed-order mode asks for bitwise repeatable results (their sums use
// atomics); elsewhere on the CUDA-core scans below.
static bool backward_on_tc(int d_K, int d_V, int P, bool use_tc) {
    return use_tc && g_opt_deterministic == 0 && prefill_backward_tc_supported(d_K, d_V, P);
}

size_t prefill_backward_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P, bool use_tc) {
    if (backward_on_tc(d_K, d_V, P, use_tc)) return prefill_backward_tc_workspace_bytes(BH, N, F, d_K, d_V, P);
    return bwd_layout(BH, N, F, d_K, d_V, P, use_tc).total;
}

cudaError_t launch_prefill_backward(const DeviceBasis &basis, int BH, int64_t N, int d_V,
                                    const void *q, const void *k, const void *v, const float *dy,
                                    float *dq, float *dk, float *dv, void *ws, size_t ws_bytes,
                                    bool use_tc, int *flags, cudaStream_t stream) {
    const int d_K = basis.d_K, P = basis.P;
    const int64_t F = basis.F;
    if (backward_on_tc(d_K, d_V, P, use_tc))
        return launch_prefill_backward_tc(basis, BH, N, d_V, q, k, v, dy, dq, dk, dv, ws, ws_bytes, flags, stream);
    const BwdLayout L = bwd_layout(BH, N, F, d_K, d_V, P, use_tc);
    if (ws_bytes < L.total) return cudaErrorInvalidValue;
    const int ntiles = (int)((F + kTF - 1) / kTF);
    const int ncomp = P > 2 ? P - 2 : 0;
    cudaError_t e = cudaSuccess;
    ScanFn q_scan = nullptr, kv_scan = nullptr;
    if (!scan_kernels(d_V, &q_scan, &kv_scan)) return cudaErrorInvalidValue;
    size_t off_ent = 0;
    int max_ent = 0;
    const uint8_t *jt = jac_table(d_K, P, &off_ent, &max_ent, &e);
    if (!jt) return e != cudaSuccess ? e : cudaErrorMemoryAllocation;
    const uint32_t *jac_off = (const uint32_t *)jt;
    const uint64_t *jac_ent = (const uint64_t *)(jt + off_ent);

    uint8_t *w = (uint8_t *)ws;
    float *partials = (float *)w;
    float *state = (float *)(w + L.off_state);
    float *y = (float *)(w + L.off_y);
    float *den = (float *)(w + L.off_den);
    float *r = (float *)(w + L.off_r);
    const __nv_bfloat16 *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k,
                        *vb = (const __nv_bfloat16 *)v;

    // forward: y and den (fresh state, carried in the front region), on tensor cores where the
    // prefill runs there
    e = use_tc ? launch_prefill_tc(basis, BH, N, d_V, q, k, v, y, nullptr, nullptr, false, ws, L.fwd, flags,
                                   stream, nullptr, den)
               : launch_prefill_simt(basis, BH, N, d_V, q, k, v, y, nullptr, nullptr, false, ws, L.fwd, stream,
                                     den);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)BH * N;
    launch_begin(kBwdR, stream);
    bwd_r_kernel<<<(unsigned)((rows + kThreads / 32 - 1) / (kThreads / 32)), kThreads, 0, stream>>>(
        dy, y, den, r, d_V, rows);
    launch_end(kBwdR, stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const size_t smemQ = ScanSmem::bytes(d_K, d_V, false, max_ent);
    const size_t smemKV = ScanSmem::bytes(d_K, d_V, true, max_ent);
    const size_t smemF = sizeof(float) * ((size_t)2 * kL * d_K + 2 * kL * (d_V + 1) + 2 * kL * kL);
    if ((e = cudaFuncSetAttribute(q_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smemQ)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kv_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smemKV)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(bwd_finish_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smemF)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(bwd_finish_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smemF)) != cudaSuccess)
        return e;
    const float inv_c = 1.0f / sqrtf((float)d_K);
    const int64_t Tseg = L.Tseg;
    const int nseg = (int)((N + Tseg - 1) / Tseg);

    // dq: segments in order, S carried forward
    for (int sg = 0; sg < nseg; ++sg) {
        const int64_t t0 = (int64_t)sg * Tseg;
        const int T = (int)(N - t0 < Tseg ? N - t0 : Tseg);
        launch_begin(kBwdQScan, stream);
        q_scan<<<dim3(BH, ntiles), kThreads, smemQ, stream>>>(
            qb, kb, vb, r, state, basis.packed, basis.packed_hi, basis.coef, jac_off, jac_ent, d_K, max_ent,
            ncomp, F, N, t0, T, (int)Tseg, sg > 0 ? 1 : 0, partials);
        launch_end(kBwdQScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        launch_begin(kBwdFinish, stream);
        bwd_finish_kernel<false><<<dim3(BH, (T + kL - 1) / kL), kThreads, smemF, stream>>>(
            qb, kb, vb, r, partials, ntiles, d_K, d_V, P, inv_c, N, t0, T, (int)Tseg, dq, nullptr);
        launch_end(kBwdFinish, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // dk, dv: segments in reverse, G carried backward
    for (int sg = nseg - 1; sg >= 0; --sg) {
        const int64_t t0 = (int64_t)sg * Tseg;
        const int T = (int)(N - t0 < Tseg ? N - t0 : Tseg);
        launch_begin(kBwdKVScan, stream);
        kv_scan<<<dim3(BH, ntiles), kThreads, smemKV, stream>>>(
            qb, kb, vb, r, state, basis.packed, basis.packed_hi, basis.coef, jac_off, jac_ent, d_K, max_ent,
            ncomp, F, N, t0, T, (int)Tseg, sg < nseg - 1 ? 1 : 0, partials);
        launch_end(kBwdKVScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        launch_begin(kBwdFinish, stream);
        bwd_finish_kernel<true><<<dim3(BH, (T + kL - 1) / kL), kThreads, smemF, stream>>>(
            qb, kb, vb, r, partials, ntiles, d_K, d_V, P, inv_c, N, t0, T, (int)Tseg, dk, dv);
        launch_end(kBwdFinish, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace sata
