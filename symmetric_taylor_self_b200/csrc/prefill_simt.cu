// Prefill on CUDA cores (fp32 throughout): the chunked form of the recurrence.
//
// [CC-TAYLOR] "Self-attention at constant cost per token via symmetry-aware
// Taylor approximation", section "Feature maps and linear attention"
// (特征映射与线性注意力): the states obey Z_T = Z_{T-1} + phi(k_T),
// S_T = S_{T-1} + phi(k_T) v_T^T and may be computed sequentially or by a
// parallel prefix scan.  Chunked form used here, for chunk c of L tokens:
//   inter-chunk: y-numerator/denominator of token t in chunk c gets
//                alpha*C*phi(q_t) . [S | Z]_{c-1}        (state before chunk c)
//   intra-chunk: sum_{s in chunk c, s <= t} w_ts [v_s | 1],
//                w_ts = sum_{p<P} (q_t.k_s / c)^p / p!  (the same kernel, by the
//                identity (q.k)^p = <phi_p(q), phi_p(k)>_C of the same section)
//   update:      [S | Z]_c = [S | Z]_{c-1} + phi(K_c)^T [V_c | 1].
// The feature dimension is split into tiles of kTF features, one CTA each; the
// inter-chunk partials of all tiles are summed in a fixed order by the second
// kernel, which adds the intra-chunk part and divides (deterministic).  The
// sequence is processed in segments so the partial buffer stays bounded; the
// state carries across segments in global memory.
//
// This path is general (any supported d_K, d_V, P) and exact to fp32; the
// tensor-core path (prefill_tc.cu) is the fast one.  The token rows are bf16, or
// fp32 (sata_prefill_f32: no input rounding at all).
#include <cuda_bf16.h>

#include "sata_internal.h"
#include "simt_tiles.cuh"

namespace sata {
namespace {

using simt::kThreads;
using simt::kTF;
using simt::kL;
constexpr size_t kPartialBudget = size_t(2) << 30;  // bytes of partials per segment

struct SimtSmem {
    static size_t bytes(int d_K, int d_V) {
        const size_t DK1 = d_K + 1, DV1 = d_V + 1;
        return sizeof(float) * ((size_t)kTF * DV1 + 2 * kL * DK1 + kL * DV1 + 2 * (size_t)kL * kTF);
    }
};

// Kernel A: inter-chunk readout partials and state update for one feature tile
// of one head over the tokens [t0, t0 + T) of a segment (compiled per d_V: the
// two contractions are register-tiled, simt_tiles.cuh; TI: the rows' type).
template <int DV, typename TI>
__global__ void __launch_bounds__(kThreads)
simt_scan_kernel(const TI *__restrict__ q, const TI *__restrict__ k, const TI *__restrict__ v, float *__restrict__ S,
                 float *__restrict__ Z, const uint32_t *__restrict__ packed,
                 const uint32_t *__restrict__ packed_hi, const float *__restrict__ coef, int d_K,
                 int64_t F, int64_t N,
                 int64_t t0, int T, int Tseg, int load_state, float *__restrict__ partials) {
    constexpr int d_V = DV, DV1 = DV + 1;
    extern __shared__ float smem[];
    const int DK1 = d_K + 1;
    float *Sx = smem;                       // [kTF][DV1]
    float *xq = Sx + kTF * DV1;             // [kL][DK1]
    float *xk = xq + kL * DK1;              // [kL][DK1]
    float *xv = xk + kL * DK1;              // [kL][DV1]
    float *phik = xv + kL * DV1;            // [kL][kTF]
    float *aq = phik + kL * kTF;            // [kL][kTF]

    const int64_t bh = blockIdx.x;
    const int tile = blockIdx.y, ntiles = gridDim.y;
    const int64_t f0 = (int64_t)tile * kTF;
    const int nf = (int)(F - f0 < (int64_t)kTF ? F - f0 : (int64_t)kTF);
    const int tid = threadIdx.x;

    // initial state of this tile
    for (int e = tid; e < kTF * DV1; e += kThreads) {
        const int f = e / DV1, j = e % DV1;
        float s = 0.f;
        if (load_state && f < nf)
            s = (j < d_V) ? S[(bh * F + f0 + f) * d_V + j] : Z[bh * F + f0 + f];
        Sx[e] = s;
    }

    for (int c0 = 0; c0 < T; c0 += kL) {
        const int nt = min(kL, T - c0);
        __syncthreads();
        simt::load_qkv_chunk(q, k, v, bh * N + t0 + c0, nt, d_K, d_V, xq, xk, xv);
        __syncthreads();
        for (int e = tid; e < kL * kTF; e += kThreads) {
            const int t = e / kTF, f = e % kTF;
            float pk = 0.f, pq = 0.f;
            if (t < nt && f < nf) {
                const uint32_t w = packed[f0 + f];
                const int a = w & 255, b = (w >> 8) & 255, l = (w >> 16) & 255;
                pk = xk[t * DK1 + a] * xk[t * DK1 + b] * xk[t * DK1 + l];
                float fq = xq[t * DK1 + a] * xq[t * DK1 + b] * xq[t * DK1 + l];
                if (packed_hi) {   // degrees above 3: the leading indices
                    const uint32_t wh = packed_hi[f0 + f];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int i = (wh >> (8 * m)) & 255;
                        pk *= xk[t * DK1 + i];
                        fq *= xq[t * DK1 + i];
                    }
                }
                pq = coef[f0 + f] * fq;
            }
            phik[e] = pk;
            aq[e] = pq;
        }
        __syncthreads();
        {   // readout against the state before this chunk (rows past nf are zero)
            constexpr int JV = (DV1 + 31) / 32;
            float acc[4][JV];
            simt::readout_cols<JV, DV1>(aq, Sx, DV1, acc);
            const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int t = warp + 8 * b;
#pragma unroll
                for (int n = 0; n < JV; ++n) {
                    const int j = lane + 32 * n;
                    if (t < nt && j < DV1)
                        partials[(((int64_t)tile * gridDim.x + bh) * Tseg + c0 + t) * DV1 + j] = acc[b][n];
                }
            }
        }
        __syncthreads();
        simt::update_rows<DV1>(Sx, phik, xv, nt);   // update with this chunk
    }
    __syncthreads();
    for (int e = tid; e < nf * DV1; e += kThreads) {
        const int f = e / DV1, j = e % DV1;
        if (j < d_V) S[(bh * F + f0 + f) * d_V + j] = Sx[e];
        else Z[bh * F + f0 + f] = Sx[e];
    }
    (void)ntiles;
}

// Kernel B: per chunk, sum the tiles' inter-chunk partials, add the intra-chunk
// block and divide.
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_finish_kernel(const TI *__restrict__ q, const TI *__restrict__ k, const TI *__restrict__ v,
                   const float *__restrict__ partials,
                   int ntiles, int d_K, int d_V, int P, float inv_c, int64_t N, int64_t t0,
                   int T, int Tseg, float *__restrict__ out, float *__restrict__ den_out) {
    extern __shared__ float smem[];
    const int DV1 = d_V + 1;
    float *xq = smem;                  // [kL][d_K]
    float *xk = xq + kL * d_K;         // [kL][d_K]
    float *xv = xk + kL * d_K;         // [kL][DV1]
    float *W = xv + kL * DV1;          // [kL][kL]
    float *acc = W + kL * kL;          // [kL][DV1]

    const int64_t bh = blockIdx.x;
    const int c0 = blockIdx.y * kL;
    const int nt = min(kL, T - c0);
    const int BH = gridDim.x;
    const int tid = threadIdx.x;
    for (int e = tid; e < kL * d_K; e += kThreads) {
        const int t = e / d_K, i = e % d_K;
        float a = 0.f, b = 0.f;
        if (t < nt) {
            const int64_t row = (bh * N + t0 + c0 + t) * d_K;
            a = simt::in_f(q[row + i]);
            b = simt::in_f(k[row + i]);
        }
        xq[e] = a;
        xk[e] = b;
    }
    for (int e = tid; e < kL * DV1; e += kThreads) {
        const int t = e / DV1, j = e % DV1;
        float a = 0.f;
        if (t < nt) a = j < d_V ? simt::in_f(v[(bh * N + t0 + c0 + t) * d_V + j]) : 1.f;
        xv[e] = a;
    }
    __syncthreads();
    for (int e = tid; e < kL * kL; e += kThreads) {
        const int t = e / kL, s = e % kL;
        float w = 0.f;
        if (t < nt && s <= t) {
            float x = 0.f;
            for (int i = 0; i < d_K; ++i) x = fmaf(xq[t * d_K + i], xk[s * d_K + i], x);
            x *= inv_c;
            w = simt::taylor_exp(x, P);   // sum_{p<P} x^p / p!
        }
        W[e] = w;
    }
    __syncthreads();
    for (int e = tid; e < nt * DV1; e += kThreads) {
        const int t = e / DV1, j = e % DV1;
        const float a = simt::sum_strided(partials + ((int64_t)bh * Tseg + c0 + t) * DV1 + j, ntiles,
                                          (int64_t)BH * Tseg * DV1);
        float b = 0.f;
        for (int s = 0; s <= t; ++s) b = fmaf(W[t * kL + s], xv[s * DV1 + j], b);
        acc[e] = a + b;
    }
    __syncthreads();
    for (int e = tid; e < nt * d_V; e += kThreads) {
        const int t = e / d_V, j = e % d_V;
        out[(bh * N + t0 + c0 + t) * d_V + j] = acc[t * DV1 + j] / acc[t * DV1 + d_V];
    }
    if (den_out)   // the denominators, for the backward pass
        for (int t = tid; t < nt; t += kThreads) den_out[bh * N + t0 + c0 + t] = acc[t * DV1 + d_V];
}

int64_t segment_tokens(int BH, int64_t N, int64_t F, int d_V) {
    const int64_t ntiles = (F + kTF - 1) / kTF;
    const int64_t per_token = ntiles * BH * (d_V + 1) * (int64_t)sizeof(float);
    int64_t T = (int64_t)(kPartialBudget / (size_t)per_token) / kL * kL;
    if (T < kL) T = kL;
    if (T > (int64_t)65535 * kL) T = (int64_t)65535 * kL;   // finish kernel's grid.y
    const int64_t Nr = (N + kL - 1) / kL * kL;
    return T < Nr ? T : Nr;
}

}  // namespace

size_t prefill_simt_workspace_bytes(int BH, int64_t N, int64_t F, int d_V, bool need_state) {
    const int64_t ntiles = (F + kTF - 1) / kTF;
    const int64_t Tseg = segment_tokens(BH, N, F, d_V);
    size_t b = (size_t)ntiles * BH * Tseg * (d_V + 1) * sizeof(float);
    b = (b + 255) / 256 * 256;
    if (need_state) b += (size_t)BH * F * (d_V + 1) * sizeof(float);
    return b;
}

namespace {
template <typename TI>
cudaError_t run_simt(const DeviceBasis &basis, int BH, int64_t N, int d_V, const TI *q, const TI *k, const TI *v,
                     float *out, float *S, float *Z, bool state_in, void *ws, size_t ws_bytes, cudaStream_t stream,
                     float *den_out) {
    const int d_K = basis.d_K;
    const int64_t F = basis.F;
    const int ntiles = (int)((F + kTF - 1) / kTF);
    const int64_t Tseg = segment_tokens(BH, N, F, d_V);
    size_t pbytes = (size_t)ntiles * BH * Tseg * (d_V + 1) * sizeof(float);
    pbytes = (pbytes + 255) / 256 * 256;
    const bool own_state = (S == nullptr);
    if (ws_bytes < prefill_simt_workspace_bytes(BH, N, F, d_V, own_state)) return cudaErrorInvalidValue;
    float *partials = (float *)ws;
    if (own_state) {  // fresh prefill: carry the state in the workspace
        S = (float *)((char *)ws + pbytes);
        Z = S + (size_t)BH * F * d_V;
        state_in = false;
    }
    using ScanFn = void (*)(const TI *, const TI *, const TI *, float *, float *, const uint32_t *,
                            const uint32_t *, const float *, int, int64_t, int64_t, int64_t, int, int, int, float *);
    ScanFn scan = nullptr;
    switch (d_V) {
        case 4: scan = simt_scan_kernel<4, TI>; break;
        case 8: scan = simt_scan_kernel<8, TI>; break;
        case 16: scan = simt_scan_kernel<16, TI>; break;
        case 32: scan = simt_scan_kernel<32, TI>; break;
        case 64: scan = simt_scan_kernel<64, TI>; break;
        case 128: scan = simt_scan_kernel<128, TI>; break;
        default: return cudaErrorInvalidValue;
    }
    const size_t smemA = SimtSmem::bytes(d_K, d_V);
    const size_t smemB = sizeof(float) * ((size_t)2 * kL * d_K + kL * (d_V + 1) + kL * kL +
                                          kL * (d_V + 1));
    cudaError_t e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smemA);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(simt_finish_kernel<TI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemB);
    if (e != cudaSuccess) return e;
    const float inv_c = 1.0f / sqrtf((float)d_K);
    for (int64_t t0 = 0; t0 < N; t0 += Tseg) {
        const int T = (int)(N - t0 < Tseg ? N - t0 : Tseg);
        const int load = (t0 > 0 || state_in) ? 1 : 0;
        launch_begin(kSimtScan, stream);
        scan<<<dim3(BH, ntiles), kThreads, smemA, stream>>>(q, k, v, S, Z, basis.packed, basis.packed_hi, basis.coef,
                                                            d_K, F, N, t0, T, (int)Tseg, load, partials);
        launch_end(kSimtScan, stream);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const int nchunks = (T + kL - 1) / kL;
        launch_begin(kSimtFinish, stream);
        simt_finish_kernel<TI><<<dim3(BH, nchunks), kThreads, smemB, stream>>>(
            q, k, v, partials, ntiles, d_K, d_V, basis.P, inv_c, N, t0, T, (int)Tseg, out, den_out);
        launch_end(kSimtFinish, stream);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
}  // namespace

cudaError_t launch_prefill_simt(const DeviceBasis &basis, int BH, int64_t N, int d_V, const void *q, const void *k,
                                const void *v, float *out, float *S, float *Z, bool state_in, void *ws,
                                size_t ws_bytes, cudaStream_t stream, float *den_out, bool f32_in) {
    if (f32_in)
        return run_simt(basis, BH, N, d_V, (const float *)q, (const float *)k, (const float *)v, out, S, Z, state_in,
                        ws, ws_bytes, stream, den_out);
    return run_simt(basis, BH, N, d_V, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
                    out, S, Z, state_in, ws, ws_bytes, stream, den_out);
}

}  // namespace sata
