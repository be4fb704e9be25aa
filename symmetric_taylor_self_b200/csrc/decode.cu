// Decode step: one token per head against the fixed-size state.
//
// [CC-TAYLOR] "Self-attention at constant cost per token via symmetry-aware
// Taylor approximation", section "Feature maps and linear attention"
// (特征映射与线性注意力): Z_T = Z_{T-1} + phi(k_T), S_T = S_{T-1} + phi(k_T) v_T^T,
// y_T = sum_p alpha_p phi_p(q_T)^T C_p S_p / sum_p alpha_p <phi_p(q_T), Z_p>_C.
// [CC-HW] "Constant-cost attention: hardware optimization", section "Fixed-size
// hidden state": the per-token cost is set by the state size, not the context.
//
// The step is bound by HBM: every state value is read once and written once
// (8 bytes per value).  Work split: CTA (g, bh) owns features
// [g*FG, (g+1)*FG) of head bh; it computes phi(k) and alpha*C*phi(q) for them
// in shared memory, then streams the S rows with 16-byte loads/stores (d_V/4
// threads per row), updating and reading in one pass.  Per-CTA partial
// numerators/denominators go to a small workspace and a second kernel sums
// them in a fixed order and divides (deterministic).
#include <cuda_bf16.h>

#include "sata_internal.h"

namespace sata {
namespace {

constexpr int kThreads = 256;
constexpr int kFG = 1024;  // features per CTA

__device__ __forceinline__ float4 fma4(float a, float4 x, float4 y) {
    return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}

template <int DV>
__global__ void __launch_bounds__(kThreads)
decode_stream_kernel(float *__restrict__ S, float *__restrict__ Z,
                     const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                     const __nv_bfloat16 *__restrict__ v, const uint32_t *__restrict__ packed,
                     const uint32_t *__restrict__ packed_hi, const float *__restrict__ coef, int d_K,
                     int64_t F, float *__restrict__ partials) {
    constexpr int TPR = DV / 4;              // threads per state row, one float4 each
    constexpr int RPI = kThreads / TPR;      // rows per block iteration
    constexpr int kWarps = kThreads / 32;
    __shared__ float xq[kMaxDK + 1], xk[kMaxDK + 1], xv[DV];
    __shared__ float phik[kFG], aq[kFG];
    __shared__ float red[kWarps][DV + 1];

    const int g = blockIdx.y, G = gridDim.y;
    const int64_t bh = blockIdx.x;
    const int64_t f0 = (int64_t)g * kFG;
    const int nf = (int)(F - f0 < (int64_t)kFG ? F - f0 : (int64_t)kFG);
    const int tid = threadIdx.x;

    // x[d_K] = 1 is the padding index of the packed basis.
    for (int i = tid; i <= d_K; i += kThreads) {
        xq[i] = i < d_K ? __bfloat162float(q[bh * d_K + i]) : 1.0f;
        xk[i] = i < d_K ? __bfloat162float(k[bh * d_K + i]) : 1.0f;
    }
    for (int i = tid; i < DV; i += kThreads) xv[i] = __bfloat162float(v[bh * DV + i]);
    __syncthreads();
    for (int f = tid; f < nf; f += kThreads) {
        const uint32_t pk = packed[f0 + f];
        const int a = pk & 255, b = (pk >> 8) & 255, l = (pk >> 16) & 255;
        float fk = xk[a] * xk[b] * xk[l], fq = xq[a] * xq[b] * xq[l];
        if (packed_hi) {   // degrees above 3: the leading indices
            const uint32_t ph = packed_hi[f0 + f];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = (ph >> (8 * m)) & 255;
                fk *= xk[i];
                fq *= xq[i];
            }
        }
        phik[f] = fk;
        aq[f] = coef[f0 + f] * fq;
    }
    __syncthreads();

    // S rows: update then read (inclusive causal range).
    const int col = tid % TPR;
    const int r0 = tid / TPR;
    const float4 vv = make_float4(xv[4 * col], xv[4 * col + 1], xv[4 * col + 2], xv[4 * col + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 *Sb = reinterpret_cast<float4 *>(S + (bh * F + f0) * DV);
    int r = r0;
    for (; r + 3 * RPI < nf; r += 4 * RPI) {
        float4 s[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) s[u] = Sb[(int64_t)(r + u * RPI) * TPR + col];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int rr = r + u * RPI;
            s[u] = fma4(phik[rr], vv, s[u]);
            Sb[(int64_t)rr * TPR + col] = s[u];
            acc = fma4(aq[rr], s[u], acc);
        }
    }
    for (; r < nf; r += RPI) {
        float4 s = Sb[(int64_t)r * TPR + col];
        s = fma4(phik[r], vv, s);
        Sb[(int64_t)r * TPR + col] = s;
        acc = fma4(aq[r], s, acc);
    }
    // Z entries: the "+1" column of the state.
    float dacc = 0.f;
    float *Zb = Z + bh * F + f0;
    for (int f = tid; f < nf; f += kThreads) {
        const float z = Zb[f] + phik[f];
        Zb[f] = z;
        dacc = fmaf(aq[f], z, dacc);
    }

    // Reduce: lanes with equal `col` are TPR apart inside a warp.
#pragma unroll
    for (int off = TPR; off < 32; off <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dacc += __shfl_xor_sync(0xffffffffu, dacc, off);
    const int warp = tid / 32, lane = tid % 32;
    if (lane < TPR) {
        red[warp][4 * lane + 0] = acc.x;
        red[warp][4 * lane + 1] = acc.y;
        red[warp][4 * lane + 2] = acc.z;
        red[warp][4 * lane + 3] = acc.w;
    }
    if (lane == 0) red[warp][DV] = dacc;
    __syncthreads();
    for (int j = tid; j <= DV; j += kThreads) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][j];
        partials[(bh * G + g) * (DV + 1) + j] = s;
    }
}

template <int DV>
__global__ void decode_finish_kernel(const float *__restrict__ partials, int G,
                                     float *__restrict__ out) {
    __shared__ float den;
    const int64_t bh = blockIdx.x;
    const int j = threadIdx.x;
    float s = 0.f;
    if (j <= DV)
        for (int g = 0; g < G; ++g) s += partials[(bh * G + g) * (DV + 1) + j];
    if (j == DV) den = s;
    __syncthreads();
    if (j < DV) out[bh * DV + j] = s / den;
}

template <int DV>
cudaError_t launch_dv(const DeviceBasis &basis, int BH, float *S, float *Z, const void *q,
                      const void *k, const void *v, float *out, float *partials,
                      cudaStream_t stream) {
    const int G = (int)((basis.F + kFG - 1) / kFG);
    dim3 grid(BH, G);
    launch_begin(kDecodeStream, stream);
    decode_stream_kernel<DV><<<grid, kThreads, 0, stream>>>(
        S, Z, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
        basis.packed, basis.packed_hi, basis.coef, basis.d_K, basis.F, partials);
    launch_end(kDecodeStream, stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int threads = ((DV + 1 + 31) / 32) * 32;
    launch_begin(kDecodeFinish, stream);
    decode_finish_kernel<DV><<<BH, threads, 0, stream>>>(partials, G, out);
    launch_end(kDecodeFinish, stream);
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(int BH, int64_t F, int d_V) {
    const int64_t G = (F + kFG - 1) / kFG;
    return (size_t)BH * (size_t)G * (size_t)(d_V + 1) * sizeof(float);
}

cudaError_t launch_decode(const DeviceBasis &basis, int BH, int d_V, float *S, float *Z,
                          const void *q, const void *k, const void *v, float *out,
                          float *partials, cudaStream_t stream) {
    switch (d_V) {
        case 4: return launch_dv<4>(basis, BH, S, Z, q, k, v, out, partials, stream);
        case 8: return launch_dv<8>(basis, BH, S, Z, q, k, v, out, partials, stream);
        case 16: return launch_dv<16>(basis, BH, S, Z, q, k, v, out, partials, stream);
        case 32: return launch_dv<32>(basis, BH, S, Z, q, k, v, out, partials, stream);
        case 64: return launch_dv<64>(basis, BH, S, Z, q, k, v, out, partials, stream);
        case 128: return launch_dv<128>(basis, BH, S, Z, q, k, v, out, partials, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sata
