// Tensor-core prefill and backward: shape dispatch to the instances of the prefill_tc_*.cuh
// and backward_tc.cuh templates
// (one prefill_tc_*.cu file per group of shapes, compiled in parallel).
#include "prefill_tc_shapes.h"
#include "sata_internal.h"

namespace sata {

// d_V = 128 holds one slot per unit (N = 129 of the MMA's 256 columns), so a unit's fixed
// work per chunk (the pair products of both sides, the handshakes) is spread over a third
// of the d_V = 64 unit's columns.  The numerator's value columns are independent and the
// denominator does not depend on v, so on the device-buffer path a d_V = 128 prefill runs
// as two d_V = 64 prefills over the two column halves of v, out and S (three slots per
// unit).  Both compute the same Z; with a caller's state the first half reads and writes a
// copy of the incoming Z, so that the second still finds it.  Returns the half width, or 0
// to run whole rows.
static int value_half(int d_K, int d_V, bool host_io) {
    return (!host_io && d_V == 128 && (d_K == 64 || d_K == 128)) ? 64 : 0;
}
// Workspace of one half; with a caller's state (need_state false) the Z copy follows it.
static size_t half_workspace(int d_K, int BH, int64_t N, int64_t F, int P, bool need_state) {
    const bool det = g_opt_deterministic != 0;
    return d_K == 64 ? tc_workspace_64_64(BH, N, F, P, need_state, 1, det)
                     : tc_workspace_128_64(BH, N, F, P, need_state, 1, det);
}
static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

bool prefill_tc_supported(int d_K, int d_V, int P) {
    if (P < 1 || P > 4) return false;
#define SATA_TC_CASE(a, b) if (d_K == a && d_V == b) return true;
    SATA_TC_SHAPES(SATA_TC_CASE)
#undef SATA_TC_CASE
    return false;
}

size_t prefill_tc_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P, bool need_state,
                                  bool host_io) {
    const int ms = host_io ? kHostSegments : 1;
    const bool det = g_opt_deterministic != 0;
    if (value_half(d_K, d_V, host_io)) {
        const size_t w = half_workspace(d_K, BH, N, F, P, need_state);
        return need_state || w == 0 ? w : round256(w) + (size_t)BH * F * sizeof(float);
    }
#define SATA_TC_CASE(a, b) \
    if (d_K == a && d_V == b) return tc_workspace_##a##_##b(BH, N, F, P, need_state, ms, det);
    SATA_TC_SHAPES(SATA_TC_CASE)
#undef SATA_TC_CASE
    return 0;
}

cudaError_t launch_prefill_tc(const DeviceBasis &basis, int BH, int64_t N, int d_V, const void *q,
                              const void *k, const void *v, float *out, float *S, float *Z, bool state_in,
                              void *ws, size_t ws_bytes, int *flags, cudaStream_t stream, const HostIO *io,
                              float *den_out) {
    if (const int h = value_half(basis.d_K, d_V, io != nullptr)) {
        const size_t wh = half_workspace(basis.d_K, BH, N, basis.F, basis.P, S == nullptr);
        if (wh == 0 || ws_bytes < wh) return cudaErrorInvalidValue;
        float *zc = nullptr;   // the first half's copy of the incoming Z
        if (S) {
            const size_t zb = (size_t)BH * basis.F * sizeof(float);
            if (ws_bytes < round256(wh) + zb) return cudaErrorInvalidValue;
            zc = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + round256(wh));
            if (state_in) {
                const cudaError_t e = cudaMemcpyAsync(zc, Z, zb, cudaMemcpyDeviceToDevice, stream);
                if (e != cudaSuccess) return e;
            }
        }
        // base pointers stay those of the whole rows (the v maximum reads whole rows)
        for (int voff = 0; voff < d_V; voff += h) {
            float *Zh = (S && voff + h < d_V) ? zc : Z;
            cudaError_t e = basis.d_K == 64 ? tc_run_64_64(basis, BH, N, q, k, v, out, S, Zh, state_in, ws, wh, flags,
                                                           stream, nullptr, den_out, d_V, voff)
                                            : tc_run_128_64(basis, BH, N, q, k, v, out, S, Zh, state_in, ws, wh, flags,
                                                            stream, nullptr, den_out, d_V, voff);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
#define SATA_TC_CASE(a, b)                                                                                     \
    if (basis.d_K == a && d_V == b)                                                                            \
        return tc_run_##a##_##b(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io,   \
                                den_out, b, 0);
    SATA_TC_SHAPES(SATA_TC_CASE)
#undef SATA_TC_CASE
    return cudaErrorNotSupported;
}

bool prefill_backward_tc_supported(int d_K, int d_V, int P) { return prefill_tc_supported(d_K, d_V, P); }

size_t prefill_backward_tc_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P) {
#define SATA_TC_CASE(a, b) \
    if (d_K == a && d_V == b) return tc_bwd_workspace_##a##_##b(BH, N, F, P);
    SATA_TC_SHAPES(SATA_TC_CASE)
#undef SATA_TC_CASE
    return 0;
}

cudaError_t launch_prefill_backward_tc(const DeviceBasis &basis, int BH, int64_t N, int d_V, const void *q,
                                       const void *k, const void *v, const float *dy, float *dq, float *dk,
                                       float *dv, void *ws, size_t ws_bytes, int *flags, cudaStream_t stream) {
#define SATA_TC_CASE(a, b)                                                                                     \
    if (basis.d_K == a && d_V == b)                                                                            \
        return tc_bwd_run_##a##_##b(basis, BH, N, q, k, v, dy, dq, dk, dv, ws, ws_bytes, flags, stream);
    SATA_TC_SHAPES(SATA_TC_CASE)
#undef SATA_TC_CASE
    return cudaErrorNotSupported;
}

}  // namespace sata
