// Tensor-core prefill and backward: shape dispatch to the instances of the prefill_tc_*.cuh
// and backward_tc.cuh templates
// (one prefill_tc_*.cu file per group of shapes, compiled in parallel).
#include "prefill_tc_shapes.h"
#include "sata_internal.h"

namespace sata {

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
#define SATA_TC_CASE(a, b)                                                                                     \
    if (basis.d_K == a && d_V == b)                                                                            \
        return tc_run_##a##_##b(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io,   \
                                den_out);
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
