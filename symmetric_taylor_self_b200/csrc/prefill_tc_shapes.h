// The (d_K, d_V) instances of the tensor-core prefill and backward, and their entry points.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "sata_internal.h"

// X(d_K, d_V) for every instance; each is defined in one prefill_tc_*.cu file.
#define SATA_TC_SHAPES(X) \
    X(16, 16) X(16, 32) X(16, 64) X(32, 16) X(32, 32) X(32, 64) X(64, 16) X(64, 32) X(64, 64) X(64, 128) \
    X(128, 64) X(128, 128)

namespace sata {
#define SATA_TC_DECLARE(a, b)                                                                                  \
    size_t tc_workspace_##a##_##b(int BH, int64_t N, int64_t F, int P, bool need_state, int min_seg, bool det); \
    cudaError_t tc_run_##a##_##b(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k,    \
                                 const void *v, float *out, float *S, float *Z, bool state_in, void *ws,        \
                                 size_t ws_bytes, int *flags, cudaStream_t stream, const HostIO *io,           \
                                 float *den_out, int dvs, int voff);
SATA_TC_SHAPES(SATA_TC_DECLARE)
#undef SATA_TC_DECLARE
#define SATA_TC_BWD_DECLARE(a, b)                                                                               \
    size_t tc_bwd_workspace_##a##_##b(int BH, int64_t N, int64_t F, int P);                                      \
    cudaError_t tc_bwd_run_##a##_##b(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k, \
                                     const void *v, const float *dy, float *dq, float *dk, float *dv, void *ws, \
                                     size_t ws_bytes, int *flags, cudaStream_t stream);
SATA_TC_SHAPES(SATA_TC_BWD_DECLARE)
#undef SATA_TC_BWD_DECLARE
}  // namespace sata
