// sata_decode_step's kernels: the shared decode-step kernels (decode_kernels.cuh)
// with the feature basis read from the library's cached tables, which serve
// every supported P.
#include "decode_kernels.cuh"

namespace sata {

size_t decode_workspace_bytes(int BH, int64_t F, int d_V) {
    return (size_t)BH * (size_t)dec::num_groups(F) * (size_t)(d_V + 1) * sizeof(float);
}

cudaError_t launch_decode(const DeviceBasis &basis, int BH, int d_V, float *S, float *Z,
                          const void *q, const void *k, const void *v, float *out,
                          float *partials, cudaStream_t stream) {
    const dec::TableBasis tb{basis.packed, basis.packed_hi, basis.coef};
    return dec::launch_any(d_V, tb, BH, basis.d_K, basis.F, S, Z, q, k, v, out, partials, stream, true);
}

}  // namespace sata
