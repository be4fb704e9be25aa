// Tensor-core prefill instances: d_K = 128, d_V = 64.
#include "prefill_tc_kernels.cuh"

namespace sata {
SATA_TC_DEFINE(128, 64)
}  // namespace sata
