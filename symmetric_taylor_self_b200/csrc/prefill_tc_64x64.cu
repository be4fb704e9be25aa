// Tensor-core prefill instances: d_K = 64, d_V = 64.
#include "prefill_tc_kernels.cuh"

namespace sata {
SATA_TC_DEFINE(64, 64)
}  // namespace sata
