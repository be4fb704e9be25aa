// Tensor-core prefill instances: d_K = 128, d_V = 128.
#include "prefill_tc_kernels.cuh"

namespace sata {
SATA_TC_DEFINE(128, 128)
}  // namespace sata
