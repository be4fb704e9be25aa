// Tensor-core prefill and backward instances: d_K = 128, d_V = 64.
#include "backward_tc.cuh"

namespace sata {
SATA_TC_DEFINE(128, 64)
SATA_TC_BWD_DEFINE(128, 64)
}  // namespace sata
