// Tensor-core prefill and backward instances: d_K = 16, d_V = 16, d_K = 16, d_V = 32, d_K = 16, d_V = 64.
#include "backward_tc.cuh"

namespace sata {
SATA_TC_DEFINE(16, 16)
SATA_TC_BWD_DEFINE(16, 16)
SATA_TC_DEFINE(16, 32)
SATA_TC_BWD_DEFINE(16, 32)
SATA_TC_DEFINE(16, 64)
SATA_TC_BWD_DEFINE(16, 64)
}  // namespace sata
