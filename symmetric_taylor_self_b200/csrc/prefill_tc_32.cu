// Tensor-core prefill and backward instances: d_K = 32, d_V = 16, d_K = 32, d_V = 32, d_K = 32, d_V = 64.
#include "backward_tc.cuh"

namespace sata {
SATA_TC_DEFINE(32, 16)
SATA_TC_BWD_DEFINE(32, 16)
SATA_TC_DEFINE(32, 32)
SATA_TC_BWD_DEFINE(32, 32)
SATA_TC_DEFINE(32, 64)
SATA_TC_BWD_DEFINE(32, 64)
}  // namespace sata
