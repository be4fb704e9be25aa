// Tensor-core prefill and backward instances: d_K = 64, d_V = 16, d_K = 64, d_V = 32.
#include "backward_tc.cuh"

namespace sata {
SATA_TC_DEFINE(64, 16)
SATA_TC_BWD_DEFINE(64, 16)
SATA_TC_DEFINE(64, 32)
SATA_TC_BWD_DEFINE(64, 32)
}  // namespace sata
