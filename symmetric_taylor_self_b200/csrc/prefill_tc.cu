// Tensor-core (tcgen05) prefill: not yet built; the dispatcher never selects it.
#include "sata_internal.h"

namespace sata {

bool prefill_tc_supported(int, int, int) { return false; }

size_t prefill_tc_workspace_bytes(int, int64_t, int64_t, int, int, bool) { return 0; }

cudaError_t launch_prefill_tc(const DeviceBasis &, int, int64_t, int, const void *, const void *,
                              const void *, float *, float *, float *, bool, void *, size_t, int *,
                              cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace sata
