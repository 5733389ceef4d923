// Tensor-core (tcgen05) path: not built yet; every problem takes the generic path.
#include "internal.h"

namespace kda {
size_t kda_tc_workspace_bytes(int, int, int, int, int) { return 0; }
bool kda_tc_supported(const KdaArgs&) { return false; }
cudaError_t launch_kda_tc(const KdaArgs&, void*, size_t, int*, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace kda
