// tcgen05 tensor-core decode kernel (not built yet).
#include "mla_common.cuh"

namespace mla {
int launch_tc(const Problem &, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
}  // namespace mla
