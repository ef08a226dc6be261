// chunk_bwd.cu -- placeholder, replaced by the tensor-core kernels.
#include "gla_internal.h"
namespace gla {
size_t bwd_workspace_bytes(int, int, int) { return 0; }
gla_status run_chunk_bwd(const ChunkProblem&, const float*, const void*, const float*, void*,
                         void*, void*, float*, float*, void*, size_t, const WaitCtl&,
                         cudaStream_t) { return GLA_ERR_UNSUPPORTED; }
}  // namespace gla
