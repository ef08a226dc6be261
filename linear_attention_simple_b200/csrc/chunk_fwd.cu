// chunk_fwd.cu -- placeholder, replaced by the tensor-core kernel.
#include "gla_internal.h"
namespace gla {
size_t fwd_workspace_bytes(int, int, int) { return 0; }
gla_status run_chunk_fwd(const ChunkProblem&, const float*, void*, float*, void*, size_t,
                         const WaitCtl&, cudaStream_t) { return GLA_ERR_UNSUPPORTED; }
}  // namespace gla
