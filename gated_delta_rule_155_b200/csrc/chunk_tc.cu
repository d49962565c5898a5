// chunk_tc.cu — tcgen05 chunked prefill (bf16 I/O, dk = dv = 128).  Not built yet.
#include "internal.h"

namespace kda {
bool chunk_tc_supported(const ChunkArgs &) { return false; }
cudaError_t launch_chunk_tc(const ChunkArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace kda
