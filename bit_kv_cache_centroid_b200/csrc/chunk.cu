// chunk.cu — placeholder until the tcgen05 chunk-attention kernel lands.
#include "internal.h"

namespace kv2 {

size_t chunk_workspace_bytes(const kv2_cache& c, int H_q, int Nq) {
  return size_t(c.B) * Nq * H_q * 16 * 2 + 256;
}

cudaError_t launch_chunk(const ChunkArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kv2
