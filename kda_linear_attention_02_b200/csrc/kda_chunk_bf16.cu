// kda_chunk_bf16.cu -- chunked KDA forward for bf16 inputs on tcgen05 (placeholder during bring-up).
#include "kda_chunk_common.cuh"
#include "kda_internal.h"

namespace kda {

size_t chunk_packet_bytes_bf16(int dk, int dv) { return 82944; }

cudaError_t launch_chunk_bf16(const ChunkArgs& a, cudaStream_t s) { return cudaErrorNotSupported; }

}  // namespace kda
