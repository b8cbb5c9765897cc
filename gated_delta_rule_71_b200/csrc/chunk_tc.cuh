// chunk_tc.cuh -- tcgen05 tensor-core chunked forward (bf16 operands, fp32 state).
#pragma once

#include "chunk_simt.cuh"

namespace gdn {

constexpr bool kTcAvailable = false;

inline int launch_chunk_tc(const ChunkArgs&, bool, cudaStream_t) { return 1; }

}  // namespace gdn
