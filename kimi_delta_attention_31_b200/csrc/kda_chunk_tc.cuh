// kda_chunk_tc.cuh -- tensor-core (tcgen05) chunkwise prefill: not built yet.
#pragma once
#include "kda_common.cuh"

namespace kda {

constexpr bool kTcPathBuilt = false;
constexpr int kTcLaunches = 2;

inline size_t tc_workspace_bytes(long long /*max_chunks*/, int /*H*/, int /*N*/) { return 0; }

inline cudaError_t launch_chunk_tc(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                   const float*, const float*, const float*, __nv_bfloat16*, float*,
                                   const int32_t*, int, int, int, int, long long, void*,
                                   cudaEvent_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kda
