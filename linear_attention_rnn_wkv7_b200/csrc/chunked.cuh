// chunked.cuh -- 64-token chunked WKV7 forward on tcgen05 tensor cores (bf16).
#pragma once
#include "common.cuh"

namespace wkv7 {

constexpr bool kChunkedBuilt = false;

inline cudaError_t launch_chunked(const void*, const void*, const void*, const void*,
                                  const void*, const void*, const float*, const uint8_t*,
                                  void*, float*, int, int, int, int, const int32_t*,
                                  cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace wkv7
