// bwd_sm100.cu -- backward attention (under construction: row statistic D only).
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fa {

cudaError_t launch_bwd_sm100(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                             const CUtensorMap&, const void*, const void*, const float*, void*,
                             void*, void*, float*, const Problem&, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace fa
