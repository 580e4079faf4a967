// Host-visible declarations of the tensor-core (tcgen05 + TMA) variant.
#pragma once

#include "common.cuh"

namespace sgmv {

// True when the tensor-core kernel can run this call (dtypes, rank,
// alignment, sizes); otherwise the generic kernel runs it.
bool tc_supports(const Problem& p);

// Enqueue the tensor-core kernel.  Returns an SGMV status.
int launch_tc(const Problem& p, int sm_count, cudaStream_t stream);

}  // namespace sgmv
