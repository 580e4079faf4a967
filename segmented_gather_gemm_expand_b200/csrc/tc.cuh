// Host-visible declarations of the tensor-core (tcgen05 + TMA) variant.
#pragma once

#include "common.cuh"

namespace sgmv {

// True when the tensor-core kernel can run these `nsl` slices of one output
// (dtypes, rank, alignment, sizes) in one launch on a device with `sm_count`
// SMs (the count the launch plans with); otherwise the generic kernel runs
// them, one launch per slice.
bool tc_supports(const Problem* slices, int nsl, int sm_count, int force_bn = 0);

// Enqueue the tensor-core kernel for `nsl` slices.  Returns an SGMV status.
int launch_tc(const Problem* slices, int nsl, int sm_count, cudaStream_t stream, int force_bn = 0);

}  // namespace sgmv
