// Tensor-core variant (placeholder until the kernel lands).
#pragma once

namespace sgmv {

bool tc_supports(const Problem&) { return false; }

int launch_tc(const Problem&, int, cudaStream_t) { return SGMV_ERR_VARIANT; }

}  // namespace sgmv
