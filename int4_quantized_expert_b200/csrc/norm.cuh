// RMSNorm in front of the layer: host interface.
#pragma once

#include "common.cuh"

namespace moe {

// out[t, :] = bf16(x[t, :] / sqrt(mean(x[t, :]^2) + eps) * gamma), one CTA per row.
moe_status launch_rmsnorm(const bf16* x, int64_t T, int D, const bf16* gamma, float eps, bf16* out,
                          cudaStream_t stream);

}  // namespace moe
