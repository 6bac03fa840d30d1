// norm_gate.h -- launchers of the post-attention norm gate (norm_gate.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hstu {

cudaError_t norm_gate_fwd_launch(const void* o, const void* u, void* y, int64_t T, int64_t N,
                                 float eps, cudaStream_t stream);
cudaError_t norm_gate_bwd_launch(const void* o, const void* u, const void* dy, void* d_o,
                                 void* d_u, int64_t T, int64_t N, float eps,
                                 cudaStream_t stream);

}  // namespace hstu
