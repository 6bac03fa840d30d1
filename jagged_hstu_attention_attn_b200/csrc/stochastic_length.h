// stochastic_length.h -- launchers of the Stochastic Length selection and the
// row gather (stochastic_length.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hstu {

constexpr int kMaxGatherTensors = 8;

cudaError_t sl_select_launch(const int64_t* offsets, int64_t B, int64_t T,
                             const uint32_t* u_tok, const uint32_t* u_seq, int64_t L,
                             int64_t* dst_offsets, int32_t* src_rows, int* status,
                             cudaStream_t stream);
cudaError_t gather_rows_launch(const void* src, int64_t src_count, void* dst, int64_t row_bytes,
                               const int32_t* src_rows, const int64_t* n_rows, int64_t max_rows,
                               cudaStream_t stream);

cudaError_t gather_rows_multi_launch(int count, const void* const* srcs, void* const* dsts,
                                     const int64_t* row_bytes, int64_t src_count,
                                     const int32_t* src_rows, const int64_t* n_rows,
                                     int64_t max_rows, cudaStream_t stream);

}  // namespace hstu
