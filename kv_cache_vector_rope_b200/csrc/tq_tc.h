// Internal interface of the tensor-core quantiser (tq_quantize_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tq {

// True when the tensor-core path applies: d 64 or 128, bf16 input rows with
// 16-byte aligned base and stride, no RoPE; one shared Pi, or (d = 64) one Pi
// per vectors_per_pi rows with vectors_per_pi a multiple of 128.
bool tc_quantize_supported(int d, int x_dtype, bool rope, int64_t vectors_per_pi, int64_t pi_stride, const void* x,
                           int64_t row_stride);

tq_status tc_quantize(int d, bool is_key, int bits, const void* x, int64_t n, int64_t row_stride, const float* Pi,
                      int64_t vectors_per_pi, int64_t pi_stride, const float* S, const float* cent, const float* bnd,
                      const tq_planes* out, int32_t* d_status, cudaStream_t st);

// Exact fp64 quantisation, one CTA per vector (tq_append.cu): vector v to
// plane row v. For calls with few vectors and one shared Pi.
cudaError_t append_quantize(int d, int bits, bool is_key, const void* x, int dtype, int64_t n, int64_t row_stride,
                            const int32_t* pos, float rope_base, const float* Pi, const float* S, const float* cent,
                            const float* bnd, const tq_planes* out, int32_t* d_status, cudaStream_t st);

}  // namespace tq
