// Shapes and arguments shared by the decode kernels (CUDA-core and tensor-core).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tq {

struct DecodeShape {
  int d, kbits, vbits;
  int batch, hq, hkv, nq;
  int64_t n_ctx, ctx_stride;
  int rows_per_cta;   // R
  int row_blocks;     // (hq/hkv*nq) / R
  int n_splits;
  int n_parts;        // partial records per query row: n_splits, or 2 n_splits (tensor-core path)
  int64_t chunk;      // tokens per split (multiple of kT)
  int64_t n_rows;     // batch*hq*nq
};

struct DecodeArgs {
  DecodeShape sh;
  const void* q;
  int q_dtype;
  const int32_t* q_pos;
  double rope_base;
  const uint8_t* kidx;
  const uint32_t* ksign;
  const float* knorm;
  const float* krnorm;
  const uint8_t* vidx;
  const float* vnorm;
  const float* PiK;
  const float* PiV;
  int64_t pi_stride;
  const float* S;
  const float* cK;
  const float* cV;
  float scale;
  void* out;
  int out_dtype;
  float* scores_out;
  float* qs;     // [n_rows][2][d]  q_rot then s
  float* part;   // [n_rows][n_parts][d + 2]  acc..., m, l
  int32_t* d_status;
};

// Tensor-core decode (tq_decode_tc.cu): d = 128, four query rows per KV
// stream, 3-bit values, 2-4 bit keys.
bool tc_decode_supported(const DecodeArgs& a);
cudaError_t tc_decode_launch(const DecodeArgs& a, cudaStream_t st);

}  // namespace tq
