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
  int n_parts;        // partial records per query row (CUDA-core path): n_splits
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
  float* qs;     // CUDA-core path: [n_rows][2][d]  q_rot then s
  float* part;   // partial records (layout per path)
  int32_t* d_status;
};

// Fused tensor-core decode (tq_decode_tc.cu): d = 128, a GQA group of four
// query heads with one query each, 3-bit values, 2-4 bit keys; one launch
// (after a memset of its arrival counters) computes the whole call.
bool tc_decode_supported(const DecodeArgs& a);
// Workspace bytes of the fused path for this shape (0 if the shape is not one
// it runs).
size_t tc_decode_workspace_bytes(const DecodeShape& s);
cudaError_t tc_decode_launch(const DecodeArgs& a, void* workspace, cudaStream_t st);

}  // namespace tq
