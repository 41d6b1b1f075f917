// tq_dequantize: rebuild vectors from their packed planes.
//
// Source: 7minutos.es "KV cache ... TurboQuant". Etapa 1: look each index up
// in the codebook and multiply by the transpose of the rotation. Etapa 2: the
// sign bits times S^T, scaled by sqrt(pi/2)/d and the residual norm, are added
// (K_tilde = K_hat + K_tilde_QJL). S acts on the rotated residual here, so the
// correction is added before the single Pi^T.
//
// gist.science "TurboESM ..." section 2D (tq_dequantize_sign_mean): the sign
// of each rotated residual coordinate and a calibrated mean magnitude e_bar
// give the first-order correction x_tilde = x_hat + ||x|| e_bar (2 sign - 1).
//
// One CTA of d threads per vector: thread i forms rotated coordinate i, then
// thread j forms output coordinate j = sum_i Pi[i][j] rot[i].
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace dev;

struct DequantArgs {
  int d, bits, is_key;
  int64_t n;
  const uint8_t* idx;
  const uint32_t* sign;
  const float* norm;
  const float* rnorm;
  const float* Pi;
  int64_t vectors_per_pi, pi_stride;
  const float* S;
  const float* cent;
  void* out;
  int out_dtype;
  int64_t out_stride;
  int sign_mean;        // 1: TurboESM correction with e_bar (no S, no rnorm)
  float e_bar;
};

__global__ void dequant_kernel(DequantArgs a) {
  extern __shared__ float dq[];
  const int d = a.d;
  float* pm = dq;        // [d] +-1 signs
  float* rot = dq + d;   // [d] rotated reconstruction
  const int64_t v = blockIdx.x;
  const int rb = d * a.bits / 8;
  const int sw = (d + 31) / 32;
  const uint8_t* row = a.idx + v * rb;
  const float nrm = a.norm[v];
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    if (a.sign_mean) {
      const float s = ((a.sign[v * sw + (i >> 5)] >> (i & 31)) & 1u) ? a.e_bar : -a.e_bar;
      rot[i] = nrm * (__ldg(a.cent + get_code(row, i, a.bits)) + s);
    } else {
      rot[i] = nrm * __ldg(a.cent + get_code(row, i, a.bits));
      if (a.is_key) pm[i] = ((a.sign[v * sw + (i >> 5)] >> (i & 31)) & 1u) ? 1.f : -1.f;
    }
  }
  __syncthreads();
  if (a.is_key && !a.sign_mean) {
    const float scale = static_cast<float>(kSqrtHalfPi / d) * a.rnorm[v];
    float corr[2] = {0.f, 0.f};
    for (int c = 0; c < 2; ++c) {
      const int j = threadIdx.x + c * blockDim.x;
      if (j < d) {
        float acc = 0.f;
        for (int i = 0; i < d; ++i) acc = fmaf(__ldg(a.S + int64_t(i) * d + j), pm[i], acc);
        corr[c] = scale * acc;
      }
    }
    __syncthreads();
    for (int c = 0; c < 2; ++c) {
      const int j = threadIdx.x + c * blockDim.x;
      if (j < d) rot[j] += corr[c];
    }
    __syncthreads();
  }
  const float* Pi = a.Pi + (a.pi_stride ? (v / a.vectors_per_pi) * a.pi_stride : 0);
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < d; ++i) acc = fmaf(__ldg(Pi + int64_t(i) * d + j), rot[i], acc);
    if (a.out_dtype == 0)
      reinterpret_cast<float*>(a.out)[v * a.out_stride + j] = acc;
    else
      reinterpret_cast<__nv_bfloat16*>(a.out)[v * a.out_stride + j] = __float2bfloat16(acc);
  }
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_dequantize(const tq_layout* layout, int32_t is_key, int64_t n_vectors, const tq_planes* planes,
                                   const float* Pi, int64_t vectors_per_pi, int64_t pi_stride, const float* S,
                                   const float* centroids, void* out, tq_dtype out_dtype, int64_t out_stride,
                                   void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_layout(layout);
  if (st != TQ_OK) return st;
  const int d = layout->d;
  if (n_vectors < 0) return fail(TQ_ERR_INVALID_ARG, "n_vectors < 0");
  if (n_vectors == 0) return TQ_OK;
  if (n_vectors > 0x7fffffffLL) return fail(TQ_ERR_UNSUPPORTED, "n_vectors above 2^31-1 per call");
  if (!planes || !planes->idx || !planes->norm || !Pi || !centroids || !out)
    return fail(TQ_ERR_INVALID_ARG, "NULL pointer argument");
  if (is_key && (!planes->sign || !planes->rnorm || !S)) return fail(TQ_ERR_INVALID_ARG, "keys need sign, rnorm and S");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "out_dtype must be TQ_F32 or TQ_BF16");
  if (out_stride < d) return fail(TQ_ERR_INVALID_ARG, "out_stride < d");
  if (pi_stride < 0 || (pi_stride > 0 && vectors_per_pi < 1))
    return fail(TQ_ERR_INVALID_ARG, "pi_stride < 0 or vectors_per_pi < 1");
  DequantArgs a{d, is_key ? layout->key_bits : layout->value_bits, is_key ? 1 : 0, n_vectors, planes->idx,
                planes->sign, planes->norm, planes->rnorm, Pi, vectors_per_pi, pi_stride, S, centroids, out,
                out_dtype == TQ_F32 ? 0 : 1, out_stride, 0, 0.f};
  dequant_kernel<<<static_cast<unsigned>(n_vectors), 128, 2 * d * sizeof(float), static_cast<cudaStream_t>(stream)>>>(a);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_dequantize launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

extern "C" tq_status tq_dequantize_sign_mean(const tq_layout* layout, int32_t is_key, int64_t n_vectors,
                                             const tq_planes* planes, const float* Pi, int64_t vectors_per_pi,
                                             int64_t pi_stride, const float* centroids, float e_bar, void* out,
                                             tq_dtype out_dtype, int64_t out_stride, void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_layout(layout);
  if (st != TQ_OK) return st;
  const int d = layout->d;
  if (n_vectors < 0) return fail(TQ_ERR_INVALID_ARG, "n_vectors < 0");
  if (n_vectors == 0) return TQ_OK;
  if (n_vectors > 0x7fffffffLL) return fail(TQ_ERR_UNSUPPORTED, "n_vectors above 2^31-1 per call");
  if (!planes || !planes->idx || !planes->sign || !planes->norm || !Pi || !centroids || !out)
    return fail(TQ_ERR_INVALID_ARG, "NULL pointer argument (idx, sign and norm planes are required)");
  if (!(e_bar >= 0.f)) return fail(TQ_ERR_INVALID_ARG, "e_bar must be >= 0");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "out_dtype must be TQ_F32 or TQ_BF16");
  if (out_stride < d) return fail(TQ_ERR_INVALID_ARG, "out_stride < d");
  if (pi_stride < 0 || (pi_stride > 0 && vectors_per_pi < 1))
    return fail(TQ_ERR_INVALID_ARG, "pi_stride < 0 or vectors_per_pi < 1");
  DequantArgs a{d, is_key ? layout->key_bits : layout->value_bits, is_key ? 1 : 0, n_vectors, planes->idx,
                planes->sign, planes->norm, nullptr, Pi, vectors_per_pi, pi_stride, nullptr, centroids, out,
                out_dtype == TQ_F32 ? 0 : 1, out_stride, 1, e_bar};
  dequant_kernel<<<static_cast<unsigned>(n_vectors), 128, 2 * d * sizeof(float), static_cast<cudaStream_t>(stream)>>>(a);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_dequantize_sign_mean launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}
