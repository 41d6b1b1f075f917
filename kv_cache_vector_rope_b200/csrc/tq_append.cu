// tq_append_kv: quantise one new vector per stream straight into its cache
// slot (the incremental decode step).
//
// Sources: 7minutos.es "KV cache ... TurboQuant" Etapa 1 (a token's indices
// are computed once, when it enters the cache) and Etapa 2 (keys: signs of
// S times the residual, and the residual norm); gist.science "TurboESM ..."
// section 2A (RoPE at the token's position, then the rotation).
//
// One CTA per stream, thread i = coordinate i, all arithmetic in fp64: a
// decode step appends only batch x kv-heads vectors, too few to fill the
// tensor-core quantiser's 128-vector tiles, and exact arithmetic needs no
// guard band or second pass. Pi (then S) is staged in shared memory with a
// padded row stride so that thread i reading row i is free of bank conflicts.
#include <cuda_runtime.h>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace dev;

struct AppendArgs {
  const void* x;
  int dtype;
  int64_t row_stride;
  const int32_t* pos;
  double rope_base;
  const float* Pi;
  const float* S;
  const float* cent;
  const float* bnd;
  int bits;
  int is_key;
  uint8_t* idx;
  uint32_t* sign;
  float* norm;
  float* rnorm;
  int64_t ctx_stride;
  int64_t slot;
  int32_t* d_status;
};

constexpr int threads_for(int d) { return (d + 31) / 32 * 32; }

template <int D>
struct AppendSmem {
  static constexpr int kLd = D + 1;                  // padded row stride (floats)
  static constexpr size_t kOffX = 0;                 // double x[D] (RoPE'd input)
  static constexpr size_t kOffR = kOffX + sizeof(double) * D;   // double r[D] (residual)
  static constexpr size_t kOffRed = kOffR + sizeof(double) * D; // double [8] partial sums
  static constexpr size_t kOffCode = kOffRed + sizeof(double) * 8;
  static constexpr size_t kOffM = (kOffCode + sizeof(int) * D + 15) / 16 * 16;
  static constexpr size_t kBytes = kOffM + sizeof(float) * size_t(D) * kLd;
};

// Sum over the CTA's threads (fp64); every thread gets the total.
template <int T>
__device__ __forceinline__ double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int k = 0; k < T / 32; ++k) t += red[k];
  return t;
}

// M (row-major D x D, 16-byte aligned) into shared memory at the padded
// stride, float4 loads issued eight at a time so that the L2 latency is paid
// once per eight loads rather than once per load.
template <int D>
__device__ __forceinline__ void stage_matrix(float* M, const float* __restrict__ src) {
  constexpr int T = threads_for(D);
  constexpr int kV = D * D / 4;                      // float4 in the matrix
  const float4* s4 = reinterpret_cast<const float4*>(src);
  for (int base = 0; base < kV; base += 8 * T) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = base + u * T + threadIdx.x;
      if (e < kV) v[u] = __ldg(s4 + e);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = base + u * T + threadIdx.x;
      if (e < kV) {
        float* dst = M + ((4 * e) / D) * AppendSmem<D>::kLd + (4 * e) % D;   // D % 4 == 0: a row holds whole float4s
        dst[0] = v[u].x;
        dst[1] = v[u].y;
        dst[2] = v[u].z;
        dst[3] = v[u].w;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(threads_for(D)) append_kernel(AppendArgs a) {
  constexpr int T = threads_for(D);
  using L = AppendSmem<D>;
  extern __shared__ __align__(16) unsigned char smem[];
  double* x = reinterpret_cast<double*>(smem + L::kOffX);
  double* r = reinterpret_cast<double*>(smem + L::kOffR);
  double* red = reinterpret_cast<double*>(smem + L::kOffRed);
  int* code = reinterpret_cast<int*>(smem + L::kOffCode);
  float* M = reinterpret_cast<float*>(smem + L::kOffM);
  const int i = threadIdx.x;
  const bool on = i < D;
  const int64_t s = blockIdx.x;
  const int64_t row = s * a.ctx_stride + a.slot;
  const int nb = (1 << a.bits) - 1;
  if (s == 0 && i == 0 && a.d_status) {
    for (int j = 1; j < nb; ++j)
      if (!(a.bnd[j] > a.bnd[j - 1])) atomicOr(a.d_status, TQ_DEV_BAD_CODEBOOK);
  }
  // x' = RoPE(x): pairs (i, i + D/2) turned by pos * base^(-2i/D).
  const bool rope = a.pos != nullptr && a.rope_base > 0.0;
  if (i < D / 2) {
    const int64_t base = s * a.row_stride;
    double x0 = load_elem(a.x, a.dtype, base + i), x1 = load_elem(a.x, a.dtype, base + i + D / 2);
    if (rope) {
      const int p = a.pos[s];
      if (p < 0 && a.d_status) atomicOr(a.d_status, TQ_DEV_BAD_POSITION);
      double sn, cs;
      sincos(rope_angle(p, i, D, a.rope_base), &sn, &cs);
      const double r0 = x0 * cs - x1 * sn, r1 = x0 * sn + x1 * cs;
      x0 = r0;
      x1 = r1;
    }
    x[i] = x0;
    x[i + D / 2] = x1;
  }
  stage_matrix<D>(M, a.Pi);
  __syncthreads();
  const double nrm = sqrt(block_sum<T>(on ? x[i] * x[i] : 0.0, red));
  // y_i = (Pi x')_i; code_i = #{j : y_i > ||x'|| t_j} (a zero vector has u = 0).
  double y = 0.0;
  if (on) {
    const float* mrow = M + i * L::kLd;
#pragma unroll 8
    for (int j = 0; j < D; ++j) y = fma(static_cast<double>(mrow[j]), x[j], y);
  }
  int c = 0;
  for (int j = 0; j < nb; ++j) {
    const double t = static_cast<double>(__ldg(a.bnd + j));
    c += (nrm > 0.0 ? (y > nrm * t) : (0.0 > t)) ? 1 : 0;
  }
  const double res = y - nrm * static_cast<double>(__ldg(a.cent + c));
  if (on) {
    code[i] = c;
    r[i] = res;
  }
  __syncthreads();
  // Pack: thread g writes the `bits` bytes of coordinates 8g .. 8g + 7.
  if (i < D / 8) {
    uint32_t word = 0;
    for (int k = 0; k < 8; ++k) word |= static_cast<uint32_t>(code[8 * i + k]) << (a.bits * k);
    uint8_t* dst = a.idx + row * (static_cast<int64_t>(D) * a.bits / 8) + i * a.bits;
    for (int b = 0; b < a.bits; ++b) dst[b] = static_cast<uint8_t>(word >> (8 * b));
  }
  if (i == 0) a.norm[row] = static_cast<float>(nrm);
  if (!a.is_key) return;
  const double rn = sqrt(block_sum<T>(on ? res * res : 0.0, red));
  __syncthreads();                                   // every thread is done with Pi
  stage_matrix<D>(M, a.S);
  __syncthreads();
  // sign_i = ((S r)_i >= 0), 32 per word (thread i -> bit i % 32 of word i / 32).
  double p = 0.0;
  if (on) {
    const float* mrow = M + i * L::kLd;
#pragma unroll 8
    for (int j = 0; j < D; ++j) p = fma(static_cast<double>(mrow[j]), r[j], p);
  }
  const uint32_t word = __ballot_sync(0xffffffffu, on && p >= 0.0);
  constexpr int kW = (D + 31) / 32;
  if ((i & 31) == 0 && (i >> 5) < kW) a.sign[row * kW + (i >> 5)] = word;
  if (i == 0) a.rnorm[row] = static_cast<float>(rn);
}

template <int D>
cudaError_t launch_append(const AppendArgs& a, int64_t n, cudaStream_t st) {
  constexpr size_t smem = AppendSmem<D>::kBytes;
  static_assert(smem <= 232448, "append shared memory plan exceeds 227 KB");
  cudaError_t e = cudaFuncSetAttribute(append_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  append_kernel<D><<<static_cast<unsigned>(n), threads_for(D), smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

// Small quantise calls (tq_quantize_kv with a shared Pi and few vectors) run
// on the same exact kernel: vector v to plane row v.
cudaError_t append_quantize(int d, int bits, bool is_key, const void* x, int dtype, int64_t n, int64_t row_stride,
                            const int32_t* pos, float rope_base, const float* Pi, const float* S, const float* cent,
                            const float* bnd, const tq_planes* out, int32_t* d_status, cudaStream_t st) {
  AppendArgs a{x, dtype, row_stride, pos, static_cast<double>(rope_base), Pi, S, cent, bnd, bits, is_key ? 1 : 0,
               out->idx, is_key ? out->sign : nullptr, out->norm, is_key ? out->rnorm : nullptr, 1, 0, d_status};
  switch (d) {
    case 64: return launch_append<64>(a, n, st);
    case 128: return launch_append<128>(a, n, st);
    default: return launch_append<200>(a, n, st);
  }
}

}  // namespace tq

extern "C" tq_status tq_append_kv(const tq_layout* layout, int32_t is_key, const void* x, tq_dtype x_dtype,
                                  int64_t n_streams, int64_t row_stride, const int32_t* positions, float rope_base,
                                  const float* Pi, const float* S, const float* centroids, const float* boundaries,
                                  const tq_planes* cache, int64_t ctx_stride, int64_t slot, int32_t* d_status,
                                  void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_layout(layout);
  if (st != TQ_OK) return st;
  const int d = layout->d;
  const int bits = is_key ? layout->key_bits : layout->value_bits;
  if (n_streams < 0) return fail(TQ_ERR_INVALID_ARG, "n_streams < 0");
  if (n_streams == 0) return TQ_OK;
  if (n_streams > 0x7FFFFFFF) return fail(TQ_ERR_INVALID_ARG, "n_streams too large");
  if (!x || !Pi || !centroids || !boundaries || !cache || !cache->idx || !cache->norm)
    return fail(TQ_ERR_INVALID_ARG, "NULL input/output pointer");
  if (is_key && (!S || !cache->sign || !cache->rnorm)) return fail(TQ_ERR_INVALID_ARG, "keys need S, sign and rnorm");
  if (x_dtype != TQ_F32 && x_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_F32 or TQ_BF16");
  if (row_stride < d) return fail(TQ_ERR_INVALID_ARG, "row_stride (%lld) < d (%d)", (long long)row_stride, d);
  if (ctx_stride < 1 || slot < 0 || slot >= ctx_stride)
    return fail(TQ_ERR_INVALID_ARG, "slot (%lld) outside [0, ctx_stride = %lld)", (long long)slot,
                (long long)ctx_stride);
  if (!aligned(Pi, 16) || (S && !aligned(S, 16))) return fail(TQ_ERR_INVALID_ARG, "Pi/S must be 16-byte aligned");
  AppendArgs a{x, x_dtype == TQ_F32 ? 0 : 1, row_stride, positions, static_cast<double>(rope_base), Pi, S,
               centroids, boundaries, bits, is_key ? 1 : 0, cache->idx, is_key ? cache->sign : nullptr,
               cache->norm, is_key ? cache->rnorm : nullptr, ctx_stride, slot, d_status};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (d) {
    case 64: e = launch_append<64>(a, n_streams, s); break;
    case 128: e = launch_append<128>(a, n_streams, s); break;
    case 200: e = launch_append<200>(a, n_streams, s); break;
    default: return fail(TQ_ERR_UNSUPPORTED, "tq_append_kv: d=%d not built (64, 128, 200)", d);
  }
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_append_kv launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}
