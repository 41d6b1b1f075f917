// tq_quantize_kv: RoPE -> Pi -> norm + Lloyd-Max codes -> (keys) QJL signs.
//
// Sources: gist.science "TurboESM ..." section 2A (RoPE first, then Pi) and
// 7minutos.es "KV cache ... TurboQuant" Etapa 1 (rotation, Lloyd-Max index per
// coordinate) and Etapa 2 (sign of S times the residual, residual norm).
//
// Exactness. A code or sign is an integer decided by floating point. This
// kernel decides it in fp32 only when the fp32 margin to the decision
// (|y_i - ||x|| t_j| for codes, |(S r)_i| for signs) is wider than a guard band
// that bounds the fp32 error with a wide safety factor; any vector with a
// decision inside its band is recomputed end to end in fp64 by one warp, so
// the stored codes and signs are those of exact arithmetic.
//
// Work split: a CTA takes tiles of kTV consecutive vectors. The rotation and
// the projection are register-tiled fp32 GEMMs over shared-memory tiles
// (4 vectors x 4 outputs per thread); per-vector bucketize, residual and
// sign packing run one warp per vector.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_tc.h"

namespace tq {
namespace {

using namespace dev;

constexpr int kThreads = 256;
constexpr int kTV = 64;        // vectors per tile
constexpr int64_t kExactMaxVectors = 1024;   // up to this many: the exact per-vector kernel
constexpr int kJC = 32;        // reduction chunk of the GEMMs
// Guard bands (relative to ||x|| for codes and to ||r|| for signs). The fp32
// error of a d<=256 dot product here is below 3e-7 of those scales.
constexpr float kCodeGuard = 1e-5f;
constexpr float kSignGuard = 1e-4f;

struct QuantArgs {
  const void* x;
  int dtype;
  int64_t n;
  int64_t row_stride;
  const int32_t* pos;
  double rope_base;
  const float* Pi;
  int64_t vectors_per_pi;
  int64_t pi_stride;
  const float* S;
  const float* cent;
  const float* bnd;
  int bits;
  int is_key;
  uint8_t* idx;
  uint32_t* sign;
  float* norm;
  float* rnorm;
  int32_t* d_status;
};

template <int D>
struct Smem {
  static constexpr int kLd = D + 4;                  // row stride (floats), 16-B aligned
  float xs[kTV][kLd];                                // RoPE'd input, later S r
  float ys[kTV][kLd];                                // Pi x', later the residual r
  float ws[kJC][kLd];                                // chunk of M^T
  uint8_t codes[kTV][D];
  uint32_t signs[kTV][(D + 31) / 32];
  float nrm[kTV];
  float rn[kTV];
  int flag[kTV];
  float cent[16];
  float bnd[16];
  double scratch[kThreads / kWarp][2][D];            // per-warp fp64 fixup rows
};

// Y[v][i] = sum_j M[i][j] X[v][j] for the tile rows whose Pi group equals `g`
// (M row-major D x D). Each thread owns up to kItems 4x4 output blocks.
template <int D>
__device__ void tile_gemm(Smem<D>& s, float (*X)[Smem<D>::kLd], float (*Y)[Smem<D>::kLd], const float* __restrict__ M,
                          const int* row_ok) {
  constexpr int kIG = D / 4;
  constexpr int kBlocks = (kTV / 4) * kIG;
  constexpr int kItems = (kBlocks + kThreads - 1) / kThreads;
  float acc[kItems][4][4];
#pragma unroll
  for (int it = 0; it < kItems; ++it)
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[it][a][b] = 0.f;

  for (int j0 = 0; j0 < D; j0 += kJC) {
    const int jc = min(kJC, D - j0);
    __syncthreads();
    // Coalesced along j (rows of M), transposed into ws[jj][i].
    for (int e = threadIdx.x; e < jc * D; e += kThreads) {
      const int i = e / jc, jj = e % jc;
      s.ws[jj][i] = __ldg(M + static_cast<int64_t>(i) * D + j0 + jj);
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int blk = threadIdx.x + it * kThreads;
      if (blk < kBlocks) {
        const int v = (blk / kIG) * 4, i = (blk % kIG) * 4;
        for (int jj = 0; jj < jc; ++jj) {
          const float4 w = *reinterpret_cast<const float4*>(&s.ws[jj][i]);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const float xv = X[v + a][j0 + jj];
            acc[it][a][0] = fmaf(w.x, xv, acc[it][a][0]);
            acc[it][a][1] = fmaf(w.y, xv, acc[it][a][1]);
            acc[it][a][2] = fmaf(w.z, xv, acc[it][a][2]);
            acc[it][a][3] = fmaf(w.w, xv, acc[it][a][3]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int blk = threadIdx.x + it * kThreads;
    if (blk < kBlocks) {
      const int v = (blk / kIG) * 4, i = (blk % kIG) * 4;
#pragma unroll
      for (int a = 0; a < 4; ++a)
        if (row_ok[v + a]) *reinterpret_cast<float4*>(&Y[v + a][i]) = make_float4(acc[it][a][0], acc[it][a][1], acc[it][a][2], acc[it][a][3]);
    }
  }
}

// fp64 recomputation of one vector by one warp; writes its planes.
template <int D>
__device__ void exact_vector(const QuantArgs& a, Smem<D>& s, int64_t v, const float* __restrict__ Pi) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  double* xd = s.scratch[w][0];
  double* yd = s.scratch[w][1];
  const int nb = (1 << a.bits) - 1;
  const bool rope = a.pos != nullptr && a.rope_base > 0.0;
  const int pos = rope ? a.pos[v] : 0;
  const int64_t base = v * a.row_stride;
  for (int i = lane; i < D / 2; i += kWarp) {
    double x0 = load_elem(a.x, a.dtype, base + i), x1 = load_elem(a.x, a.dtype, base + i + D / 2);
    if (rope) {
      double sn, cs;
      sincos(rope_angle(pos, i, D, a.rope_base), &sn, &cs);
      const double r0 = x0 * cs - x1 * sn, r1 = x0 * sn + x1 * cs;
      x0 = r0;
      x1 = r1;
    }
    xd[i] = x0;
    xd[i + D / 2] = x1;
  }
  __syncwarp();
  double ss = 0.0;
  for (int j = lane; j < D; j += kWarp) ss += xd[j] * xd[j];
  const double nrm = sqrt(warp_sum(ss));
  for (int i = lane; i < D; i += kWarp) {
    double acc = 0.0;
    const float* row = Pi + static_cast<int64_t>(i) * D;
    for (int j = 0; j < D; ++j) acc = fma(static_cast<double>(__ldg(row + j)), xd[j], acc);
    yd[i] = acc;
  }
  __syncwarp();
  // Codes and the residual (kept in yd).
  double rs = 0.0;
  for (int i = lane; i < D; i += kWarp) {
    const double y = yd[i];
    // code = #{j : y/||x|| > t_j}; a zero vector has u = 0.
    int c = 0;
    for (int j = 0; j < nb; ++j) {
      const double t = static_cast<double>(s.bnd[j]);
      c += (nrm > 0.0 ? (y > nrm * t) : (0.0 > t)) ? 1 : 0;
    }
    const double r = y - nrm * static_cast<double>(s.cent[c]);
    yd[i] = r;
    xd[i] = static_cast<double>(c);  // park the code; x is no longer needed
    rs += r * r;
  }
  __syncwarp();
  const double rnrm = sqrt(warp_sum(rs));
  // Pack codes: lane g handles group g (8 codes -> bits bytes).
  uint8_t* irow = a.idx + v * (static_cast<int64_t>(D) * a.bits / 8);
  for (int g = lane; g < D / 8; g += kWarp) {
    uint32_t word = 0;
    for (int j = 0; j < 8; ++j) word |= static_cast<uint32_t>(xd[8 * g + j]) << (a.bits * j);
    for (int b = 0; b < a.bits; ++b) irow[g * a.bits + b] = static_cast<uint8_t>(word >> (8 * b));
  }
  if (lane == 0) a.norm[v] = static_cast<float>(nrm);
  if (a.is_key) {
    constexpr int kW = (D + 31) / 32;
    for (int wd = 0; wd < kW; ++wd) {
      const int i = wd * 32 + lane;
      bool bit = false;
      if (i < D) {
        double acc = 0.0;
        const float* row = a.S + static_cast<int64_t>(i) * D;
        for (int j = 0; j < D; ++j) acc = fma(static_cast<double>(__ldg(row + j)), yd[j], acc);
        bit = acc >= 0.0;
      }
      const uint32_t word = __ballot_sync(0xffffffffu, bit);
      if (lane == 0) a.sign[v * kW + wd] = word;
    }
    if (lane == 0) a.rnorm[v] = static_cast<float>(rnrm);
  }
  __syncwarp();
}

template <int D>
__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kThreads / kWarp;
  constexpr int kW = (D + 31) / 32;
  const int nc = 1 << a.bits, nb = nc - 1;
  if (threadIdx.x < nc) s.cent[threadIdx.x] = a.cent[threadIdx.x];
  if (threadIdx.x < nb) s.bnd[threadIdx.x] = a.bnd[threadIdx.x];
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.d_status) {
    for (int j = 1; j < nb; ++j)
      if (!(s.bnd[j] > s.bnd[j - 1])) atomicOr(a.d_status, TQ_DEV_BAD_CODEBOOK);
  }
  const bool rope = a.pos != nullptr && a.rope_base > 0.0;
  const int64_t n_tiles = (a.n + kTV - 1) / kTV;
  __shared__ int row_ok[kTV];

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t v0 = tile * kTV;
    // 1. Load (and RoPE) the tile.
    for (int e = threadIdx.x; e < kTV * (D / 2); e += kThreads) {
      const int t = e / (D / 2), i = e % (D / 2);
      const int64_t v = v0 + t;
      float x0 = 0.f, x1 = 0.f;
      if (v < a.n) {
        const int64_t base = v * a.row_stride;
        x0 = load_elem(a.x, a.dtype, base + i);
        x1 = load_elem(a.x, a.dtype, base + i + D / 2);
        if (rope) {
          const int p = a.pos[v];
          if (p < 0 && a.d_status) atomicOr(a.d_status, TQ_DEV_BAD_POSITION);
          double sn, cs;
          sincos(rope_angle(p, i, D, a.rope_base), &sn, &cs);
          const double r0 = x0 * cs - x1 * sn, r1 = x0 * sn + x1 * cs;
          x0 = static_cast<float>(r0);
          x1 = static_cast<float>(r1);
        }
      }
      s.xs[t][i] = x0;
      s.xs[t][i + D / 2] = x1;
    }
    if (threadIdx.x < kTV) s.flag[threadIdx.x] = 0;
    __syncthreads();
    // 2. Norms (fp64 accumulation of the fp32 tile).
    for (int t = warp; t < kTV; t += kWarps) {
      double ss = 0.0;
      for (int j = lane; j < D; j += kWarp) ss += static_cast<double>(s.xs[t][j]) * s.xs[t][j];
      ss = warp_sum(ss);
      if (lane == 0) s.nrm[t] = static_cast<float>(sqrt(ss));
    }
    // 3. Y = Pi x' for each Pi group present in the tile.
    const int64_t last = (a.n < v0 + kTV ? a.n : v0 + kTV) - 1;
    const int64_t g_first = a.pi_stride ? v0 / a.vectors_per_pi : 0;
    const int64_t g_last = a.pi_stride ? last / a.vectors_per_pi : 0;
    for (int64_t g = g_first; g <= g_last; ++g) {
      __syncthreads();
      if (threadIdx.x < kTV) {
        const int64_t v = v0 + threadIdx.x;
        row_ok[threadIdx.x] = (v < a.n) && (a.pi_stride == 0 || v / a.vectors_per_pi == g);
      }
      tile_gemm<D>(s, s.xs, s.ys, a.Pi + g * a.pi_stride, row_ok);
    }
    __syncthreads();
    // 4. Bucketize, residual, norms (one warp per vector).
    for (int t = warp; t < kTV; t += kWarps) {
      const float nrm = s.nrm[t];
      const float band = kCodeGuard * nrm;
      bool close = false;
      float rs = 0.f;
      for (int i = lane; i < D; i += kWarp) {
        const float y = s.ys[t][i];
        int c = 0;
        for (int j = 0; j < nb; ++j) {
          const float th = nrm * s.bnd[j];
          c += (y > th) ? 1 : 0;
          close |= fabsf(y - th) <= band;
        }
        s.codes[t][i] = static_cast<uint8_t>(c);
        const float r = y - nrm * s.cent[c];
        s.ys[t][i] = r;
        rs = fmaf(r, r, rs);
      }
      rs = warp_sum(rs);
      const bool any = __any_sync(0xffffffffu, close);
      if (lane == 0) {
        s.rn[t] = sqrtf(rs);
        if (any) s.flag[t] = 1;
      }
    }
    // 5. Keys: P = S r and the sign bits.
    if (a.is_key) {
      __syncthreads();
      if (threadIdx.x < kTV) row_ok[threadIdx.x] = 1;
      tile_gemm<D>(s, s.ys, s.xs, a.S, row_ok);
      __syncthreads();
      for (int t = warp; t < kTV; t += kWarps) {
        const float band = kSignGuard * s.rn[t];
        bool close = false;
        for (int wd = 0; wd < kW; ++wd) {
          const int i = wd * 32 + lane;
          bool bit = false;
          if (i < D) {
            const float p = s.xs[t][i];
            bit = p >= 0.f;
            close |= fabsf(p) <= band;
          }
          const uint32_t word = __ballot_sync(0xffffffffu, bit);
          if (lane == 0) s.signs[t][wd] = word;
        }
        if (__any_sync(0xffffffffu, close) && lane == 0) s.flag[t] = 1;
      }
    }
    __syncthreads();
    // 6. Store every vector decided in fp32.
    const int rb = D * a.bits / 8;
    for (int t = warp; t < kTV; t += kWarps) {
      const int64_t v = v0 + t;
      if (v >= a.n || s.flag[t]) continue;
      uint8_t* irow = a.idx + v * rb;
      for (int g = lane; g < D / 8; g += kWarp) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) word |= static_cast<uint32_t>(s.codes[t][8 * g + j]) << (a.bits * j);
        for (int b = 0; b < a.bits; ++b) irow[g * a.bits + b] = static_cast<uint8_t>(word >> (8 * b));
      }
      if (lane == 0) a.norm[v] = s.nrm[t];
      if (a.is_key) {
        for (int wd = lane; wd < kW; wd += kWarp) a.sign[v * kW + wd] = s.signs[t][wd];
        if (lane == 0) a.rnorm[v] = s.rn[t];
      }
    }
    // 7. Recompute the flagged vectors in fp64.
    for (int t = warp; t < kTV; t += kWarps) {
      const int64_t v = v0 + t;
      if (v >= a.n || !s.flag[t]) continue;
      const int64_t g = a.pi_stride ? v / a.vectors_per_pi : 0;
      exact_vector<D>(a, s, v, a.Pi + g * a.pi_stride);
    }
    __syncthreads();
  }
}

template <int D>
cudaError_t launch(const QuantArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(Smem<D>);
  cudaError_t e = cudaFuncSetAttribute(quantize_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_kernel<D>, kThreads, smem);
  const int64_t tiles = (a.n + kTV - 1) / kTV;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, int64_t(sms) * std::max(1, per_sm))));
  quantize_kernel<D><<<grid, kThreads, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

// TQ_QUANTIZE_PATH selects a kernel where several apply (all compute the
// same planes; tests cover each): "cuda-core" the tiled CUDA-core kernel,
// "tensor-core" the tensor-core kernel where it applies (no exact small-call
// path), unset or anything else the default choice.
bool getenv_path(const char* name) {
  const char* e = std::getenv("TQ_QUANTIZE_PATH");
  return e != nullptr && std::strcmp(e, name) == 0;
}
bool getenv_force_cuda_core() { return getenv_path("cuda-core"); }

}  // namespace tq

extern "C" tq_status tq_quantize_kv(const tq_layout* layout, int32_t is_key, const void* x, tq_dtype x_dtype,
                                    int64_t n_vectors, int64_t row_stride, const int32_t* positions, float rope_base,
                                    const float* Pi, int64_t vectors_per_pi, int64_t pi_stride, const float* S,
                                    const float* centroids, const float* boundaries, const tq_planes* out,
                                    int32_t* d_status, void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_layout(layout);
  if (st != TQ_OK) return st;
  const int d = layout->d;
  const int bits = is_key ? layout->key_bits : layout->value_bits;
  if (n_vectors < 0) return fail(TQ_ERR_INVALID_ARG, "n_vectors < 0");
  if (n_vectors == 0) return TQ_OK;
  if (!x || !Pi || !centroids || !boundaries || !out || !out->idx || !out->norm)
    return fail(TQ_ERR_INVALID_ARG, "NULL input/output pointer");
  if (is_key && (!S || !out->sign || !out->rnorm)) return fail(TQ_ERR_INVALID_ARG, "keys need S, sign and rnorm");
  if (x_dtype != TQ_F32 && x_dtype != TQ_BF16) return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_F32 or TQ_BF16");
  if (row_stride < d) return fail(TQ_ERR_INVALID_ARG, "row_stride (%lld) < d (%d)", (long long)row_stride, d);
  if (pi_stride < 0 || (pi_stride > 0 && vectors_per_pi < 1))
    return fail(TQ_ERR_INVALID_ARG, "pi_stride < 0 or vectors_per_pi < 1");
  if (!aligned(Pi, 16) || (S && !aligned(S, 16)) || (pi_stride % 4) != 0)
    return fail(TQ_ERR_INVALID_ARG, "Pi/S must be 16-byte aligned (pi_stride a multiple of 4)");
  QuantArgs a{x, x_dtype == TQ_F32 ? 0 : 1, n_vectors, row_stride, positions, static_cast<double>(rope_base),
              Pi, vectors_per_pi, pi_stride, S, centroids, boundaries, bits, is_key ? 1 : 0,
              out->idx, is_key ? out->sign : nullptr, out->norm, is_key ? out->rnorm : nullptr, d_status};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool rope = positions != nullptr && rope_base > 0.f;
  // Few vectors and one shared Pi: the exact one-CTA-per-vector kernel (a
  // tile kernel would run on a handful of SMs). TQ_QUANTIZE_PATH=cuda-core
  // keeps such calls on the tiled CUDA-core kernel.
  if (!getenv_force_cuda_core() && !getenv_path("tensor-core") && n_vectors <= kExactMaxVectors && pi_stride == 0 &&
      (d == 64 || d == 128 || d == 200) && aligned(Pi, 16) && (!S || aligned(S, 16))) {
    cudaError_t e = append_quantize(d, bits, is_key != 0, x, x_dtype == TQ_F32 ? 0 : 1, n_vectors, row_stride,
                                    positions, rope_base, Pi, S, centroids, boundaries, out, d_status, s);
    if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_quantize_kv launch: %s", cudaGetErrorString(e));
    return TQ_OK;
  }
  if (!getenv_force_cuda_core() && tc_quantize_supported(d, x_dtype, rope, vectors_per_pi, pi_stride, x, row_stride))
    return tc_quantize(d, is_key != 0, bits, x, n_vectors, row_stride, Pi, vectors_per_pi, pi_stride, S, centroids,
                       boundaries, out, d_status, s);
  cudaError_t e;
  switch (d) {
    case 64: e = launch<64>(a, s); break;
    case 128: e = launch<128>(a, s); break;
    case 200: e = launch<200>(a, s); break;
    default: return fail(TQ_ERR_UNSUPPORTED, "tq_quantize_kv: d=%d not built (64, 128, 200)", d);
  }
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tq_quantize_kv launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

