// Device helpers shared by the CUDA translation units of libtq.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tq {
namespace dev {

constexpr int kWarp = 32;
// sqrt(pi/2): the QJL estimator's scale is sqrt(pi/2)/d (7minutos.es, Etapa 2).
constexpr double kSqrtHalfPi = 1.2533141373155002512;

__device__ __forceinline__ float load_elem(const void* base, int dtype, int64_t i) {
  if (dtype == 0) return __ldg(reinterpret_cast<const float*>(base) + i);
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Rotate-half RoPE angle for pair i of a d-dimensional vector at `pos`,
// in double precision: pos * base^(-2i/d).
__device__ __forceinline__ double rope_angle(int pos, int i, int d, double base) {
  return static_cast<double>(pos) * pow(base, -2.0 * i / d);
}

// Extracts code `i` (bits wide) from a packed index row (little-endian groups
// of 8 codes in `bits` bytes).
__device__ __forceinline__ int get_code(const uint8_t* row, int i, int bits) {
  const int bit = i * bits;
  const int byte = bit >> 3;
  const int sh = bit & 7;
  unsigned w = row[byte];
  if (sh + bits > 8) w |= static_cast<unsigned>(row[byte + 1]) << 8;
  return (w >> sh) & ((1u << bits) - 1u);
}

}  // namespace dev
}  // namespace tq
