// Tensor-core quantiser (sm_100a, tcgen05) for bf16 inputs, d in {64, 128},
// one shared Pi, no RoPE (the post-RoPE K/V of the ESM- and Llama-shaped
// caches). Computes exactly what tq_quantize_kv specifies; codes and signs are
// those of exact arithmetic (see "Exactness").
//
// Sources: 7minutos.es "KV cache ... TurboQuant" Etapa 1 (y = Pi x, Lloyd-Max
// index per coordinate of y/||x||) and Etapa 2 (sign of S times the residual,
// residual norm); gist.science "TurboESM ..." section 2A (RoPE before Pi).
//
// Per CTA (persistent, one per SM), tiles of 128 vectors:
//   warp 0      TMA: 128 x d bf16 tile -> shared memory (128-byte swizzle)
//   warp 1      MMA issuer (one thread) + TMEM owner:
//                 Y = X (Pi1 + Pi2 + Pi3)^T        3 chains, A/B in smem
//                 P = (R1 + R2) (S1 + S2)^T         R1S1 + R1S2 + R2S1, A in TMEM
//               Pi = Pi1+Pi2+Pi3 and S = S1+S2 are bf16 splits made in the
//               prologue; x is bf16, so X Pi_t^T is exact per product and only
//               the fp32 accumulation rounds.
//   warps 2-9   epilogue, two warpgroups splitting the d columns: norms from
//               the smem tile, codes by binary search on ||x|| t_j, residual r
//               (fp32 kept in TMEM, bf16 splits R1/R2 for the second MMA), sign
//               bits, packing and stores.
// TMEM: Y/P double buffer (2d columns), R1|R2 (d), r fp32 (d).
//
// Exactness. A code is decided in fp32 only when y is farther than
// 3e-6 ||x|| from every boundary it was compared with; otherwise that
// coordinate's y is recomputed in fp64 from x and Pi (warp-cooperative) and
// the code decided there. A sign is decided from the MMA only when
// |p| > 1e-4 ||r||; otherwise p is recomputed in fp64 from the fp32 residual,
// and if that value is within 1e-5 ||r|| of zero, from a residual rebuilt
// entirely in fp64 (every coordinate of the row, one lane per coordinate).
//
// Every wait is bounded (2 s); a timeout sets TQ_DEV_TIMEOUT in *d_status and
// the CTA drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_sm100.cuh"
#include "tq_tc.h"

namespace tq {
namespace {

using namespace sm100;
using dev::warp_sum;

constexpr int kThreads = 320;         // 10 warps
// Guard bands. The fp32 accumulation of the 3-way split rotation errs by
// ~1e-7 ||x|| per coordinate (std), the 2x2-way split projection by ~3e-6 ||r||,
// and the fp32 residual moves an fp64 projection by ~5e-7 ||r||: each band is
// more than 20 standard deviations of the error it covers.
constexpr float kCodeGuard = 3e-6f;
constexpr float kSignGuard = 1e-4f;
constexpr double kSignGuard2 = 1e-5;

template <int D, bool KEY>
struct Cfg {
  static constexpr int kM = 128;
  static constexpr int kKSteps = D / 16;
  static constexpr int kTileBytes = kM * D * 2;
  static constexpr int kMatBytes = D * D * 2;
  static constexpr int kStages = (KEY && D == 128) ? 1 : (D == 128 ? 3 : 4);
  static constexpr int kSSplits = KEY ? 2 : 0;
  static constexpr int kColY = 0;                    // buffers at 0 and D
  static constexpr int kColR1 = 2 * D;
  static constexpr int kColR2 = 2 * D + D / 2;
  static constexpr int kColR32 = 3 * D;
  static constexpr int kTmemCols = KEY ? 4 * D : 2 * D;
  static constexpr int kChunks = D / 32;             // 32-column chunks
  static constexpr int kChunksPerWg = kChunks / 2;
  // Shared memory plan (offsets from a 1024-aligned base).
  static constexpr int kOffPi = 0;
  static constexpr int kOffS = kOffPi + 3 * kMatBytes;
  static constexpr int kOffX = kOffS + kSSplits * kMatBytes;
  static constexpr int kOffBar = kOffX + kStages * kTileBytes;
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // misc: tmem base (4) + abort (4) + cent[16] + bnd[16] + nrm partials [2][128] double + rsq [2][128] float
  static constexpr int kOffCent = kOffMisc + 16;
  static constexpr int kOffBnd = kOffCent + 64;
  static constexpr int kOffNrm = kOffBnd + 64;
  static constexpr int kOffRsq = kOffNrm + 2 * 2 * kM * 8;     // norm partials double-buffered by tile parity
  static constexpr int kOffScratch = kOffRsq + 2 * kM * 4;   // 8 warps x 32 floats
  static constexpr int kSmemBytes = kOffScratch + 8 * 32 * 4 + 1024;   // + alignment slack
};

struct TcArgs {
  const __nv_bfloat16* x;
  int64_t n;
  int64_t row_stride;
  const float* Pi;
  const float* S;
  const float* cent;
  const float* bnd;
  uint8_t* idx;
  uint32_t* sign;
  float* norm;
  float* rnorm;
  int32_t* d_status;
};

// Barrier over the 256 epilogue threads that also ORs a predicate across them,
// so every epilogue warp takes the same abort decision.
__device__ __forceinline__ bool epi_sync_or(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, 1, 256, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p))
      : "memory");
  return r != 0;
}

// Splits v into bf16 terms hi (+ mid (+ lo)) that add up to v to ~2^-25.
__device__ __forceinline__ void split3(float v, __nv_bfloat16& a, __nv_bfloat16& b, __nv_bfloat16& c) {
  a = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(a);
  b = __float2bfloat16_rn(r1);
  c = __float2bfloat16_rn(r1 - __bfloat162float(b));
}

// Exact (fp64) y_i = Pi_i . x_row, warp-cooperative (all lanes call it).
template <int D>
__device__ __noinline__ double exact_y(const float* __restrict__ M, int i, const __nv_bfloat16* __restrict__ xrow) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
#pragma unroll
  for (int j = lane; j < D; j += 32)
    acc = fma(static_cast<double>(__ldg(M + i * D + j)), static_cast<double>(__bfloat162float(xrow[j])), acc);
  return warp_sum(acc);
}

// Exact code of y64 (zero vector: u = 0).
template <int NB>
__device__ __forceinline__ int exact_code(double y64, double nrm64, const float* bnd) {
  int c = 0;
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    const double tj = static_cast<double>(bnd[j]);
    c += (nrm64 > 0.0 ? (y64 > nrm64 * tj) : (0.0 > tj)) ? 1 : 0;
  }
  return c;
}

// p_i = S_i . r for the row held by lane L, with r the fp32 residual stored in
// TMEM columns [col_r, col_r + D) of each lane (warp-cooperative).
template <int D>
__device__ __noinline__ double p_from_tmem(const float* __restrict__ S, int i, int L, uint32_t lane_addr, uint32_t col_r) {
  const int lane = threadIdx.x & 31;
  double sv[D / 32];
#pragma unroll
  for (int c4 = 0; c4 < D / 32; ++c4) sv[c4] = static_cast<double>(__ldg(S + i * D + c4 * 32 + lane));
  double acc = 0.0;
#pragma unroll
  for (int c4 = 0; c4 < D / 32; ++c4) {
    uint32_t rr[32];
    tmem_ld32(lane_addr + col_r + c4 * 32, rr);
    tmem_ld_wait();
    float mine = 0.f;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float vL = __shfl_sync(0xffffffffu, __uint_as_float(rr[u]), L);
      if (lane == u) mine = vL;
    }
    acc = fma(sv[c4], static_cast<double>(mine), acc);
  }
  return warp_sum(acc);
}

// p_i with the residual of row xrow rebuilt in fp64: lane j' owns the
// coordinates j = j' + 32 m, computing y_j, its code and r_j exactly.
template <int D, int NB>
__device__ __noinline__ double p_rebuild(const float* __restrict__ Pi, const float* __restrict__ S, int i,
                                         const __nv_bfloat16* __restrict__ xrow, double nrm64, const float* bnd,
                                         const float* cent) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
#pragma unroll 1
  for (int m = 0; m < D / 32; ++m) {
    const int j = lane + 32 * m;
    double y = 0.0;
    const float4* row = reinterpret_cast<const float4*>(Pi + j * D);
#pragma unroll 4
    for (int k4 = 0; k4 < D / 4; ++k4) {
      const float4 w = __ldg(row + k4);
      y = fma(static_cast<double>(w.x), static_cast<double>(__bfloat162float(xrow[4 * k4 + 0])), y);
      y = fma(static_cast<double>(w.y), static_cast<double>(__bfloat162float(xrow[4 * k4 + 1])), y);
      y = fma(static_cast<double>(w.z), static_cast<double>(__bfloat162float(xrow[4 * k4 + 2])), y);
      y = fma(static_cast<double>(w.w), static_cast<double>(__bfloat162float(xrow[4 * k4 + 3])), y);
    }
    const int c = exact_code<NB>(y, nrm64, bnd);
    const double r = y - nrm64 * static_cast<double>(cent[c]);
    acc = fma(static_cast<double>(__ldg(S + i * D + j)), r, acc);
  }
  return warp_sum(acc);
}

template <int D, bool KEY, int BITS>
__global__ void __launch_bounds__(kThreads, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap tmap, TcArgs a) {
  using C = Cfg<D, KEY>;
  constexpr int kNb = (1 << BITS) - 1;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* pi_s = sm + C::kOffPi;
  unsigned char* s_s = sm + C::kOffS;
  unsigned char* x_s = sm + C::kOffX;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* yfull = bars + 2 * C::kStages;          // [2]
  uint64_t* accfree = yfull + 2;                      // [2]
  uint64_t* rfull = accfree + 2;                      // [1]
  uint64_t* pfull = rfull + 1;                        // [2]
  uint64_t* drain = pfull + 2;                        // [1] final MMA drain
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);
  float* cent_s = reinterpret_cast<float*>(sm + C::kOffCent);
  float* bnd_s = reinterpret_cast<float*>(sm + C::kOffBnd);
  double* nrm_part = reinterpret_cast<double*>(sm + C::kOffNrm);
  float* rsq_part = reinterpret_cast<float*>(sm + C::kOffRsq);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (a.n + C::kM - 1) / C::kM;

  // ---------------------------------------------------------------- prologue
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&yfull[b], 1);
      mbar_init(&accfree[b], 8);
      mbar_init(&pfull[b], 1);
    }
    mbar_init(rfull, 8);
    mbar_init(drain, 1);
    *abort_s = 0;
    mbar_fence_init();
  }
  if (tid < 16) cent_s[tid] = tid <= kNb ? a.cent[tid] : 0.f;
  if (tid < 16) bnd_s[tid] = tid < kNb ? a.bnd[tid] : 0.f;
  if (warp == 1) {
    tmem_alloc(tmem_base_s, C::kTmemCols);
    tmem_relinquish();
  }
  // bf16 splits of Pi (3) and S (2) in the K-major 128B-swizzled layout.
  for (int e = tid; e < D * D; e += kThreads) {
    const int i = e / D, j = e % D;
    const uint32_t off = sw128_offset(i, j, D);
    __nv_bfloat16 h, m, l;
    split3(__ldg(a.Pi + e), h, m, l);
    *reinterpret_cast<__nv_bfloat16*>(pi_s + off) = h;
    *reinterpret_cast<__nv_bfloat16*>(pi_s + C::kMatBytes + off) = m;
    *reinterpret_cast<__nv_bfloat16*>(pi_s + 2 * C::kMatBytes + off) = l;
    if (KEY) {
      split3(__ldg(a.S + e), h, m, l);
      *reinterpret_cast<__nv_bfloat16*>(s_s + off) = h;
      *reinterpret_cast<__nv_bfloat16*>(s_s + C::kMatBytes + off) = m;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;
  if (blockIdx.x == 0 && tid == 0 && a.d_status) {
    for (int j = 1; j < kNb; ++j)
      if (!(bnd_s[j] > bnd_s[j - 1])) atomicOr(a.d_status, TQ_DEV_BAD_CODEBOOK);
  }

  auto fail = [&]() {
    *abort_s = 1;
    if (a.d_status) atomicOr(a.d_status, TQ_DEV_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int it = 0;
      int armed[C::kStages > 0 ? C::kStages : 1];
      for (int s = 0; s < C::kStages; ++s) armed[s] = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
        const int st = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (*abort_s) break;
        if (!mbar_wait(&empty[st], ph ^ 1)) { fail(); break; }
        mbar_expect_tx(&full[st], C::kTileBytes);
        unsigned char* dst = x_s + st * C::kTileBytes;
#pragma unroll
        for (int k = 0; k < D / 64; ++k) tma_load_2d(dst + k * C::kM * 128, &tmap, &full[st], k * 64, int(t * C::kM));
        armed[st] = it + 1;
      }
      // Never leave a copy in flight: wait for the last load of every stage.
      for (int s = 0; s < C::kStages; ++s) {
        if (armed[s]) mbar_wait(&full[s], ((armed[s] - 1) / C::kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, D);
      const uint32_t pi_base = smem_u32(pi_s), s_base = smem_u32(s_s), x_base = smem_u32(x_s);
      // Descriptors differ only in the start-address field (low 14 bits,
      // address >> 4): build the bases once, add constant offsets per K-step.
      const uint64_t pi_desc0 = desc_k_sw128(pi_base), s_desc0 = desc_k_sw128(s_base), x_desc0 = desc_k_sw128(x_base);
      auto issue_y = [&](int it) {
        const int st = it % C::kStages;
        const int b = it & 1;
        const uint32_t d_tmem = tmem + C::kColY + b * D;
        const uint64_t xa = x_desc0 + static_cast<uint64_t>((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int sp = 0; sp < 3; ++sp) {
#pragma unroll
          for (int k = 0; k < C::kKSteps; ++k) {
            constexpr int kAtomA = 128 * 128, kAtomB = D * 128;
            const uint64_t ad = xa + static_cast<uint64_t>(((k >> 2) * kAtomA + (k & 3) * 32) >> 4);
            const uint64_t bd = pi_desc0 + static_cast<uint64_t>((sp * C::kMatBytes + (k >> 2) * kAtomB + (k & 3) * 32) >> 4);
            umma_ss(d_tmem, ad, bd, kIdesc, (sp | k) != 0);
          }
        }
        umma_commit(&yfull[b]);
      };
      auto issue_p = [&](int it) {
        const int b = it & 1;
        const uint32_t d_tmem = tmem + C::kColY + b * D;
        // (A, B) pairs: R1 S1, R1 S2, R2 S1.
#pragma unroll
        for (int pr = 0; pr < 3; ++pr) {
          const uint32_t acol = (pr == 2) ? C::kColR2 : C::kColR1;
          const int boff = (pr == 1) ? C::kMatBytes : 0;
#pragma unroll
          for (int k = 0; k < C::kKSteps; ++k) {
            constexpr int kAtomB = D * 128;
            const uint64_t bd = s_desc0 + static_cast<uint64_t>((boff + (k >> 2) * kAtomB + (k & 3) * 32) >> 4);
            umma_ts(d_tmem, tmem + acol + k * 8, bd, kIdesc, (pr | k) != 0);
          }
        }
        umma_commit(&pfull[b]);
      };
      // Issue whatever is ready: Y of the next tile (its X landed and its
      // accumulator buffer is free) and, for keys, P of the oldest tile whose
      // residual is in TMEM. Neither waits behind the other.
      const int my_tiles = (n_tiles > blockIdx.x) ? static_cast<int>((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
      int ny = 0, np = 0;
      uint64_t last = globaltimer_ns();
      while (KEY ? (np < my_tiles) : (ny < my_tiles)) {
        if (*abort_s) break;
        bool progress = false;
        if (ny < my_tiles) {
          const int st = ny % C::kStages;
          const uint32_t ph = (ny / C::kStages) & 1;
          const uint32_t bph = (ny >> 1) & 1;
          if (mbar_try_wait(&full[st], ph) && mbar_try_wait(&accfree[ny & 1], bph ^ 1)) {
            tc_fence_after();
            issue_y(ny);
            ++ny;
            progress = true;
          }
        }
        if (KEY && np < ny && mbar_try_wait(rfull, np & 1)) {
          tc_fence_after();
          issue_p(np);
          ++np;
          progress = true;
        }
        if (progress) {
          last = globaltimer_ns();
        } else if (globaltimer_ns() - last > 2000000000ull) {
          fail();
          break;
        }
      }
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int ew = warp - 2;                 // 0..7
    const int g = ew >> 2;                   // column half
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;           // row within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float th[kNb > 0 ? kNb : 1];
    int it = 0;
    for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
      const int st = it % C::kStages;
      const uint32_t ph = (it / C::kStages) & 1;
      const int b = it & 1;
      const uint32_t bph = (it >> 1) & 1;
      const int64_t v = t * C::kM + row;
      const bool valid = v < a.n;
      // ||x||^2 from the shared tile (this warpgroup's half of x).
      bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], ph));
      {
        const unsigned char* xt = x_s + st * C::kTileBytes;
        double ss = 0.0;
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) {
          const int k0 = g * (D / 2) + cc * 8;
          const uint4 w = *reinterpret_cast<const uint4*>(xt + sw128_offset(row, k0, C::kM));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float lo = __uint_as_float(ws[h] << 16), hi = __uint_as_float(ws[h] & 0xffff0000u);
            ss += static_cast<double>(lo * lo) + static_cast<double>(hi * hi);
          }
        }
        nrm_part[((it & 1) * 2 + g) * C::kM + row] = ss;
      }
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&yfull[b], bph));
      tc_fence_after();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);     // X tile no longer needed
      if (!ok && lane == 0) fail();
      if (epi_sync_or(!ok || *abort_s != 0)) break;
      const double nrm64 = sqrt(nrm_part[(it & 1) * 2 * C::kM + row] + nrm_part[((it & 1) * 2 + 1) * C::kM + row]);
      const float nrm = static_cast<float>(nrm64);
      const float band = kCodeGuard * nrm;
#pragma unroll
      for (int j = 0; j < kNb; ++j) th[j] = nrm * bnd_s[j];

      uint32_t codew[C::kChunksPerWg][BITS];
      float rsq = 0.f;
#pragma unroll
      for (int cc = 0; cc < C::kChunksPerWg; ++cc) {
        const int ch = g * C::kChunksPerWg + cc;
        uint32_t ybits[32];
        tmem_ld32(lane_addr + C::kColY + b * D + ch * 32, ybits);
        tmem_ld_wait();
        int code[32];
        float r[32];
        uint32_t flags = 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float y = __uint_as_float(ybits[k]);
          int c;
          float dmin;
          if (BITS == 3) {
            const bool b2 = y > th[3];
            const float tA = b2 ? th[5] : th[1];
            const bool b1 = y > tA;
            const float tB = b2 ? (b1 ? th[6] : th[4]) : (b1 ? th[2] : th[0]);
            const bool b0 = y > tB;
            c = (b2 ? 4 : 0) + (b1 ? 2 : 0) + (b0 ? 1 : 0);
            dmin = fminf(fabsf(y - th[3]), fminf(fabsf(y - tA), fabsf(y - tB)));
          } else {
            c = 0;
            dmin = INFINITY;
#pragma unroll
            for (int j = 0; j < kNb; ++j) {
              c += (y > th[j]) ? 1 : 0;
              dmin = fminf(dmin, fabsf(y - th[j]));
            }
          }
          if (dmin <= band) flags |= 1u << k;
          code[k] = c;
          r[k] = fmaf(-nrm, cent_s[c], y);
        }
        if (!valid) flags = 0;
        // Exact fp64 decision for every coordinate near a boundary: one
        // (lane, coordinate) at a time, the whole warp computing its dot product.
#pragma unroll 1
        for (unsigned m = __ballot_sync(0xffffffffu, flags != 0u); m != 0u;
             m = __ballot_sync(0xffffffffu, flags != 0u)) {
          const int L = __ffs(m) - 1;
          const int kL = __ffs(__shfl_sync(0xffffffffu, flags, L)) - 1;
          const int64_t vL = __shfl_sync(0xffffffffu, v, L);
          const double y64 = exact_y<D>(a.Pi, ch * 32 + kL, a.x + vL * a.row_stride);
          if (lane == L) {
            const int c = exact_code<kNb>(y64, nrm64, bnd_s);
            const float rr = static_cast<float>(y64 - nrm64 * static_cast<double>(cent_s[c]));
            flags &= ~(1u << kL);
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k == kL) {
                code[k] = c;
                r[k] = rr;
              }
          }
        }
        // Pack this chunk's codes (32 codes -> BITS words).
#pragma unroll
        for (int w = 0; w < BITS; ++w) codew[cc][w] = 0u;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int bp = k * BITS;
          codew[cc][bp >> 5] |= static_cast<uint32_t>(code[k]) << (bp & 31);
          if ((bp & 31) + BITS > 32) codew[cc][(bp >> 5) + 1] |= static_cast<uint32_t>(code[k]) >> (32 - (bp & 31));
        }
        if (KEY) {
          uint32_t r1[16], r2[16], rb[32];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            rsq = fmaf(r[k], r[k], fmaf(r[k + 1], r[k + 1], rsq));
            const __nv_bfloat162 h = __floats2bfloat162_rn(r[k], r[k + 1]);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 l = __floats2bfloat162_rn(r[k] - hf.x, r[k + 1] - hf.y);
            r1[k / 2] = *reinterpret_cast<const uint32_t*>(&h);
            r2[k / 2] = *reinterpret_cast<const uint32_t*>(&l);
            rb[k] = __float_as_uint(r[k]);
            rb[k + 1] = __float_as_uint(r[k + 1]);
          }
          tmem_st16(lane_addr + C::kColR1 + ch * 16, r1);
          tmem_st16(lane_addr + C::kColR2 + ch * 16, r2);
          tmem_st32(lane_addr + C::kColR32 + ch * 32, rb);
        }
      }
      // Stores of this warpgroup's part of the row.
      if (valid) {
        constexpr int kRowBytes = D * BITS / 8;
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.idx + v * kRowBytes) + g * C::kChunksPerWg * BITS;
#pragma unroll
        for (int cc = 0; cc < C::kChunksPerWg; ++cc)
#pragma unroll
          for (int w = 0; w < BITS; ++w) dst[cc * BITS + w] = codew[cc][w];
        if (g == 0) a.norm[v] = nrm;
      }
      if (!KEY) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accfree[b]);
        continue;
      }
      tmem_st_wait();
      tc_fence_before();
      rsq_part[g * C::kM + row] = rsq;
      __syncwarp();
      if (lane == 0) mbar_arrive(rfull);
      if (epi_sync_or(*abort_s != 0)) break;
      const float rn = sqrtf(rsq_part[row] + rsq_part[C::kM + row]);
      // On a timeout the loop ends at the next iteration's barrier; results of
      // this tile are then meaningless and *d_status says so.
      if (!__all_sync(0xffffffffu, mbar_wait(&pfull[b], bph)) && lane == 0) fail();
      tc_fence_after();
      const float sband = kSignGuard * rn;
#pragma unroll
      for (int cc = 0; cc < C::kChunksPerWg; ++cc) {
        const int ch = g * C::kChunksPerWg + cc;
        uint32_t pbits[32];
        tmem_ld32(lane_addr + C::kColY + b * D + ch * 32, pbits);
        tmem_ld_wait();
        uint32_t word = 0, flags = 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p = __uint_as_float(pbits[k]);
          word |= (p >= 0.f ? 1u : 0u) << k;
          if (fabsf(p) <= sband) flags |= 1u << k;
        }
        if (!valid) flags = 0;
        // fp64 recomputation of p_i = S_i . r for signs near zero.
#pragma unroll 1
        for (unsigned m = __ballot_sync(0xffffffffu, flags != 0u); m != 0u;
             m = __ballot_sync(0xffffffffu, flags != 0u)) {
          const int L = __ffs(m) - 1;
          const int kL = __ffs(__shfl_sync(0xffffffffu, flags, L)) - 1;
          const int i = ch * 32 + kL;
          const double p1 = p_from_tmem<D>(a.S, i, L, lane_addr, C::kColR32);
          const float rnL = __shfl_sync(0xffffffffu, rn, L);
          bool bit = p1 >= 0.0;
          if (fabs(p1) <= kSignGuard2 * rnL) {
            const int64_t vL = __shfl_sync(0xffffffffu, v, L);
            const double nL = __shfl_sync(0xffffffffu, nrm64, L);
            bit = p_rebuild<D, kNb>(a.Pi, a.S, i, a.x + vL * a.row_stride, nL, bnd_s, cent_s) >= 0.0;
          }
          if (lane == L) {
            word = bit ? (word | (1u << kL)) : (word & ~(1u << kL));
            flags &= ~(1u << kL);
          }
        }
        if (valid) a.sign[v * C::kChunks + ch] = word;
      }
      if (valid && g == 0) a.rnorm[v] = rn;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accfree[b]);
    }
  }

  // ------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    // Every MMA this CTA issued must have completed before TMEM is released.
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// --------------------------------------------------------------------- host
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

template <int D, bool KEY, int BITS>
cudaError_t launch_tc(const TcArgs& a, const CUtensorMap& map, cudaStream_t st) {
  using C = Cfg<D, KEY>;
  static_assert(C::kSmemBytes <= 232448, "shared memory plan exceeds 227 KB");
  cudaError_t e = cudaFuncSetAttribute(quantize_tc_kernel<D, KEY, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (a.n + 127) / 128;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  quantize_tc_kernel<D, KEY, BITS><<<grid, kThreads, C::kSmemBytes, st>>>(map, a);
  return cudaGetLastError();
}

template <int D, bool KEY>
cudaError_t launch_bits(int bits, const TcArgs& a, const CUtensorMap& map, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_tc<D, KEY, 2>(a, map, st);
    case 3: return launch_tc<D, KEY, 3>(a, map, st);
    default: return launch_tc<D, KEY, 4>(a, map, st);
  }
}

}  // namespace

bool tc_quantize_supported(int d, int x_dtype, bool rope, int64_t pi_stride, const void* x, int64_t row_stride) {
  if (!(d == 64 || d == 128)) return false;
  if (x_dtype != TQ_BF16 || rope || pi_stride != 0) return false;
  if (!aligned(x, 16) || (row_stride * 2) % 16 != 0) return false;
  return encode_fn() != nullptr;
}

tq_status tc_quantize(int d, bool is_key, int bits, const void* x, int64_t n, int64_t row_stride, const float* Pi,
                      const float* S, const float* cent, const float* bnd, const tq_planes* out, int32_t* d_status,
                      cudaStream_t st) {
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode_fn()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  TcArgs a{static_cast<const __nv_bfloat16*>(x), n, row_stride, Pi, S, cent, bnd, out->idx,
           is_key ? out->sign : nullptr, out->norm, is_key ? out->rnorm : nullptr, d_status};
  cudaError_t e;
  if (d == 128)
    e = is_key ? launch_bits<128, true>(bits, a, map, st) : launch_bits<128, false>(bits, a, map, st);
  else
    e = is_key ? launch_bits<64, true>(bits, a, map, st) : launch_bits<64, false>(bits, a, map, st);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "tensor-core quantize launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace tq
